// readout.cuh -- readout epilogue of the linear branch: one pass over the
// scan's output o and the content-dependent gate z,
//   y = o / sqrt(mean_j o_j^2 + eps) * gamma * sigmoid(z)
// per (b, t, h) row of d_v channels (the RMS norm runs over one head of one
// token, the gate multiplies the normalised readout).
//
// HBM-bound: one warp per row, each lane a run of d_v/32 consecutive channels
// read and written with one vector access per tensor; the sum of squares is a
// warp shuffle reduction.  A persistent grid (a few CTAs per SM) strides over
// the rows.  y may be o itself (same dtype): a row is read in full before it
// is written, by the same warp.
#pragma once

#include "common.cuh"

namespace gdn {
namespace rd {

constexpr int kThreads = 256;

template <typename T, int N> struct Vec;
template <> struct Vec<float, 2> { using type = float2; };
template <> struct Vec<float, 4> { using type = float4; };
template <> struct Vec<__nv_bfloat16, 2> { using type = unsigned int; };
template <> struct Vec<__nv_bfloat16, 4> { using type = uint2; };

template <typename T, int N>
__device__ __forceinline__ void load_run(const T *p, float (&x)[N]) {
    const typename Vec<T, N>::type v = *reinterpret_cast<const typename Vec<T, N>::type *>(p);
    const T *e = reinterpret_cast<const T *>(&v);
#pragma unroll
    for (int i = 0; i < N; ++i) x[i] = to_f32(e[i]);
}

template <typename T, int N>
__device__ __forceinline__ void store_run(T *p, const float (&x)[N]) {
    typename Vec<T, N>::type v;
    T *e = reinterpret_cast<T *>(&v);
#pragma unroll
    for (int i = 0; i < N; ++i) e[i] = from_f32<T>(x[i]);
    *reinterpret_cast<typename Vec<T, N>::type *>(p) = v;
}

template <int DV, typename To, typename Tz, typename Ty>
__global__ void __launch_bounds__(kThreads)
readout_kernel(const To *o, const Tz *z, const float *__restrict__ gamma, float eps, Ty *y, long long rows)
{
    constexpr int N = DV / 32;   // channels per lane
    const int lane = threadIdx.x & 31;
    const long long warps = (long long)gridDim.x * (kThreads / 32);
    float g[N];
#pragma unroll
    for (int i = 0; i < N; ++i) g[i] = gamma ? gamma[lane * N + i] : 1.f;
    for (long long r = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); r < rows; r += warps) {
        const size_t base = (size_t)r * DV + lane * N;
        float x[N], zz[N];
        load_run<To, N>(o + base, x);
        load_run<Tz, N>(z + base, zz);
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < N; ++i) ss = fmaf(x[i], x[i], ss);
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, d);
        const float inv = rsqrtf(ss * (1.f / DV) + eps);
        float out[N];
#pragma unroll
        for (int i = 0; i < N; ++i) out[i] = x[i] * inv * g[i] / (1.f + __expf(-zz[i]));
        store_run<Ty, N>(y + base, out);
    }
}

}  // namespace rd
}  // namespace gdn
