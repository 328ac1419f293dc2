// token_step.cuh -- short causal calls (a few tokens), token by token on the
// CUDA cores.
//
// For a call of a few tokens the chunked path's fixed cost (a chunk prep task,
// then the chain's first step) is most of the time.  This kernel walks the
// tokens directly with the state slice in registers.  With S = S_{t-1}:
//   p = S^T k_t,   r = S^T q_t,   kq = k_t . q_t
//   S_t = alpha_t S + k_t (beta_t (v_t - alpha_t p))^T
//   o_t = S_t^T q_t = alpha_t r + kq beta_t (v_t - alpha_t p)
// which is S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T with
// the products taken apart.  Every value is fp32.
//
// Grid (DV / 32, B * H), block 256 (8 warps).  Thread (warp w, lane j) holds
// column j of its CTA's 32-column slice, rows w, w + 8, ..., so p and r are a
// sum over the 8 warps of one partial each: one barrier per token (the
// partials are double-buffered).  The call's k, q (fp32), its v slice, kq and
// the gates are staged in shared memory first, with every load in flight at
// once.
#pragma once

#include "common.cuh"

namespace gdn {
namespace tok {

constexpr int kCols = 32;      // state columns per CTA
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxT = 64;      // longest call this kernel takes

template <int DK>
struct TokSmem {
    static constexpr int kK = 0;                              // [kMaxT][DK] fp32
    static constexpr int kQ = kK + kMaxT * DK * 4;            // [kMaxT][DK]
    static constexpr int kV = kQ + kMaxT * DK * 4;            // [kMaxT][kCols]
    static constexpr int kA = kV + kMaxT * kCols * 4;         // alpha [kMaxT]
    static constexpr int kB = kA + kMaxT * 4;                 // beta
    static constexpr int kKQ = kB + kMaxT * 4;                // k . q
    static constexpr int kRed = kKQ + kMaxT * 4;              // [2][2][kWarps][kCols]
    static constexpr int kBytes = kRed + 2 * 2 * kWarps * kCols * 4;
};

template <int DK, int DV, typename Tin, typename Tout>
__global__ void __launch_bounds__(kThreads)
token_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
             const float *__restrict__ alpha, const float *__restrict__ beta,
             const float *__restrict__ state_in, float *__restrict__ state_out, Tout *__restrict__ o,
             int T, int H)
{
    using SM = TokSmem<DK>;
    constexpr int RPT = DK / kWarps;   // rows per thread
    extern __shared__ __align__(16) unsigned char smem[];
    float *ks = reinterpret_cast<float *>(smem + SM::kK);
    float *qs = reinterpret_cast<float *>(smem + SM::kQ);
    float *vs = reinterpret_cast<float *>(smem + SM::kV);
    float *as = reinterpret_cast<float *>(smem + SM::kA);
    float *bs = reinterpret_cast<float *>(smem + SM::kB);
    float *kqs = reinterpret_cast<float *>(smem + SM::kKQ);
    float *red = reinterpret_cast<float *>(smem + SM::kRed);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.y, b = bh / H, h = bh % H;
    const int j = blockIdx.x * kCols + lane;

    // ---- stage the call's inputs: [B, T, H, d] rows (b, t, h)
    for (int e = tid; e < T * DK; e += kThreads) {
        const int t = e / DK, i = e % DK;
        const size_t row = ((size_t)b * T + t) * H + h;
        ks[e] = to_f32(k[row * DK + i]);
        qs[e] = to_f32(q[row * DK + i]);
    }
    for (int e = tid; e < T * kCols; e += kThreads) {
        const int t = e / kCols, c = e % kCols;
        vs[e] = to_f32(v[(((size_t)b * T + t) * H + h) * DV + blockIdx.x * kCols + c]);
    }
    for (int t = tid; t < T; t += kThreads) {
        const size_t g = ((size_t)b * T + t) * H + h;
        as[t] = alpha[g];
        bs[t] = beta[g];
    }
    float S[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m)
        S[m] = state_in ? state_in[((size_t)bh * DK + warp + kWarps * m) * DV + j] : 0.f;
    __syncthreads();
    // k . q per token, one warp per token
    for (int t = warp; t < T; t += kWarps) {
        float s = 0.f;
        for (int i = lane; i < DK; i += 32) s = fmaf(ks[t * DK + i], qs[t * DK + i], s);
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) s += __shfl_xor_sync(0xffffffffu, s, d);
        if (lane == 0) kqs[t] = s;
    }
    __syncthreads();

    // ---- the tokens
    for (int t = 0; t < T; ++t) {
        const float *kt = ks + t * DK, *qt = qs + t * DK;
        float *rb = red + (t & 1) * 2 * kWarps * kCols;
        // this token's scalars, read before the barrier so they are in flight across it
        const float a = as[t], bt = bs[t], vj = vs[t * kCols + lane], kq = kqs[t];
        float kr[RPT];
        float pp[4] = {0.f, 0.f, 0.f, 0.f}, rr[4] = {0.f, 0.f, 0.f, 0.f};   // independent chains
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            kr[m] = kt[warp + kWarps * m];
            pp[m & 3] = fmaf(S[m], kr[m], pp[m & 3]);
            rr[m & 3] = fmaf(S[m], qt[warp + kWarps * m], rr[m & 3]);
        }
        rb[warp * kCols + lane] = (pp[0] + pp[1]) + (pp[2] + pp[3]);
        rb[(kWarps + warp) * kCols + lane] = (rr[0] + rr[1]) + (rr[2] + rr[3]);
        __syncthreads();
        float p0 = 0.f, p1 = 0.f, r0 = 0.f, r1 = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; w += 2) {
            p0 += rb[w * kCols + lane];
            p1 += rb[(w + 1) * kCols + lane];
            r0 += rb[(kWarps + w) * kCols + lane];
            r1 += rb[(kWarps + w + 1) * kCols + lane];
        }
        const float p = p0 + p1, r = r0 + r1;
        const float u = bt * (vj - a * p);   // beta (v - alpha p)
        if (warp == 0) o[(((size_t)b * T + t) * H + h) * DV + j] = from_f32<Tout>(fmaf(kq, u, a * r));
#pragma unroll
        for (int m = 0; m < RPT; ++m) S[m] = fmaf(a, S[m], kr[m] * u);
    }

    if (state_out) {
#pragma unroll
        for (int m = 0; m < RPT; ++m) state_out[((size_t)bh * DK + warp + kWarps * m) * DV + j] = S[m];
    }
}

}  // namespace tok
}  // namespace gdn
