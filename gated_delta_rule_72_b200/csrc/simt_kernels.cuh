// simt_kernels.cuh -- chunkwise gated delta-net scan on CUDA cores, fp32.
//
// This is the full-precision path: every contraction is an fp32 FFMA, so
// fp32 inputs meet a 1e-4 (max-abs over rms) tolerance that TF32 or bf16
// tensor-core operands cannot.  It runs any supported shape and either dtype.
//
// Chunk algebra (chunk of C = 64 tokens in processing order r = 0..C-1,
// state S entering the chunk; the reverse pass processes a chunk back to
// front, which turns its recurrence into the forward one over reversed rows):
//   g_r   = sum_{m<=r} log alpha_m
//   L_rs  = beta_r e^{g_r - g_s} (k_r . k_s)            s < r
//   T     = (I + L)^{-1}                                 (unit lower triangular)
//   W     = T diag(beta e^g) K ,   U = T diag(beta) V
//   Delta = U - W S
//   O     = diag(dq) Q S + P Delta
//   S'    = ds S + (diag(dkk) K)^T Delta
// forward: dq_r = e^{g_r},  P_rs = e^{g_r - g_s} (q_r . k_s), s <= r
// reverse (strict readout, token r itself excluded):
//          dq_r = e^{g_{r-1}}, P_rs = e^{g_{r-1} - g_s} (q_r . k_s), s < r
// both:    dkk_s = e^{g_{C-1} - g_s},  ds = e^{g_{C-1}}
// Every exponent is a difference g_a - g_b with a >= b (or g_a alone), so it
// is <= 0 and the factors never overflow, whatever the gate range.
//
// Two kernels: prep (fully parallel over chunk x head x direction) writes the
// per-chunk operands to the workspace; chain (one CTA per head x direction x
// d_v slice) walks the chunks in order with its state slice in shared memory.
#pragma once

#include "common.cuh"

namespace gdn {
namespace simt {

// Per-chunk record written by prep_kernel, all fp32, in processing order:
//   W [C][DK] | Qh [C][DK] (= diag(dq) Q) | Kt [C][DK] (= diag(dkk) K)
//   U [C][DV] | P [C][C] | ds (padded to 4 floats)
template <int DK, int DV>
struct Record {
    static constexpr int kW = 0;
    static constexpr int kQ = kW + kChunk * DK;
    static constexpr int kK = kQ + kChunk * DK;
    static constexpr int kU = kK + kChunk * DK;
    static constexpr int kP = kU + kChunk * DV;
    static constexpr int kDs = kP + kChunk * kChunk;
    static constexpr int kFloats = kDs + 4;
};

template <int DK, int DV>
struct PrepSmem {
    static constexpr int kLdk = DK + 1;   // padded row strides (bank spread)
    static constexpr int kLdv = DV + 1;
    static constexpr int kLdc = kChunk + 1;
    static constexpr int kK = 0;
    static constexpr int kQ = kK + kChunk * kLdk;
    static constexpr int kV = kQ + kChunk * kLdk;
    static constexpr int kA = kV + kChunk * kLdv;     // K K^T, then L
    static constexpr int kB = kA + kChunk * kLdc;     // Q K^T
    static constexpr int kT = kB + kChunk * kLdc;     // (I+L)^{-1}
    static constexpr int kG = kT + kChunk * kLdc;     // g (C floats)
    static constexpr int kBeta = kG + kChunk;
    static constexpr int kWb = kBeta + kChunk;        // beta e^g (C floats)
    static constexpr int kFloats = kWb + kChunk;
    static constexpr size_t kBytes = sizeof(float) * kFloats;
};

// grid (nC, B*H, ndir), block 256.
template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(256)
prep_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
            const float* __restrict__ alpha, const float* __restrict__ beta,
            float* __restrict__ ws, int T, int H, int nC, int dir0)
{
    using SM = PrepSmem<DK, DV>;
    using RC = Record<DK, DV>;
    extern __shared__ float sm[];
    float* Ks = sm + SM::kK;
    float* Qs = sm + SM::kQ;
    float* Vs = sm + SM::kV;
    float* A = sm + SM::kA;
    float* Bq = sm + SM::kB;
    float* Tm = sm + SM::kT;
    float* g = sm + SM::kG;
    float* bt = sm + SM::kBeta;
    float* wb = sm + SM::kWb;

    const int c = blockIdx.x, bh = blockIdx.y, dir = dir0 + blockIdx.z;
    const int b = bh / H, h = bh % H;
    const int tid = threadIdx.x;

    // 1. rows in processing order; rows past the end are identity steps
    for (int idx = tid; idx < kChunk * DK; idx += blockDim.x) {
        const int r = idx / DK, d = idx % DK;
        const int t = token_of_row(c, r, dir);
        float kv = 0.f, qv = 0.f;
        if (t < T) {
            const size_t off = (((size_t)b * T + t) * H + h) * DK + d;
            kv = to_f32(k[off]);
            qv = to_f32(q[off]);
        }
        Ks[r * SM::kLdk + d] = kv;
        Qs[r * SM::kLdk + d] = qv;
    }
    for (int idx = tid; idx < kChunk * DV; idx += blockDim.x) {
        const int r = idx / DV, d = idx % DV;
        const int t = token_of_row(c, r, dir);
        Vs[r * SM::kLdv + d] = t < T ? to_f32(v[(((size_t)b * T + t) * H + h) * DV + d]) : 0.f;
    }
    if (tid < kChunk) {
        const int t = token_of_row(c, tid, dir);
        const size_t off = ((size_t)b * T + t) * H + h;
        g[tid] = t < T ? logf(alpha[off]) : 0.f;
        bt[tid] = t < T ? beta[off] : 0.f;
    }
    __syncthreads();
    if (tid == 0) {  // inclusive prefix sum of log alpha
        float acc = 0.f;
        for (int r = 0; r < kChunk; ++r) { acc += g[r]; g[r] = acc; }
    }
    // 2. Gram matrices K K^T and Q K^T
    for (int idx = tid; idx < kChunk * kChunk; idx += blockDim.x) {
        const int r = idx / kChunk, s = idx % kChunk;
        float akk = 0.f, aqk = 0.f;
        const float* kr = Ks + r * SM::kLdk;
        const float* qr = Qs + r * SM::kLdk;
        const float* ks = Ks + s * SM::kLdk;
#pragma unroll 8
        for (int d = 0; d < DK; ++d) {
            akk = fmaf(kr[d], ks[d], akk);
            aqk = fmaf(qr[d], ks[d], aqk);
        }
        A[r * SM::kLdc + s] = akk;
        Bq[r * SM::kLdc + s] = aqk;
    }
    __syncthreads();
    // 3. L (strictly lower) in place of K K^T; P (readout decay mask) in place of Q K^T
    for (int idx = tid; idx < kChunk * kChunk; idx += blockDim.x) {
        const int r = idx / kChunk, s = idx % kChunk;
        const float lv = s < r ? bt[r] * __expf(g[r] - g[s]) * A[r * SM::kLdc + s] : 0.f;
        A[r * SM::kLdc + s] = lv;
        float pv;
        if (dir == 0) pv = s <= r ? __expf(g[r] - g[s]) * Bq[r * SM::kLdc + s] : 0.f;
        else pv = s < r ? __expf(g[r - 1] - g[s]) * Bq[r * SM::kLdc + s] : 0.f;
        Bq[r * SM::kLdc + s] = pv;
    }
    if (tid < kChunk) wb[tid] = bt[tid] * __expf(g[tid]);
    __syncthreads();
    // 4. T = (I + L)^{-1} by forward substitution, one column per thread
    if (tid < kChunk) {
        const int j = tid;
        for (int r = 0; r < kChunk; ++r) {
            float val;
            if (r < j) val = 0.f;
            else if (r == j) val = 1.f;
            else {
                float acc = 0.f;
                for (int m = j; m < r; ++m) acc = fmaf(A[r * SM::kLdc + m], Tm[m * SM::kLdc + j], acc);
                val = -acc;
            }
            Tm[r * SM::kLdc + j] = val;
        }
    }
    __syncthreads();
    // 5. W, U, scaled Q and K, P, ds -> workspace record
    float* rec = ws + ((size_t)(dir * gridDim.y + bh) * nC + c) * RC::kFloats;
    const float gl = g[kChunk - 1];
    for (int idx = tid; idx < kChunk * DK; idx += blockDim.x) {
        const int r = idx / DK, d = idx % DK;
        float w = 0.f;
        for (int m = 0; m <= r; ++m)
            w = fmaf(Tm[r * SM::kLdc + m], wb[m] * Ks[m * SM::kLdk + d], w);
        rec[RC::kW + idx] = w;
        const float dq = dir == 0 ? __expf(g[r]) : (r > 0 ? __expf(g[r - 1]) : 1.f);
        rec[RC::kQ + idx] = dq * Qs[r * SM::kLdk + d];
        rec[RC::kK + idx] = __expf(gl - g[r]) * Ks[r * SM::kLdk + d];
    }
    for (int idx = tid; idx < kChunk * DV; idx += blockDim.x) {
        const int r = idx / DV, d = idx % DV;
        float u = 0.f;
        for (int m = 0; m <= r; ++m) u = fmaf(Tm[r * SM::kLdc + m], bt[m] * Vs[m * SM::kLdv + d], u);
        rec[RC::kU + idx] = u;
    }
    for (int idx = tid; idx < kChunk * kChunk; idx += blockDim.x)
        rec[RC::kP + idx] = Bq[(idx / kChunk) * SM::kLdc + idx % kChunk];
    if (tid == 0) {
        rec[RC::kDs] = __expf(gl);
        rec[RC::kDs + 1] = rec[RC::kDs + 2] = rec[RC::kDs + 3] = 0.f;
    }
}

template <int DK, int NS>
struct ChainSmem {
    static constexpr int kLdk = DK + 4;   // keeps rows 16-byte aligned
    static constexpr int kS = 0;                          // S   [DK][NS]
    static constexpr int kW = kS + DK * NS;                // W   [C][kLdk]
    static constexpr int kQ = kW + kChunk * kLdk;          // Qh  [C][kLdk]
    static constexpr int kK = kQ + kChunk * kLdk;          // Kt  [C][kLdk]
    static constexpr int kU = kK + kChunk * kLdk;          // U   [C][NS]
    static constexpr int kP = kU + kChunk * NS;            // P   [C][C+4]
    static constexpr int kD = kP + kChunk * (kChunk + 4);  // Delta [C][NS]
    static constexpr int kFloats = kD + kChunk * NS;
    static constexpr size_t kBytes = sizeof(float) * kFloats;
};

// Output modes of the chain kernel.
enum OutMode { kOutStore = 0, kOutPartial = 1, kOutAddPartial = 2 };

// grid (DV/NS, B*H, 1), block 256.  One CTA walks every chunk of one (b,h)
// in direction `dir`, holding S[:, slice] in shared memory.
//   kOutStore      o <- O (cast to Tout)
//   kOutPartial    part <- O (fp32; the first half of a bidirectional pair)
//   kOutAddPartial o <- part + O, rounded once
template <int DK, int DV, int NS, typename Tout>
__global__ void __launch_bounds__(256)
chain_kernel(const float* __restrict__ ws, const float* __restrict__ state_in,
             float* __restrict__ state_out, Tout* __restrict__ o, float* __restrict__ part,
             int T, int H, int nC, int dir, int out_mode, int nbh)
{
    using SM = ChainSmem<DK, NS>;
    using RC = Record<DK, DV>;
    extern __shared__ __align__(16) float sm[];
    float* S = sm + SM::kS;
    float* Ws = sm + SM::kW;
    float* Qs = sm + SM::kQ;
    float* Kt = sm + SM::kK;
    float* Us = sm + SM::kU;
    float* Ps = sm + SM::kP;
    float* Dl = sm + SM::kD;
    __shared__ float ds_sh;

    const int slice = blockIdx.x, bh = blockIdx.y;
    const int b = bh / H, h = bh % H;
    const int tid = threadIdx.x;
    const int j0 = slice * NS;

    for (int idx = tid; idx < DK * NS; idx += blockDim.x) {
        const int d = idx / NS, j = idx % NS;
        S[idx] = state_in ? state_in[((size_t)bh * DK + d) * DV + j0 + j] : 0.f;
    }

    for (int step = 0; step < nC; ++step) {
        const int c = dir == 0 ? step : nC - 1 - step;
        const float* rec = ws + ((size_t)(dir * nbh + bh) * nC + c) * RC::kFloats;
        __syncthreads();  // previous chunk fully consumed
        for (int idx = tid; idx < kChunk * DK / 4; idx += blockDim.x) {
            const int r = idx / (DK / 4), d4 = idx % (DK / 4);
            const float4 w4 = reinterpret_cast<const float4*>(rec + RC::kW)[idx];
            const float4 q4 = reinterpret_cast<const float4*>(rec + RC::kQ)[idx];
            const float4 k4 = reinterpret_cast<const float4*>(rec + RC::kK)[idx];
            reinterpret_cast<float4*>(Ws + r * SM::kLdk)[d4] = w4;
            reinterpret_cast<float4*>(Qs + r * SM::kLdk)[d4] = q4;
            reinterpret_cast<float4*>(Kt + r * SM::kLdk)[d4] = k4;
        }
        for (int idx = tid; idx < kChunk * NS; idx += blockDim.x) {
            const int r = idx / NS, j = idx % NS;
            Us[idx] = rec[RC::kU + r * DV + j0 + j];
        }
        for (int idx = tid; idx < kChunk * kChunk; idx += blockDim.x)
            Ps[(idx / kChunk) * (kChunk + 4) + idx % kChunk] = rec[RC::kP + idx];
        if (tid == 0) ds_sh = rec[RC::kDs];
        __syncthreads();
        // Delta = U - W S
        for (int idx = tid; idx < kChunk * NS; idx += blockDim.x) {
            const int r = idx / NS, j = idx % NS;
            float acc = Us[idx];
            const float* wr = Ws + r * SM::kLdk;
#pragma unroll 8
            for (int d = 0; d < DK; ++d) acc = fmaf(-wr[d], S[d * NS + j], acc);
            Dl[idx] = acc;
        }
        __syncthreads();
        // O = Qh S + P Delta -> output
        for (int idx = tid; idx < kChunk * NS; idx += blockDim.x) {
            const int r = idx / NS, j = idx % NS;
            float acc = 0.f;
            const float* qr = Qs + r * SM::kLdk;
#pragma unroll 8
            for (int d = 0; d < DK; ++d) acc = fmaf(qr[d], S[d * NS + j], acc);
            const float* pr = Ps + r * (kChunk + 4);
#pragma unroll 8
            for (int s = 0; s < kChunk; ++s) acc = fmaf(pr[s], Dl[s * NS + j], acc);
            const int t = token_of_row(c, r, dir);
            if (t < T) {
                const size_t off = (((size_t)b * T + t) * H + h) * DV + j0 + j;
                if (out_mode == kOutStore) o[off] = from_f32<Tout>(acc);
                else if (out_mode == kOutPartial) part[off] = acc;
                else o[off] = from_f32<Tout>(part[off] + acc);
            }
        }
        __syncthreads();  // every read of the old S is done
        // S <- ds S + Kt^T Delta
        const float dsv = ds_sh;
        for (int idx = tid; idx < DK * NS; idx += blockDim.x) {
            const int d = idx / NS, j = idx % NS;
            float acc = dsv * S[idx];
#pragma unroll 8
            for (int r = 0; r < kChunk; ++r) acc = fmaf(Kt[r * SM::kLdk + d], Dl[r * NS + j], acc);
            S[idx] = acc;
        }
    }
    __syncthreads();
    if (state_out) {
        for (int idx = tid; idx < DK * NS; idx += blockDim.x) {
            const int d = idx / NS, j = idx % NS;
            state_out[((size_t)bh * DK + d) * DV + j0 + j] = S[idx];
        }
    }
}

}  // namespace simt
}  // namespace gdn
