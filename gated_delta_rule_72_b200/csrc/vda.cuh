// vda.cuh -- frame-wise delta operator (VDA): the kernels that run on the
// CUDA cores, in fp32 (vda_tc.cuh has the tensor-core Gram and readout used
// for bf16 inputs with d_k = 128).
//
// The sequence is split into F frames of U consecutive tokens.  For frame f
// (keys K_f: U x dk, values V_f: U x dv, per-token write strengths beta, a
// per-frame decay alpha_f):
//   A_f = K_f^T diag(beta) K_f,   B_f = K_f^T diag(beta) V_f
//   S_f = (I + A_f)^{-1} (alpha_f S_{f-1} + B_f)          (causal)
//   R_f = (I + A_f)^{-1} (alpha_f R_{f+1} + B_f)          (reverse)
// the state closest to the decayed memory that fits all of the frame's
// key-value pairs in the least-squares sense.  Readout of a token u of frame
// f: o_u = S_f^T q_u (+ R_{f+1}^T q_u for a bidirectional scan: the frames
// after f only).
//
// Four steps:
//   vda_gram    (frame x head, fully parallel)  A_f and B_f
//   vda_factor  (frame x head, fully parallel)  P_f = (I + A_f)^{-1} by a
//               Cholesky factorisation: none of it depends on the state
//   vda_chain   (head x direction x 32 state columns, sequential over frames)
//               S <- P_f (alpha_f S + B_f), the slice of the state in shared
//               memory; stores the state each frame's readout uses
//   vda_readout (token block x head, fully parallel)  o = Q (S + R)
#pragma once

#include "common.cuh"

namespace gdn {
namespace vda {

constexpr int kThreads = 256;
constexpr int kChainThreads = 512;
constexpr int kGramTok = 32;     // tokens staged per gram step

// ---------------------------------------------------------------------------
// A_f (DK x DK) and B_f (DK x DV) of one frame and head.  Thread tile: 8 rows
// (key index i) x 16 columns of [K | V] (key index or value index j).
// ---------------------------------------------------------------------------
template <int DK, int DV>
struct GramSmem {
    static constexpr int kW = DK + DV;                       // [K | V] row
    static constexpr int kRows = kGramTok * kW;              // staged [token][K | V]
    static constexpr int kBytes = (kRows + kGramTok * DK + kGramTok) * 4;   // + beta K, beta
};

template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(kThreads)
vda_gram_kernel(const Tin *__restrict__ k, const Tin *__restrict__ v, const float *__restrict__ beta,
                float *__restrict__ A, float *__restrict__ Bm, int F, int U, int H)
{
    using SM = GramSmem<DK, DV>;
    constexpr int W = SM::kW;
    constexpr int TR = 8, TC = 16;                 // thread tile
    constexpr int NCT = W / TC;                    // column tiles
    constexpr int kTiles = (DK / TR) * NCT;        // 64 .. 256: the other threads only stage
    static_assert(kTiles <= kThreads && DK % TC == 0, "thread tiles");
    extern __shared__ __align__(16) float gsm[];
    float *kv = gsm;                               // [tok][K | V]
    float *bk = gsm + SM::kRows;                   // [tok][beta K]
    float *bs = bk + kGramTok * DK;                // [tok]
    const int f = blockIdx.x, bh = blockIdx.y, b = bh / H, h = bh % H;
    const int T = F * U;
    const int tid = threadIdx.x;
    const int i0 = (tid / NCT) * TR, j0 = (tid % NCT) * TC;
    float acc[TR][TC];
#pragma unroll
    for (int r = 0; r < TR; ++r)
#pragma unroll
        for (int c = 0; c < TC; ++c) acc[r][c] = 0.f;

    for (int u0 = 0; u0 < U; u0 += kGramTok) {
        const int n = min(kGramTok, U - u0);
        __syncthreads();
        for (int e = tid; e < kGramTok * W; e += kThreads) {
            const int tk = e / W, c = e % W;
            float x = 0.f;
            if (tk < n) {
                const size_t row = ((size_t)b * T + (size_t)f * U + u0 + tk) * H + h;
                x = c < DK ? to_f32(k[row * DK + c]) : to_f32(v[row * DV + (c - DK)]);
            }
            kv[e] = x;
        }
        for (int tk = tid; tk < kGramTok; tk += kThreads)
            bs[tk] = tk < n ? beta[((size_t)b * T + (size_t)f * U + u0 + tk) * H + h] : 0.f;
        __syncthreads();
        for (int e = tid; e < kGramTok * DK; e += kThreads) bk[e] = bs[e / DK] * kv[(e / DK) * W + e % DK];
        __syncthreads();
        if (tid >= kTiles) continue;
#pragma unroll 2
        for (int tk = 0; tk < kGramTok; ++tk) {
            float a[TR], bcol[TC];
#pragma unroll
            for (int r = 0; r < TR; r += 4) {
                const float4 x = *reinterpret_cast<const float4 *>(bk + tk * DK + i0 + r);
                a[r] = x.x; a[r + 1] = x.y; a[r + 2] = x.z; a[r + 3] = x.w;
            }
#pragma unroll
            for (int c = 0; c < TC; c += 4) {
                const float4 x = *reinterpret_cast<const float4 *>(kv + tk * W + j0 + c);
                bcol[c] = x.x; bcol[c + 1] = x.y; bcol[c + 2] = x.z; bcol[c + 3] = x.w;
            }
#pragma unroll
            for (int r = 0; r < TR; ++r)
#pragma unroll
                for (int c = 0; c < TC; ++c) acc[r][c] = fmaf(a[r], bcol[c], acc[r][c]);
        }
    }
    if (tid >= kTiles) return;
    // columns j < DK belong to A, the rest to B
    const size_t fh = (size_t)f * gridDim.y + bh;
#pragma unroll
    for (int r = 0; r < TR; ++r) {
        const int i = i0 + r;
#pragma unroll
        for (int c = 0; c < TC; c += 4) {
            const int j = j0 + c;
            const float4 x = make_float4(acc[r][c], acc[r][c + 1], acc[r][c + 2], acc[r][c + 3]);
            if (j < DK) *reinterpret_cast<float4 *>(A + (fh * DK + i) * DK + j) = x;
            else *reinterpret_cast<float4 *>(Bm + (fh * DK + i) * DV + (j - DK)) = x;
        }
    }
}

// ---------------------------------------------------------------------------
// Factor (frame x head, fully parallel: nothing here depends on the state):
// P_f = (I + A_f)^{-1}, written over A_f.
//
// M = I + A_f = L L^T (Cholesky, right-looking, one barrier per column: step
// j reads the pivot and column j of the lower triangle, writes L's column j
// transposed into the upper triangle (row j, which no later step reads or
// writes) and subtracts the column's outer product from the trailing lower
// triangle; warp w takes the rows i = w mod 16, its lanes the columns).
// Then L Y = I and L^T P = Y with no block barrier: each warp owns 8
// right-hand-side columns, each column's 4 lanes split its rows (i = g mod
// 4), so a step only involves lanes of one warp.
// ---------------------------------------------------------------------------
template <int DK, int DV>
struct FactorSmem {
    static constexpr int kW = DK;                          // right-hand sides: I
    static constexpr int kLdM = DK + 1;                    // odd stride: column walks are conflict-free
    static constexpr int kLdX = kW + 8;                    // 4 row groups of a column on 4 bank groups
    static constexpr int kM = 0;
    static constexpr int kX = kM + DK * kLdM * 4;
    static constexpr int kD = kX + DK * kLdX * 4;          // 1 / diagonal of L
    static constexpr int kBytes = kD + DK * 4;
};

template <int DK, int DV>
__global__ void __launch_bounds__(kChainThreads)
vda_factor_kernel(float *__restrict__ A)
{
    using SM = FactorSmem<DK, DV>;
    constexpr int LD = SM::kLdM, LX = SM::kLdX, W = SM::kW;
    constexpr int NW = kChainThreads / 32;
    static_assert(W % 8 == 0, "right-hand-side columns in groups of 8 (warp-uniform loop bounds)");
    extern __shared__ __align__(16) unsigned char fsm[];
    float *M = reinterpret_cast<float *>(fsm + SM::kM);
    float *X = reinterpret_cast<float *>(fsm + SM::kX);
    float *rdL = reinterpret_cast<float *>(fsm + SM::kD);
    const size_t fh = (size_t)blockIdx.x * gridDim.y + blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float *Af = A + fh * DK * DK;
    for (int e = tid; e < DK * DK; e += kChainThreads) {
        const int i = e / DK, j = e % DK;
        M[i * LD + j] = Af[e] + (i == j ? 1.f : 0.f);
        X[i * LX + j] = i == j ? 1.f : 0.f;
    }
    __syncthreads();
    // ---- Cholesky
    for (int j = 0; j < DK; ++j) {
        const float piv = M[j * LD + j];
        const float r = rsqrtf(piv), r2 = r * r;
        for (int i = j + 1 + ((warp - (j + 1)) & (NW - 1)); i < DK; i += NW) {
            const float mij = M[i * LD + j];
            if (lane == 0) M[j * LD + i] = mij * r;        // L[i][j], kept at (j, i)
            const float fct = mij * r2;
            int cc = j + 1 + lane;
            for (; cc + 96 <= i; cc += 128) {              // four columns loaded before any store
                float lc[4], m[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    lc[q] = M[(cc + 32 * q) * LD + j];
                    m[q] = M[i * LD + cc + 32 * q];
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) M[i * LD + cc + 32 * q] = fmaf(-fct, lc[q], m[q]);
            }
            for (; cc <= i; cc += 32) M[i * LD + cc] = fmaf(-fct, M[cc * LD + j], M[i * LD + cc]);
        }
        if (tid == 0) rdL[j] = r;                          // 1 / L[j][j]
        __syncthreads();
    }
    // ---- L Y = I, then L^T P = Y, column by column inside each warp.
    // A step's row updates are independent: four rows are loaded before any is
    // stored, so their shared-memory latencies overlap.
    const int g = lane >> 3;
    auto update_rows = [&](int i, int i_end, int c, float y, int lstride, int loff) {
        // X[i][c] -= L * y for rows i, i+4, ... < i_end; L of row i at M[i*lstride + loff]
        for (; i + 12 < i_end; i += 16) {
            float l[4], x[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                l[q] = M[(i + 4 * q) * lstride + loff];
                x[q] = X[(i + 4 * q) * LX + c];
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) X[(i + 4 * q) * LX + c] = fmaf(-l[q], y, x[q]);
        }
        for (; i < i_end; i += 4) X[i * LX + c] = fmaf(-M[i * lstride + loff], y, X[i * LX + c]);
    };
    for (int c = warp * 8 + (lane & 7); c < W; c += NW * 8) {
        for (int j = 0; j < DK; ++j) {
            const float y = X[j * LX + c] * rdL[j];
            __syncwarp();
            if ((j & 3) == g) X[j * LX + c] = y;
            update_rows(j + 1 + ((g - (j + 1)) & 3), DK, c, y, 1, j * LD);    // L[i][j] at (j, i)
            __syncwarp();
        }
        for (int j = DK - 1; j >= 0; --j) {
            const float y = X[j * LX + c] * rdL[j];
            __syncwarp();
            if ((j & 3) == g) X[j * LX + c] = y;
            update_rows(g, j, c, y, LD, j);                                   // L[j][i] at (i, j)
            __syncwarp();
        }
    }
    __syncthreads();
    for (int e = tid; e < DK * DK; e += kChainThreads) Af[e] = X[(e / DK) * LX + e % DK];
}

// ---------------------------------------------------------------------------
// The frame chain of one head, direction and slice of kSlice state columns
// (the columns are independent: P_f acts on each alike): S <- P_f (alpha_f S
// + B_f) per frame, in the direction's order.  The state each readout needs
// goes to `st` ([dir][F][B*H][DK][DV]): the causal direction stores S_f, the
// reverse one R_{f+1} (before the frame is written), as fp32 or (kImage) as
// the tensor-core readout's operand image.  Thread tile 4 rows x 2 columns;
// P_f (symmetric: row k of P is column k) is staged in shared memory.
// ---------------------------------------------------------------------------
constexpr int kSlice = 32;

// State image for the tensor-core readout: [S_hi | S_lo] as bf16, the
// operand layout of a 128B-swizzled MN-major B tile (rows = the key index,
// groups of 64 columns 16 KB apart); S_hi + S_lo = S to about 2^-16.  Same
// byte size as the fp32 state.
__device__ __forceinline__ int img_off(int i, int n) {
    const int L = i * 128 + (n & 63) * 2;
    return (n >> 6) * 16384 + (L ^ (((L >> 7) & 7) << 4));
}
template <int DV>
__device__ __forceinline__ void store_image_row8(unsigned char *img, int i, int n, const float *x) {
    uint4 hi, lo;
    uint32_t *ph = reinterpret_cast<uint32_t *>(&hi), *pl = reinterpret_cast<uint32_t *>(&lo);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const __nv_bfloat162 hv = __floats2bfloat162_rn(x[2 * q], x[2 * q + 1]);
        const float2 hf = __bfloat1622float2(hv);
        const __nv_bfloat162 lv = __floats2bfloat162_rn(x[2 * q] - hf.x, x[2 * q + 1] - hf.y);
        ph[q] = *reinterpret_cast<const uint32_t *>(&hv);
        pl[q] = *reinterpret_cast<const uint32_t *>(&lv);
    }
    *reinterpret_cast<uint4 *>(img + img_off(i, n)) = hi;
    *reinterpret_cast<uint4 *>(img + img_off(i, n + DV)) = lo;
}

template <int DK, int DV>
struct ChainSmem {
    static constexpr int kP = 0;                           // [DK][DK]
    static constexpr int kS = kP + DK * DK * 4;            // [DK][kSlice]
    static constexpr int kBytes = kS + DK * kSlice * 4;
};

template <int DK, int DV, bool kImage>
__global__ void __launch_bounds__(kChainThreads)
vda_chain_kernel(const float *__restrict__ P, const float *__restrict__ Bm, const float *__restrict__ alpha_f,
                 const float *s_in, const float *s_in_bwd, float *s_out, float *s_out_bwd,
                 float *__restrict__ st, int F, int H)
{
    using SM = ChainSmem<DK, DV>;
    constexpr int TR = 4, TCc = 2;
    constexpr int NCT = kSlice / TCc;                  // column tiles
    constexpr int kTiles = (DK / TR) * NCT;
    static_assert(kTiles <= kChainThreads && DV % kSlice == 0, "thread tiles");
    extern __shared__ __align__(16) unsigned char csm[];
    float *Ps = reinterpret_cast<float *>(csm + SM::kP);
    float *S = reinterpret_cast<float *>(csm + SM::kS);
    const int bh = blockIdx.x, nbh = gridDim.x, dir = blockIdx.y, j0 = blockIdx.z * kSlice;
    const int b = bh / H, h = bh % H;
    const int tid = threadIdx.x;
    const float *src0 = dir ? s_in_bwd : s_in;   // (an output state may be its own input)
    float *dst_end = dir ? s_out_bwd : s_out;
    const size_t sdim = (size_t)DK * DV;
    for (int e = tid; e < DK * kSlice; e += kChainThreads) {
        const int i = e / kSlice, c = e % kSlice;
        S[e] = src0 ? src0[bh * sdim + (size_t)i * DV + j0 + c] : 0.f;
    }
    const bool worker = tid < kTiles;
    const int i0 = (tid / NCT) * TR, c0 = (tid % NCT) * TCc;
    // the slice's state to `dst` (fp32, or operand image: 8 columns per 16-byte chunk)
    auto store_state = [&](float *dst) {
        if (kImage) {
            for (int e = tid; e < DK * (kSlice / 8); e += kChainThreads) {
                const int i = e / (kSlice / 8), q = e % (kSlice / 8);
                store_image_row8<DV>(reinterpret_cast<unsigned char *>(dst), i, j0 + 8 * q, S + i * kSlice + 8 * q);
            }
        } else {
            for (int e = tid; e < DK * kSlice; e += kChainThreads) {
                const int i = e / kSlice, c = e % kSlice;
                dst[(size_t)i * DV + j0 + c] = S[e];
            }
        }
    };

    for (int step = 0; step < F; ++step) {
        const int f = dir ? F - 1 - step : step;
        const size_t fh = (size_t)f * nbh + bh;
        const float a = alpha_f[((size_t)b * F + f) * H + h];
        float *dst = st + ((size_t)dir * F * nbh + fh) * sdim;
        __syncthreads();                                   // S complete, P free
        if (dir) store_state(dst);                         // the reverse readout of frame f reads R_{f+1}
        for (int e = tid * 4; e < DK * DK; e += kChainThreads * 4)
            *reinterpret_cast<float4 *>(Ps + e) = *reinterpret_cast<const float4 *>(P + fh * DK * DK + e);
        __syncthreads();
        for (int e = tid; e < DK * kSlice; e += kChainThreads) {   // S <- alpha S + B
            const int i = e / kSlice, c = e % kSlice;
            S[e] = fmaf(a, S[e], Bm[fh * sdim + (size_t)i * DV + j0 + c]);
        }
        __syncthreads();
        float acc[TR][TCc];
        if (worker) {
#pragma unroll
            for (int r = 0; r < TR; ++r)
#pragma unroll
                for (int cc = 0; cc < TCc; ++cc) acc[r][cc] = 0.f;
#pragma unroll 8
            for (int kk = 0; kk < DK; ++kk) {
                const float4 pv = *reinterpret_cast<const float4 *>(Ps + kk * DK + i0);   // P[i0..][kk]
                const float2 sv = *reinterpret_cast<const float2 *>(S + kk * kSlice + c0);
                const float pa[TR] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
                for (int r = 0; r < TR; ++r) {
                    acc[r][0] = fmaf(pa[r], sv.x, acc[r][0]);
                    acc[r][1] = fmaf(pa[r], sv.y, acc[r][1]);
                }
            }
        }
        __syncthreads();                                   // every read of the old S is done
        if (worker)
#pragma unroll
            for (int r = 0; r < TR; ++r)
                *reinterpret_cast<float2 *>(S + (i0 + r) * kSlice + c0) = make_float2(acc[r][0], acc[r][1]);
        if (!dir) {
            __syncthreads();
            store_state(dst);
        }
    }
    __syncthreads();
    if (dst_end)
        for (int e = tid; e < DK * kSlice; e += kChainThreads) {
            const int i = e / kSlice, c = e % kSlice;
            dst_end[bh * sdim + (size_t)i * DV + j0 + c] = S[e];
        }
}

// ---------------------------------------------------------------------------
// Readout: 64 tokens of one frame per CTA, o = Q (S + R): the two directions'
// states are added once while they are staged.  Thread tile: 4 tokens x 8
// value columns (DV = 128; 4 columns for DV = 64).
// ---------------------------------------------------------------------------
template <int DK, int DV>
struct ReadSmem {
    static constexpr int kQ = 0;                             // [DK][64] (transposed)
    static constexpr int kS = kQ + DK * 64 * 4;              // [DK][DV]
    static constexpr int kBytes = kS + DK * DV * 4;
};

template <int DK, int DV, typename Tin, typename Tout>
__global__ void __launch_bounds__(kThreads)
vda_readout_kernel(const Tin *__restrict__ q, const float *__restrict__ st, Tout *__restrict__ o, int F, int U,
                   int H, int ndir)
{
    using SM = ReadSmem<DK, DV>;
    constexpr int TC = DV / 16;                    // value columns per thread
    extern __shared__ __align__(16) unsigned char rsm[];
    float *Qt = reinterpret_cast<float *>(rsm + SM::kQ);
    float *Ss = reinterpret_cast<float *>(rsm + SM::kS);
    const int nblk = (U + 63) / 64;
    const int f = blockIdx.x / nblk, u0 = (blockIdx.x % nblk) * 64;
    const int bh = blockIdx.y, nbh = gridDim.y, b = bh / H, h = bh % H;
    const int T = F * U, n = min(64, U - u0);
    const int tid = threadIdx.x;
    const size_t sdim = (size_t)DK * DV;
    for (int e = tid; e < 64 * DK; e += kThreads) {
        const int tk = e / DK, i = e % DK;
        Qt[i * 64 + tk] = tk < n ? to_f32(q[(((size_t)b * T + (size_t)f * U + u0 + tk) * H + h) * DK + i]) : 0.f;
    }
    {
        const float *s0 = st + ((size_t)f * nbh + bh) * sdim;
        const float *s1 = s0 + (size_t)F * nbh * sdim;            // the reverse direction's
        for (int e = tid * 4; e < DK * DV; e += kThreads * 4) {
            float4 x = *reinterpret_cast<const float4 *>(s0 + e);
            if (ndir == 2) {
                const float4 y = *reinterpret_cast<const float4 *>(s1 + e);
                x.x += y.x; x.y += y.y; x.z += y.z; x.w += y.w;
            }
            *reinterpret_cast<float4 *>(Ss + e) = x;
        }
    }
    __syncthreads();
    const int t0 = (tid / 16) * 4, c0 = (tid % 16) * TC;
    float acc[4][TC];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < TC; ++c) acc[r][c] = 0.f;
    {
        const float *Sd = Ss;
#pragma unroll 4
        for (int i = 0; i < DK; ++i) {
            const float4 qv = *reinterpret_cast<const float4 *>(Qt + i * 64 + t0);
            const float qa[4] = {qv.x, qv.y, qv.z, qv.w};
            float sv[TC];
#pragma unroll
            for (int c = 0; c < TC; c += 4) {
                const float4 x = *reinterpret_cast<const float4 *>(Sd + i * DV + c0 + c);
                sv[c] = x.x; sv[c + 1] = x.y; sv[c + 2] = x.z; sv[c + 3] = x.w;
            }
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c < TC; ++c) acc[r][c] = fmaf(qa[r], sv[c], acc[r][c]);
        }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        if (t0 + r >= n) break;
        Tout *dst = o + (((size_t)b * T + (size_t)f * U + u0 + t0 + r) * H + h) * DV + c0;
#pragma unroll
        for (int c = 0; c < TC; ++c) dst[c] = from_f32<Tout>(acc[r][c]);
    }
}

}  // namespace vda
}  // namespace gdn
