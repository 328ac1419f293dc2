// vda.cuh -- frame-wise delta operator (VDA) on the CUDA cores, fp32.
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
// Three kernels:
//   vda_gram    (frame x head, fully parallel)  A_f and B_f
//   vda_chain   (head x direction, sequential over frames)  Cholesky of
//               I + A_f and two triangular solves per frame, the state in
//               shared memory; stores the state each frame's readout uses
//   vda_readout (token block x head, fully parallel)  o = Q S (+ Q R)
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
// The frame chain of one head and direction.  Per frame (in the direction's
// order): M = I + A_f, X = alpha_f S + B_f; M = L L^T (Cholesky); L Y = X,
// L^T S' = Y.  The state each readout needs goes to `st`
// ([dir][F][B*H][DK][DV]): the causal direction stores S_f, the reverse one
// R_{f+1} (before the frame is written).
//
// Cholesky, right-looking, one barrier per column: step j reads the pivot
// and column j of the lower triangle, writes L's column j transposed into the
// upper triangle (row j, which no later step reads or writes) and subtracts
// the column's outer product from the trailing lower triangle; warp w takes
// the rows i = w mod 16, its lanes the columns.  The diagonal of L goes to
// its own array.  The triangular solves need no block barrier: each warp owns
// 8 columns of X and each column's 4 lanes split its rows (i = g mod 4), so a
// step only needs the column's own lanes, which share the warp.
// ---------------------------------------------------------------------------
template <int DK, int DV>
struct ChainSmem {
    static constexpr int kLdM = DK + 1;                    // odd stride: column walks are conflict-free
    static constexpr int kLdX = DV + 8;                    // 4 row groups of a column on 4 bank groups
    static constexpr int kM = 0;
    static constexpr int kS = kM + DK * kLdM * 4;          // state [DK][DV]
    static constexpr int kX = kS + DK * DV * 4;            // right-hand side / solution [DK][kLdX]
    static constexpr int kD = kX + DK * kLdX * 4;          // diagonal of L, and its inverse
    static constexpr int kBytes = kD + 2 * DK * 4;
};

template <int DK, int DV>
__global__ void __launch_bounds__(kChainThreads)
vda_chain_kernel(const float *__restrict__ A, const float *__restrict__ Bm, const float *__restrict__ alpha_f,
                 const float *s_in, const float *s_in_bwd, float *s_out, float *s_out_bwd,
                 float *__restrict__ st, int F, int H)
{
    using SM = ChainSmem<DK, DV>;
    constexpr int LD = SM::kLdM, LX = SM::kLdX;
    constexpr int NW = kChainThreads / 32;
    static_assert(DV <= NW * 8, "8 columns of X per warp");
    extern __shared__ __align__(16) unsigned char csm[];
    float *M = reinterpret_cast<float *>(csm + SM::kM);
    float *S = reinterpret_cast<float *>(csm + SM::kS);
    float *X = reinterpret_cast<float *>(csm + SM::kX);
    float *dL = reinterpret_cast<float *>(csm + SM::kD);
    float *rdL = dL + DK;
    const int bh = blockIdx.x, nbh = gridDim.x, dir = blockIdx.y;
    const int b = bh / H, h = bh % H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const float *src0 = dir ? s_in_bwd : s_in;   // (an output state may be its own input)
    float *dst_end = dir ? s_out_bwd : s_out;
    const size_t sdim = (size_t)DK * DV;
    for (int e = tid; e < DK * DV; e += kChainThreads) S[e] = src0 ? src0[bh * sdim + e] : 0.f;
    // solve lanes: column c of X, row group g
    const int c = warp * 8 + (lane & 7), g = lane >> 3;
    const bool solver = c < DV;

    for (int step = 0; step < F; ++step) {
        const int f = dir ? F - 1 - step : step;
        const size_t fh = (size_t)f * nbh + bh;
        const float a = alpha_f[((size_t)b * F + f) * H + h];
        __syncthreads();
        float *dst = st + ((size_t)dir * F * nbh + fh) * sdim;
        if (dir)   // the reverse readout of frame f reads R_{f+1}
            for (int e = tid; e < DK * DV; e += kChainThreads) dst[e] = S[e];
        for (int e = tid; e < DK * DK; e += kChainThreads) {
            const int i = e / DK, j = e % DK;
            M[i * LD + j] = A[fh * DK * DK + e] + (i == j ? 1.f : 0.f);
        }
        for (int e = tid; e < DK * DV; e += kChainThreads)
            X[(e / DV) * LX + e % DV] = fmaf(a, S[e], Bm[fh * sdim + e]);
        __syncthreads();
        // ---- Cholesky
        for (int j = 0; j < DK; ++j) {
            const float piv = M[j * LD + j];
            const float r = rsqrtf(piv), r2 = r * r;
            for (int i = j + 1 + ((warp - (j + 1)) & (NW - 1)); i < DK; i += NW) {
                const float mij = M[i * LD + j];
                if (lane == 0) M[j * LD + i] = mij * r;        // L[i][j], kept at (j, i)
                const float fct = mij * r2;
                for (int cc = j + 1 + lane; cc <= i; cc += 32)
                    M[i * LD + cc] = fmaf(-fct, M[cc * LD + j], M[i * LD + cc]);
            }
            if (tid == 0) {
                dL[j] = piv * r;
                rdL[j] = r;
            }
            __syncthreads();
        }
        // ---- L Y = X, then L^T S' = Y, column by column inside each warp
        if (solver) {
            for (int j = 0; j < DK; ++j) {
                const float y = X[j * LX + c] * rdL[j];
                __syncwarp();
                if ((j & 3) == g) X[j * LX + c] = y;
                for (int i = j + 1 + ((g - (j + 1)) & 3); i < DK; i += 4)
                    X[i * LX + c] = fmaf(-M[j * LD + i], y, X[i * LX + c]);   // L[i][j] at (j, i)
                __syncwarp();
            }
            for (int j = DK - 1; j >= 0; --j) {
                const float y = X[j * LX + c] * rdL[j];
                __syncwarp();
                if ((j & 3) == g) X[j * LX + c] = y;
                for (int i = g; i < j; i += 4)
                    X[i * LX + c] = fmaf(-M[i * LD + j], y, X[i * LX + c]);   // L[j][i] at (i, j)
                __syncwarp();
            }
        }
        __syncthreads();
        for (int e = tid; e < DK * DV; e += kChainThreads) {
            const float x = X[(e / DV) * LX + e % DV];
            S[e] = x;
            if (!dir) dst[e] = x;
        }
    }
    __syncthreads();
    if (dst_end)
        for (int e = tid; e < DK * DV; e += kChainThreads) dst_end[bh * sdim + e] = S[e];
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
