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
//               blocked Cholesky factorisation: none of it depends on the state
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
// P_f = (I + A_f)^{-1}, written over A_f, on blocks of 32 x 32 (NB = DK / 32
// block rows), fp32:
//   1. M = I + A_f = L L^T, a blocked right-looking Cholesky.  Per block
//      column: warp 0 factors the diagonal block in registers, a thread per
//      row below it solves for the panel L_ip (forward substitution against
//      L_pp), and all threads apply the trailing update M_ij -= L_ip L_jp^T.
//      Three barriers per block column instead of one per column.
//   2. Y = L^{-1}: the diagonal blocks' inverses (a warp each), then
//      recursive doubling over the blocks: Y_10 = -Y_11 (L_10 Y_00) in each
//      pair of blocks, then the same on the pair of pairs.
//   3. P = Y^T Y (P_ij = sum over k >= max(i, j) of Y_ki Y_kj).
// ---------------------------------------------------------------------------
template <int DK, int DV>
struct FactorSmem {
    static constexpr int kLdM = DK + 1;                    // L: odd stride, column walks conflict-free
    static constexpr int kLdY = DK + 4;                    // Y = L^{-1}: rows 16-byte aligned
    static constexpr int kLdX = DK / 2 + 1;                // doubling scratch
    static constexpr int kM = 0;
    static constexpr int kY = kM + (DK * kLdM * 4 + 15) / 16 * 16;
    static constexpr int kX = kY + DK * kLdY * 4;
    static constexpr int kD = kX + (DK / 2) * kLdX * 4;    // 1 / diagonal of L
    static constexpr int kBytes = kD + DK * 4;
};

// Warp-level pieces of the factor (p0: first row of a 32 x 32 diagonal
// block; runtime, so that one copy of this straight-line code serves every
// block).
//
// Cholesky of the diagonal block in registers: lane i holds row i, column j's
// entries reach the other lanes by shuffles.  Entries right of the diagonal
// (k > lane) take part in the arithmetic but only ever feed entries right of
// the diagonal, and are written as zeros.  rd[p0 + j] = 1 / L_jj.
__device__ __forceinline__ void chol_diag_block(float *M, float *rd, int LM, int p0, int lane) {
    float a[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) a[k] = M[(p0 + lane) * LM + p0 + k];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const float r = rsqrtf(__shfl_sync(0xffffffffu, a[j], j));
        if (lane == j) rd[p0 + j] = r;
        a[j] *= r;
#pragma unroll
        for (int k = j + 1; k < 32; ++k) a[k] = fmaf(-a[j], __shfl_sync(0xffffffffu, a[j], k), a[k]);
    }
#pragma unroll
    for (int k = 0; k < 32; ++k) M[(p0 + lane) * LM + p0 + k] = k <= lane ? a[k] : 0.f;
}

// Panel row `row` below the diagonal block: x L_pp^T = m by forward
// substitution, in place (L_pp read with every lane at the same address).
__device__ __forceinline__ void chol_panel_row(float *M, const float *rd, int LM, int p0, int row) {
    float x[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) x[k] = M[row * LM + p0 + k];
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        float acc = x[k];
#pragma unroll
        for (int j = 0; j < k; ++j) acc = fmaf(-x[j], M[(p0 + k) * LM + p0 + j], acc);
        x[k] = acc * rd[p0 + k];
    }
#pragma unroll
    for (int k = 0; k < 32; ++k) M[row * LM + p0 + k] = x[k];
}

// Inverse of the diagonal block: lane c computes column c,
// y_i = (delta_ic - sum_{k<i} L_ik y_k) / L_ii (zero above the diagonal by itself).
__device__ __forceinline__ void diag_block_inverse(const float *M, const float *rd, float *Y, int LM, int LY,
                                                   int p0, int lane) {
    float y[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        float acc = i == lane ? 1.f : 0.f;
#pragma unroll
        for (int k = 0; k < i; ++k) acc = fmaf(-M[(p0 + i) * LM + p0 + k], y[k], acc);
        y[i] = acc * rd[p0 + i];
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) Y[(p0 + i) * LY + p0 + lane] = y[i];
}

// Trailing update after block column p0: M_ij -= sum_k L_ik L_jk over the R x R
// square below and right of the panel (only its lower triangle is used
// later).  Thread rows ti + 32 a, columns tj + 16 b.
template <int DK, int R>
__device__ __forceinline__ void chol_trailing(float *M, int p0, int tid) {
    constexpr int LM = DK + 1, NA = R / 32, NBc = R / 16;
    const int ti = tid & 31, tj = tid >> 5, base = p0 + 32;
    float acc[NA][NBc];
#pragma unroll
    for (int x = 0; x < NA; ++x)
#pragma unroll
        for (int z = 0; z < NBc; ++z) acc[x][z] = 0.f;
#pragma unroll 4
    for (int k = 0; k < 32; ++k) {
        float li[NA], lj[NBc];
#pragma unroll
        for (int x = 0; x < NA; ++x) li[x] = M[(base + ti + 32 * x) * LM + p0 + k];
#pragma unroll
        for (int z = 0; z < NBc; ++z) lj[z] = M[(base + tj + 16 * z) * LM + p0 + k];
#pragma unroll
        for (int x = 0; x < NA; ++x)
#pragma unroll
            for (int z = 0; z < NBc; ++z) acc[x][z] = fmaf(li[x], lj[z], acc[x][z]);
    }
#pragma unroll
    for (int x = 0; x < NA; ++x)
#pragma unroll
        for (int z = 0; z < NBc; ++z) M[(base + ti + 32 * x) * LM + base + tj + 16 * z] -= acc[x][z];
}

// One level of the recursive doubling for Y = L^{-1}: for every pair of
// adjacent diagonal blocks of size S (bottom block rows [r0, r0+S), top
// [r0-S, r0)), Y_bt = -Y_bb (L_bt Y_tt).  Each thread a 2 x 2 tile of the
// products; X is the scratch for L_bt Y_tt.
template <int DK, int S>
__device__ __forceinline__ void inverse_level(const float *M, float *Y, float *X, int tid) {
    constexpr int LM = DK + 1, LY = DK + 4, LX = DK / 2 + 1;
    constexpr int NPAIR = DK / (2 * S), TILES = (S / 2) * (S / 2);      // 2 x 2 tiles per pair
    static_assert(NPAIR * S <= DK / 2, "scratch rows");
    for (int u = tid; u < NPAIR * TILES; u += kChainThreads) {   // X = L_bt Y_tt (Y_tt lower)
        const int pr = u / TILES, t = u % TILES, i = 2 * (t / (S / 2)), j = 2 * (t % (S / 2));
        const int top = 2 * S * pr, bot = top + S;
        float *Xp = X + (pr * S) * LX;
        float x00 = 0.f, x01 = 0.f, x10 = 0.f, x11 = 0.f;
#pragma unroll 8
        for (int k = 0; k < S; ++k) {
            const float l0 = M[(bot + i) * LM + top + k], l1 = M[(bot + i + 1) * LM + top + k];
            const float y0 = Y[(top + k) * LY + top + j], y1 = Y[(top + k) * LY + top + j + 1];
            x00 = fmaf(l0, y0, x00); x01 = fmaf(l0, y1, x01);
            x10 = fmaf(l1, y0, x10); x11 = fmaf(l1, y1, x11);
        }
        Xp[i * LX + j] = x00; Xp[i * LX + j + 1] = x01;
        Xp[(i + 1) * LX + j] = x10; Xp[(i + 1) * LX + j + 1] = x11;
    }
    __syncthreads();
    for (int u = tid; u < NPAIR * TILES; u += kChainThreads) {   // Y_bt = -Y_bb X (Y_bb lower)
        const int pr = u / TILES, t = u % TILES, i = 2 * (t / (S / 2)), j = 2 * (t % (S / 2));
        const int top = 2 * S * pr, bot = top + S;
        const float *Xp = X + (pr * S) * LX;
        float y00 = 0.f, y01 = 0.f, y10 = 0.f, y11 = 0.f;
#pragma unroll 8
        for (int k = 0; k < S; ++k) {
            const float a0 = Y[(bot + i) * LY + bot + k], a1 = Y[(bot + i + 1) * LY + bot + k];
            const float x0 = Xp[k * LX + j], x1 = Xp[k * LX + j + 1];
            y00 = fmaf(a0, x0, y00); y01 = fmaf(a0, x1, y01);
            y10 = fmaf(a1, x0, y10); y11 = fmaf(a1, x1, y11);
        }
        Y[(bot + i) * LY + top + j] = -y00; Y[(bot + i) * LY + top + j + 1] = -y01;
        Y[(bot + i + 1) * LY + top + j] = -y10; Y[(bot + i + 1) * LY + top + j + 1] = -y11;
    }
    __syncthreads();
}

template <int DK, int DV>
__global__ void __launch_bounds__(kChainThreads)
vda_factor_kernel(float *__restrict__ A)
{
    using SM = FactorSmem<DK, DV>;
    constexpr int LM = SM::kLdM, LY = SM::kLdY, NB = DK / 32;
    static_assert(DK == 64 || DK == 128, "d_k of the factor");
    extern __shared__ __align__(16) unsigned char fsm[];
    float *M = reinterpret_cast<float *>(fsm + SM::kM);
    float *Y = reinterpret_cast<float *>(fsm + SM::kY);
    float *X = reinterpret_cast<float *>(fsm + SM::kX);
    float *rd = reinterpret_cast<float *>(fsm + SM::kD);
    const size_t fh = (size_t)blockIdx.x * gridDim.y + blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float *Af = A + fh * DK * DK;
    for (int e = tid; e < DK * DK; e += kChainThreads) {
        const int i = e / DK, j = e % DK;
        M[i * LM + j] = Af[e] + (i == j ? 1.f : 0.f);
        Y[i * LY + j] = 0.f;
    }
    __syncthreads();
    // ---- 1. Cholesky, block column by block column: the diagonal block (warp
    //      0), the panel below it (a thread per row), the trailing update (all)
#pragma unroll 1
    for (int p = 0; p < NB; ++p) {
        const int p0 = 32 * p, R = DK - p0 - 32;
        if (warp == 0) chol_diag_block(M, rd, LM, p0, lane);
        __syncthreads();
        if (R == 0) break;
        if (tid < R) chol_panel_row(M, rd, LM, p0, p0 + 32 + tid);
        __syncthreads();
        if (R == DK - 32) chol_trailing<DK, DK - 32>(M, p0, tid);
        else if (R == DK - 64) chol_trailing<DK, (DK > 64 ? DK - 64 : 32)>(M, p0, tid);
        else chol_trailing<DK, 32>(M, p0, tid);
        __syncthreads();
    }
    // ---- 2. Y = L^{-1}: the diagonal blocks (a warp each), then recursive
    //      doubling on pairs of 32-blocks and (for d_k = 128) of 64-blocks
    if (warp < NB) diag_block_inverse(M, rd, Y, LM, LY, 32 * warp, lane);
    __syncthreads();
    inverse_level<DK, 32>(M, Y, X, tid);
    if constexpr (NB == 4) inverse_level<DK, 64>(M, Y, X, tid);
    // ---- 3. P = Y^T Y.  Warp w owns row tiles of 4 rows (w and, for d_k = 128,
    //      31 - w, so that every warp has the same number of terms); lane l
    //      columns CW l .. CW l + CW - 1.  Terms k < the tile's first row are
    //      zero (Y lower triangular) and skipped.
    constexpr int CW = DK / 32;
    constexpr int NT = DK / 64;                       // row tiles per warp
#pragma unroll
    for (int tt = 0; tt < NT; ++tt) {
        const int i0 = 4 * (tt == 0 ? warp : (DK / 4 - 1 - warp));
        float acc[4][CW];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < CW; ++c) acc[r][c] = 0.f;
        for (int k = i0; k < DK; ++k) {
            const float4 yi = *reinterpret_cast<const float4 *>(Y + k * LY + i0);
            float yj[CW];
            if constexpr (CW == 4) {
                const float4 v = *reinterpret_cast<const float4 *>(Y + k * LY + CW * lane);
                yj[0] = v.x; yj[1] = v.y; yj[2] = v.z; yj[3] = v.w;
            } else {
                const float2 v = *reinterpret_cast<const float2 *>(Y + k * LY + CW * lane);
                yj[0] = v.x; yj[1] = v.y;
            }
            const float yr[4] = {yi.x, yi.y, yi.z, yi.w};
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c < CW; ++c) acc[r][c] = fmaf(yr[r], yj[c], acc[r][c]);
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            float *dst = Af + (size_t)(i0 + r) * DK + CW * lane;
            if constexpr (CW == 4) *reinterpret_cast<float4 *>(dst) = make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
            else *reinterpret_cast<float2 *>(dst) = make_float2(acc[r][0], acc[r][1]);
        }
    }
}

// ---------------------------------------------------------------------------
// The frame chain of one head, direction and slice of kSlice state columns
// (the columns are independent: P_f acts on each alike): S <- P_f (alpha_f S
// + B_f) per frame, in the direction's order.  The state each readout needs
// goes to `st` ([dir][F][B*H][DK][DV]): the causal direction stores S_f, the
// reverse one R_{f+1} (before the frame is written), as fp32 or (kImage) as
// the tensor-core readout's operand image.  Thread tile 4 rows x 2 columns;
// P_f (symmetric: row k of P is column k) and the slice of B_f are staged in
// shared memory, double-buffered: the next frame's are fetched (cp.async)
// while this frame's product runs.
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
    static constexpr int kP = 0;                           // 2 x [DK][DK]
    static constexpr int kB = kP + 2 * DK * DK * 4;        // 2 x [DK][kSlice]
    static constexpr int kS = kB + 2 * DK * kSlice * 4;    // [DK][kSlice]
    static constexpr int kBytes = kS + DK * kSlice * 4;
};

// 16-byte asynchronous copy global -> shared (completion by cp_async_wait_all)
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

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
    float *Bs = reinterpret_cast<float *>(csm + SM::kB);
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

    // the frame of step `stp`: P_f and the slice of B_f into buffer `buf`
    auto fetch = [&](int stp, int buf) {
        const int f = dir ? F - 1 - stp : stp;
        const size_t fh = (size_t)f * nbh + bh;
        const float *Pg = P + fh * DK * DK;
        float *Pd = Ps + buf * DK * DK;
        for (int e = tid * 4; e < DK * DK; e += kChainThreads * 4) cp_async16(Pd + e, Pg + e);
        float *Bd = Bs + buf * DK * kSlice;
        for (int e = tid * 4; e < DK * kSlice; e += kChainThreads * 4)
            cp_async16(Bd + e, Bm + fh * sdim + (size_t)(e / kSlice) * DV + j0 + e % kSlice);
        cp_async_commit();
    };
    auto alpha_of = [&](int stp) { return alpha_f[((size_t)b * F + (dir ? F - 1 - stp : stp)) * H + h]; };
    fetch(0, 0);
    float a_next = alpha_of(0);

    for (int step = 0; step < F; ++step) {
        const int f = dir ? F - 1 - step : step;
        const size_t fh = (size_t)f * nbh + bh;
        const float a = a_next;
        const int buf = step & 1;
        const float *Pf = Ps + buf * DK * DK, *Bf = Bs + buf * DK * kSlice;
        float *dst = st + ((size_t)dir * F * nbh + fh) * sdim;
        cp_async_wait_all();
        __syncthreads();                                   // P_f, B_f landed; S complete; the other buffers free
        if (step + 1 < F) {
            fetch(step + 1, buf ^ 1);
            a_next = alpha_of(step + 1);
        }
        if (dir) {                                         // the reverse readout of frame f reads R_{f+1}
            store_state(dst);
            __syncthreads();
        }
        for (int e = tid; e < DK * kSlice; e += kChainThreads) S[e] = fmaf(a, S[e], Bf[e]);   // S <- alpha S + B
        __syncthreads();
        float acc[TR][TCc];
        if (worker) {
#pragma unroll
            for (int r = 0; r < TR; ++r)
#pragma unroll
                for (int cc = 0; cc < TCc; ++cc) acc[r][cc] = 0.f;
#pragma unroll 8
            for (int kk = 0; kk < DK; ++kk) {
                const float4 pv = *reinterpret_cast<const float4 *>(Pf + kk * DK + i0);   // P[i0..][kk]
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
