// tc_kernels.cuh -- chunkwise gated delta-net scan on the sm_100a tensor
// cores (tcgen05 + TMEM, operands fed by TMA), one fused kernel.
//
// One CTA of 128 threads owns one (b, h) sequence, one direction and one
// slice of NS columns of the d_v dimension of the state; it walks the chunks
// of 64 tokens in order with its d_k x NS state slice on chip (fp32 master
// copy in registers, a tf32 copy in shared memory as an MMA operand).  The
// columns of the state evolve independently (the recurrence multiplies S only
// from the left), so slices of one head never communicate.
//
// Per chunk (processing order r = 0..63; the reverse pass walks a chunk back
// to front, which turns it into the forward recurrence over reversed rows):
//   g_r = sum_{m<=r} log alpha_m,  Gram  G = [K; Q] K^T        (kind::f16, bf16 in, exact)
//   L_rs = beta_r e^{g_r-g_s} (KK^T)_rs  (s<r),  P (readout mask, see below)
//   T = (I + L)^{-1}                                            (CUDA cores, fp32)
//   W = (T diag(beta e^g)) K,   U = (T diag(beta)) V_slice      (kind::tf32)
//   X = W S,  Y = Q S                                           (kind::tf32)
//   Delta = U - X
//   O = diag(dq) Y + P Delta                                    (kind::tf32)
//   S' = ds S + K^T (diag(dkk) Delta)                           (kind::tf32)
// forward: dq_r = e^{g_r},  P_rs = e^{g_r-g_s}(QK^T)_rs, s <= r
// reverse: dq_r = e^{g_{r-1}}, P_rs = e^{g_{r-1}-g_s}(QK^T)_rs, s < r (strict readout)
// dkk_s = e^{g_63 - g_s},  ds = e^{g_63}.  Every exponent is <= 0.
//
// Precision: every computed operand (T, W, U, P, Delta, S) enters the tensor
// cores as tf32 rounded to nearest; the Gram matrices use the bf16 inputs
// directly (products exact, fp32 accumulation).  bf16 rounding of P, U or S
// alone would move max|o - exact| / rms(o) past 1e-2 on long sequences.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace gdn {
namespace tc {

using namespace gdn::sm100;

#ifdef GDN_TC_DEBUG
// Development aid (not built into the library): CTA (0,0) copies the first
// chunk's intermediates here.
__device__ float g_tc_dbg[2048];
#define TC_DBG(cond, idx, val) do { if ((cond) && blockIdx.x == 0 && blockIdx.y == 0 && step == 0) g_tc_dbg[idx] = (val); } while (0)
#else
#define TC_DBG(cond, idx, val) do { } while (0)
#endif

constexpr int kDK = 128;        // key dimension handled by this kernel
constexpr int kThreads = 128;
constexpr uint32_t kWaitTries = 1u << 22;  // bounded mbarrier polls (seconds)

// Shared-memory plan for slice width NS (bytes).
template <int NS>
struct Smem {
    // TMA landing zone: two 64-column K-blocks of [K rows 0..63 | Q rows 0..63],
    // 128B-swizzled (bf16), then the V slice [64][NS] bf16.
    static constexpr int kStage = 0;
    static constexpr int kStageKQ = 2 * 2 * 64 * 128;             // 32768
    static constexpr int kStageV = kStage + kStageKQ;
    static constexpr int kStageBytes = kStageKQ + 64 * NS * 2;
    // scratch for the inverse, aliasing the landing zone once it is consumed
    static constexpr int kL = kStage;                              // [64][65] fp32
    static constexpr int kT = kL + 64 * 65 * 4;                    // [64][65] fp32
    static constexpr int kX = kT + 64 * 65 * 4;                    // 3 x [16][16] fp32
    static_assert(kX + 3 * 256 * 4 <= kStageBytes, "inverse scratch must fit the landing zone");
    // tf32 operands
    static constexpr int kKt = 36864;                              // K^T K-major  (MN d_k=128, K 64 rows)
    static constexpr int kQt = kKt + 128 * 64 * 4;                 // Q   K-major  (MN 64 rows, K d_k)
    static constexpr int kVt = kQt + 64 * 128 * 4;                 // V^T K-major  (MN NS, K 64 rows)
    static constexpr int kT1 = kVt + NS * 64 * 4;                  // T diag(b e^g)  K-major 64x64
    static constexpr int kT2 = kT1 + 64 * 64 * 4;                  // T diag(b)      K-major 64x64
    static constexpr int kWt = kT2 + 64 * 64 * 4;                  // W  K-major   (64 x 128)
    static constexpr int kPt = kWt + 64 * 128 * 4;                 // P  K-major   (64 x 64)
    static constexpr int kSt = kPt + 64 * 64 * 4;                  // S^T K-major (MN NS, K d_k)
    static constexpr int kDt = kSt + NS * 128 * 4;                 // Delta^T K-major (MN NS, K 64 rows)
    static constexpr int kDKt = kDt + NS * 64 * 4;                 // (dkk Delta)^T, same layout
    // per-chunk gate vectors and control words
    static constexpr int kGate = kDKt + NS * 64 * 4;               // g, beta, dq, dkk, b e^g
    static constexpr int kBar = kGate + 5 * 64 * 4;                // 2 mbarriers
    static constexpr int kCtl = kBar + 16;                         // tmem base, abort flag, ds
    static constexpr int kBytes = kCtl + 16;
    // requested dynamic size: the base is rounded up to 1024 bytes in the kernel
    static constexpr int kAlloc = kBytes + 1024;
    static_assert(kStageBytes <= kKt, "landing zone overlaps operands");
    static_assert(kAlloc <= 232448, "shared memory budget");
};

// TMEM columns of the accumulators.
constexpr uint32_t kColG = 0;      // 128 lanes x 64: rows 0..63 K K^T, rows 64..127 Q K^T
constexpr uint32_t kColW = 64;     // M=64 x 128
constexpr uint32_t kColU = 192;    // M=64 x NS
constexpr uint32_t kColX = 224;    // M=64 x NS
constexpr uint32_t kColY = 256;    // M=64 x NS
constexpr uint32_t kColP = 288;    // M=64 x NS
constexpr uint32_t kColS = 320;    // M=128 x NS
constexpr uint32_t kTmemCols = 512;

// Byte offsets inside the operand layouts (see sm100.cuh).  Every tf32
// operand is K-major (tcgen05 kind::tf32 produced no result with MN-major
// operands on this hardware; kind::f16 takes either).
// K-major tf32 tile of MN extent E: offset(mn, k) = (k/4)*(E*16) + mn*16 + (k%4)*4,
// i.e. leading byte offset (between K cells) E*16, stride byte offset 128.
template <int E>
__device__ __forceinline__ int kmaj(int mn, int k) { return (k >> 2) * (E * 16) + mn * 16 + (k & 3) * 4; }
__device__ __forceinline__ int kmaj64(int mn, int k) { return kmaj<64>(mn, k); }

__device__ __forceinline__ float4 tf32x4(float a, float b, float c, float d) {
    return make_float4(to_tf32(a), to_tf32(b), to_tf32(c), to_tf32(d));
}

// Output modes (bidirectional pairs write a partial, then add to it).
enum OutMode { kOutStore = 0, kOutPartial = 1, kOutAddPartial = 2 };

// grid (DV/NS, B*H), block 128, dynamic smem Smem<NS>::kBytes.
template <int DV, int NS, bool REV, typename Tout>
__global__ void __launch_bounds__(kThreads, 1)
scan_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
            const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ alpha,
            const float *__restrict__ beta, const float *__restrict__ state_in,
            float *__restrict__ state_out, Tout *__restrict__ o, float *__restrict__ part,
            int T, int H, int nC, int out_mode, unsigned int *__restrict__ err)
{
    using SM = Smem<NS>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    // 128B-swizzled TMA tiles and their MMA descriptors need a 1024-byte
    // aligned shared-memory address
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    unsigned char *stage = smem + SM::kStage;
    float *Lsm = reinterpret_cast<float *>(smem + SM::kL);
    float *Tsm = reinterpret_cast<float *>(smem + SM::kT);
    float *Xsm = reinterpret_cast<float *>(smem + SM::kX);
    float *g_s = reinterpret_cast<float *>(smem + SM::kGate);
    float *beta_s = g_s + 64;
    float *dq_s = g_s + 128;
    float *dkk_s = g_s + 192;
    float *bg_s = g_s + 256;
    uint64_t *tma_bar = reinterpret_cast<uint64_t *>(smem + SM::kBar);
    uint64_t *mma_bar = tma_bar + 1;
    uint32_t *tmem_base_s = reinterpret_cast<uint32_t *>(smem + SM::kCtl);
    volatile int *abort_s = reinterpret_cast<volatile int *>(smem + SM::kCtl + 4);
    float *ds_s = reinterpret_cast<float *>(smem + SM::kCtl + 8);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slice = blockIdx.x, bh = blockIdx.y;
    const int b = bh / H, h = bh % H;
    const int j0 = slice * NS;
    const uint32_t sbase = smem_u32(smem);

    if (tid == 0) {
        mbar_init(tma_bar, 1);
        mbar_init(mma_bar, 1);
        fence_mbar_init();
        *abort_s = 0;
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(tmem_base_s, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_s;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;   // this warp's TMEM lane quarter

    // state slice: thread d holds row d (fp32), tf32 copy to the B operand St
    float S[NS];
    {
        const float *src = state_in ? state_in + ((size_t)bh * kDK + tid) * DV + j0 : nullptr;
#pragma unroll
        for (int n = 0; n < NS; ++n) S[n] = src ? src[n] : 0.f;
        unsigned char *St = smem + SM::kSt;
#pragma unroll
        for (int n = 0; n < NS; ++n) *reinterpret_cast<float *>(St + kmaj<NS>(n, tid)) = to_tf32(S[n]);
    }

    auto issue_tma = [&](int c) {
        mbar_arrive_expect_tx(tma_bar, SM::kStageBytes);
        const int t0 = c * 64;
        tma_load_4d(stage + 0, &tm_k, tma_bar, 0, h, t0, b);
        tma_load_4d(stage + 16384, &tm_k, tma_bar, 64, h, t0, b);
        tma_load_4d(stage + 8192, &tm_q, tma_bar, 0, h, t0, b);
        tma_load_4d(stage + 16384 + 8192, &tm_q, tma_bar, 64, h, t0, b);
        tma_load_4d(stage + SM::kStageV, &tm_v, tma_bar, j0, h, t0, b);
    };
    // bounded wait on a barrier by every thread; a timeout anywhere aborts the CTA
    auto wait_all = [&](uint64_t *bar, uint32_t parity) {
        if (!mbar_wait(bar, parity, kWaitTries)) {
            *abort_s = 1;
            if (err) atomicAdd(err, 1u);
        }
    };

    if (tid == 0) issue_tma(REV ? nC - 1 : 0);
    uint32_t tma_phase = 0, mma_phase = 0;

    for (int step = 0; step < nC; ++step) {
        const int c = REV ? nC - 1 - step : step;
        // ---- gates of this chunk (processing order) ------------------------------
        if (tid < 64) {
            const int t = token_of_row(c, tid, REV ? 1 : 0);
            const size_t off = ((size_t)b * T + t) * H + h;
            g_s[tid] = t < T ? __logf(alpha[off]) : 0.f;
            beta_s[tid] = t < T ? beta[off] : 0.f;
        }
        wait_all(tma_bar, tma_phase);
        tma_phase ^= 1;
        __syncthreads();
        TC_DBG(tid == 0, 0, (float)*abort_s);
        TC_DBG(tid < 64, 1600 + tid, __uint_as_float(reinterpret_cast<const uint32_t *>(stage)[tid]));
        if (*abort_s) break;
        if (warp == 0) {  // inclusive prefix sum of log alpha over 64 rows (2 per lane)
            float a0 = g_s[2 * lane], a1 = g_s[2 * lane + 1];
            float s = a0 + a1;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, s, d);
                if (lane >= d) s += y;
            }
            const float ex = s - (a0 + a1);   // exclusive prefix of pairs
            g_s[2 * lane] = ex + a0;
            g_s[2 * lane + 1] = ex + a0 + a1;
        }
        // ---- bf16 landing tiles -> tf32 operand layouts ----------------------------
        {
            const unsigned char *kst = stage;
            float *Kt = reinterpret_cast<float *>(smem + SM::kKt);
            // K^T, K-major (MN = d, K = row): cell (d, rows r0..r0+3)
            for (int cell = tid; cell < 128 * 16; cell += kThreads) {
                const int d = cell & 127, r0 = (cell >> 7) * 4;
                const int kb = d >> 6, col = d & 63;
                float v[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int f = REV ? 63 - (r0 + e) : r0 + e;       // forward row in the tile
                    const unsigned char *src = kst + kb * 16384 + f * 128 +
                                               ((((col >> 3) ^ (f & 7))) << 4) + (col & 7) * 2;
                    v[e] = __uint_as_float((uint32_t)(*reinterpret_cast<const uint16_t *>(src)) << 16);
                }
                *reinterpret_cast<float4 *>(reinterpret_cast<unsigned char *>(Kt) + kmaj<128>(d, r0)) =
                    make_float4(v[0], v[1], v[2], v[3]);
            }
            // Q as K-major (MN = row, K = d_k): cell (r, d/4)
            float *Qt = reinterpret_cast<float *>(smem + SM::kQt);
            for (int cell = tid; cell < 64 * 32; cell += kThreads) {
                const int r = cell & 63, dc = cell >> 6;
                const int f = REV ? 63 - r : r;
                const int d = dc * 4;
                const int kb = d >> 6, col = d & 63;
                const unsigned char *src = kst + kb * 16384 + 8192 + f * 128 +
                                           ((((col >> 3) ^ (f & 7))) << 4) + (col & 7) * 2;
                const uint2 raw = *reinterpret_cast<const uint2 *>(src);
                const float v0 = __uint_as_float(raw.x << 16), v1 = __uint_as_float(raw.x & 0xffff0000u);
                const float v2 = __uint_as_float(raw.y << 16), v3 = __uint_as_float(raw.y & 0xffff0000u);
                *reinterpret_cast<float4 *>(reinterpret_cast<unsigned char *>(Qt) + kmaj64(r, d)) =
                    make_float4(v0, v1, v2, v3);
            }
            // V^T slice, K-major (MN = n, K = row); landing tile is [64][NS] bf16
            float *Vt = reinterpret_cast<float *>(smem + SM::kVt);
            for (int cell = tid; cell < NS * 16; cell += kThreads) {
                const int n = cell % NS, r0 = (cell / NS) * 4;
                float v[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int f = REV ? 63 - (r0 + e) : r0 + e;
                    v[e] = __uint_as_float((uint32_t)(*reinterpret_cast<const uint16_t *>(
                               stage + SM::kStageV + (f * NS + n) * 2)) << 16);
                }
                *reinterpret_cast<float4 *>(reinterpret_cast<unsigned char *>(Vt) + kmaj<NS>(n, r0)) =
                    make_float4(v[0], v[1], v[2], v[3]);
            }
        }
        __syncthreads();  // g complete, conversions complete
        if (tid < 64) {
            const float gr = g_s[tid], gl = g_s[63];
            dq_s[tid] = REV ? (tid > 0 ? __expf(g_s[tid - 1]) : 1.f) : __expf(gr);
            dkk_s[tid] = __expf(gl - gr);
            bg_s[tid] = beta_s[tid] * __expf(gr);
            if (tid == 0) *ds_s = __expf(gl);
        }
        fence_async_shared();
        __syncthreads();
        // ---- Gram matrices on the tensor cores (bf16, exact products) -------------
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t id = idesc(128, 64, 1, 0, 0);
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint32_t a = sbase + SM::kStage + (s >> 2) * 16384 + (s & 3) * 32;
                mma_bf16(tmem + kColG, sdesc_sw128(a), sdesc_sw128(a), id, s > 0);
            }
            mma_commit(mma_bar);
        }
        wait_all(mma_bar, mma_phase);
        mma_phase ^= 1;
        tc_fence_after();
        // ---- L and P from the Gram accumulator ------------------------------------
        {
            float G[64];
#pragma unroll
            for (int q = 0; q < 4; ++q) tmem_ld16(tmem + lane_base + kColG + q * 16, G + q * 16);
            tmem_wait_ld();
#pragma unroll
            for (int f = 0; f < 64; ++f) {
                TC_DBG(tid == 0, 64 + f, G[f]);
                TC_DBG(tid == 64, 128 + f, G[f]);
            }
            TC_DBG(tid == 0, 1, (float)tmem);
            const int fl = tid & 63;                   // forward row of this lane
            const int r = REV ? 63 - fl : fl;          // processing row
            const float gr = g_s[r];
            if (tid < 64) {
                const float br = beta_s[r];
#pragma unroll
                for (int f = 0; f < 64; ++f) {
                    const int s = REV ? 63 - f : f;
                    Lsm[r * 65 + s] = s < r ? br * __expf(gr - g_s[s]) * G[f] : 0.f;
                }
            } else {
                const float gq = REV ? (r > 0 ? g_s[r - 1] : 0.f) : gr;
                unsigned char *Pt = smem + SM::kPt;
#pragma unroll
                for (int sc = 0; sc < 16; ++sc) {
                    float v[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int s = sc * 4 + e;
                        const int f = REV ? 63 - s : s;
                        const bool keep = REV ? (s < r) : (s <= r);
                        v[e] = keep ? __expf(gq - g_s[s]) * G[f] : 0.f;
                    }
                    *reinterpret_cast<float4 *>(Pt + kmaj64(r, sc * 4)) = tf32x4(v[0], v[1], v[2], v[3]);
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        // ---- T = (I + L)^{-1}, blocked 16 x 16 -------------------------------------
        {
            // diagonal blocks by forward substitution: thread (blk, j) owns column j
            if (tid < 64) {
                const int blk = tid >> 4, j = tid & 15, o0 = blk * 16;
                float x[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float acc = (i == j) ? 1.f : 0.f;
#pragma unroll
                    for (int m = 0; m < i; ++m) acc = fmaf(-Lsm[(o0 + i) * 65 + o0 + m], x[m], acc);
                    x[i] = acc;
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) Tsm[(o0 + i) * 65 + o0 + j] = x[i];
            } else {
                // zero the strictly upper blocks
                for (int e = tid - 64; e < 64 * 64; e += 64) {
                    const int i = e >> 6, jj = e & 63;
                    if ((jj >> 4) > (i >> 4)) Tsm[i * 65 + jj] = 0.f;
                }
            }
            __syncthreads();
            // off-diagonal blocks, one diagonal band at a time:
            //   T_ij = -T_ii * sum_{k=j}^{i-1} L_ik T_kj
            for (int band = 1; band < 4; ++band) {
                const int nblk = 4 - band;                 // blocks (j+band, j), j < nblk
                for (int e = tid; e < nblk * 256; e += kThreads) {
                    const int j = e >> 8, ii = (e >> 4) & 15, jj = e & 15;
                    const int i = j + band;
                    float acc = 0.f;
                    for (int k = j; k < i; ++k) {
#pragma unroll
                        for (int m = 0; m < 16; ++m)
                            acc = fmaf(Lsm[(i * 16 + ii) * 65 + k * 16 + m], Tsm[(k * 16 + m) * 65 + j * 16 + jj], acc);
                    }
                    Xsm[j * 256 + ii * 16 + jj] = acc;
                }
                __syncthreads();
                for (int e = tid; e < nblk * 256; e += kThreads) {
                    const int j = e >> 8, ii = (e >> 4) & 15, jj = e & 15;
                    const int i = j + band;
                    float acc = 0.f;
#pragma unroll
                    for (int m = 0; m < 16; ++m)
                        acc = fmaf(Tsm[(i * 16 + ii) * 65 + i * 16 + m], Xsm[j * 256 + m * 16 + jj], acc);
                    Tsm[(i * 16 + ii) * 65 + j * 16 + jj] = -acc;
                }
                __syncthreads();
            }
            TC_DBG(tid < 64, 192 + tid, Tsm[5 * 65 + tid]);
            TC_DBG(tid < 64, 1700 + tid, Tsm[tid * 65 + 3]);
            // A operands T diag(beta e^g) and T diag(beta), tf32, K-major 64 x 64
            unsigned char *T1 = smem + SM::kT1;
            unsigned char *T2 = smem + SM::kT2;
            for (int cell = tid; cell < 64 * 16; cell += kThreads) {
                const int r = cell & 63, s = (cell >> 6) * 4;
                const float t0 = Tsm[r * 65 + s], t1 = Tsm[r * 65 + s + 1];
                const float t2 = Tsm[r * 65 + s + 2], t3 = Tsm[r * 65 + s + 3];
                *reinterpret_cast<float4 *>(T1 + kmaj64(r, s)) =
                    tf32x4(t0 * bg_s[s], t1 * bg_s[s + 1], t2 * bg_s[s + 2], t3 * bg_s[s + 3]);
                *reinterpret_cast<float4 *>(T2 + kmaj64(r, s)) =
                    tf32x4(t0 * beta_s[s], t1 * beta_s[s + 1], t2 * beta_s[s + 2], t3 * beta_s[s + 3]);
            }
        }
        fence_async_shared();
        __syncthreads();
        // the landing zone is free again: fetch the next chunk while this one finishes
        if (tid == 0 && step + 1 < nC) issue_tma(REV ? c - 1 : c + 1);
        // ---- W = T1 K, U = T2 V ------------------------------------------------------
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idw = idesc(64, 128, 2, 0, 0);
            constexpr uint32_t idu = idesc(64, NS, 2, 0, 0);
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                mma_tf32(tmem + kColW, sdesc_noswz(sbase + SM::kT1 + 2 * s * 1024, 1024, 128),
                         sdesc_noswz(sbase + SM::kKt + 2 * s * 2048, 2048, 128), idw, s > 0);
                mma_tf32(tmem + kColU, sdesc_noswz(sbase + SM::kT2 + 2 * s * 1024, 1024, 128),
                         sdesc_noswz(sbase + SM::kVt + 2 * s * (NS * 16), NS * 16, 128), idu, s > 0);
            }
            mma_commit(mma_bar);
        }
        wait_all(mma_bar, mma_phase);
        mma_phase ^= 1;
        tc_fence_after();
        // M=64 accumulators: row 16*warp + lane sits in lane 32*warp + lane (lane < 16)
        const bool row_lane = lane < 16;
        const int r64 = warp * 16 + lane;
        float U[NS];
        {
            unsigned char *Wt = smem + SM::kWt;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                float w[16];
                tmem_ld16(tmem + lane_base + kColW + q * 16, w);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) TC_DBG(tid == 0, 256 + q * 16 + e, w[e]);
                if (row_lane) {
#pragma unroll
                    for (int e = 0; e < 16; e += 4)
                        *reinterpret_cast<float4 *>(Wt + kmaj64(r64, q * 16 + e)) =
                            tf32x4(w[e], w[e + 1], w[e + 2], w[e + 3]);
                }
            }
#pragma unroll
            for (int q = 0; q < NS / 16; ++q) tmem_ld16(tmem + lane_base + kColU + q * 16, U + q * 16);
            tmem_wait_ld();
#pragma unroll
            for (int n = 0; n < NS; ++n) TC_DBG(tid == 0, 384 + n, U[n]);
        }
        fence_async_shared();
        tc_fence_before();
        __syncthreads();
        // ---- X = W S, Y = Q S ----------------------------------------------------------
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t id = idesc(64, NS, 2, 0, 0);
#pragma unroll
            for (int s = 0; s < 16; ++s) {
                const uint64_t bd = sdesc_noswz(sbase + SM::kSt + 2 * s * (NS * 16), NS * 16, 128);
                mma_tf32(tmem + kColX, sdesc_noswz(sbase + SM::kWt + 2 * s * 1024, 1024, 128), bd, id, s > 0);
                mma_tf32(tmem + kColY, sdesc_noswz(sbase + SM::kQt + 2 * s * 1024, 1024, 128), bd, id, s > 0);
            }
            mma_commit(mma_bar);
        }
        wait_all(mma_bar, mma_phase);
        mma_phase ^= 1;
        tc_fence_after();
        float Y[NS];
        {
            float X[NS];
#pragma unroll
            for (int q = 0; q < NS / 16; ++q) {
                tmem_ld16(tmem + lane_base + kColX + q * 16, X + q * 16);
                tmem_ld16(tmem + lane_base + kColY + q * 16, Y + q * 16);
            }
            tmem_wait_ld();
#pragma unroll
            for (int n = 0; n < NS; ++n) { TC_DBG(tid == 0, 416 + n, X[n]); TC_DBG(tid == 0, 448 + n, Y[n]); }
            if (row_lane) {
                unsigned char *Dt = smem + SM::kDt;
                unsigned char *DKt = smem + SM::kDKt;
                const float dk = dkk_s[r64];
#pragma unroll
                for (int n = 0; n < NS; n += 4) {
                    const float d0 = U[n] - X[n], d1 = U[n + 1] - X[n + 1];
                    const float d2 = U[n + 2] - X[n + 2], d3 = U[n + 3] - X[n + 3];
                    *reinterpret_cast<float *>(Dt + kmaj<NS>(n, r64)) = to_tf32(d0);
                    *reinterpret_cast<float *>(Dt + kmaj<NS>(n + 1, r64)) = to_tf32(d1);
                    *reinterpret_cast<float *>(Dt + kmaj<NS>(n + 2, r64)) = to_tf32(d2);
                    *reinterpret_cast<float *>(Dt + kmaj<NS>(n + 3, r64)) = to_tf32(d3);
                    *reinterpret_cast<float *>(DKt + kmaj<NS>(n, r64)) = to_tf32(dk * d0);
                    *reinterpret_cast<float *>(DKt + kmaj<NS>(n + 1, r64)) = to_tf32(dk * d1);
                    *reinterpret_cast<float *>(DKt + kmaj<NS>(n + 2, r64)) = to_tf32(dk * d2);
                    *reinterpret_cast<float *>(DKt + kmaj<NS>(n + 3, r64)) = to_tf32(dk * d3);
                }
            }
        }
        fence_async_shared();
        tc_fence_before();
        __syncthreads();
        // ---- P Delta and K^T (dkk Delta) -----------------------------------------------
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idp = idesc(64, NS, 2, 0, 0);
            constexpr uint32_t ids = idesc(128, NS, 2, 0, 0);
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint32_t boff = 2 * s * (NS * 16);
                mma_tf32(tmem + kColP, sdesc_noswz(sbase + SM::kPt + 2 * s * 1024, 1024, 128),
                         sdesc_noswz(sbase + SM::kDt + boff, NS * 16, 128), idp, s > 0);
                mma_tf32(tmem + kColS, sdesc_noswz(sbase + SM::kKt + 2 * s * 2048, 2048, 128),
                         sdesc_noswz(sbase + SM::kDKt + boff, NS * 16, 128), ids, s > 0);
            }
            mma_commit(mma_bar);
        }
        wait_all(mma_bar, mma_phase);
        mma_phase ^= 1;
        tc_fence_after();
        {
            // output rows
            float Pd[NS];
#pragma unroll
            for (int q = 0; q < NS / 16; ++q) tmem_ld16(tmem + lane_base + kColP + q * 16, Pd + q * 16);
            // state rows (all 128 lanes)
            float Sd[NS];
#pragma unroll
            for (int q = 0; q < NS / 16; ++q) tmem_ld16(tmem + lane_base + kColS + q * 16, Sd + q * 16);
            tmem_wait_ld();
#pragma unroll
            for (int n = 0; n < NS; ++n) { TC_DBG(tid == 0, 480 + n, Pd[n]); TC_DBG(tid == 0, 512 + n, Sd[n]); }
            if (row_lane) {
                const int t = token_of_row(c, r64, REV ? 1 : 0);
                if (t < T) {
                    const float dq = dq_s[r64];
                    const size_t off = (((size_t)b * T + t) * H + h) * DV + j0;
#pragma unroll
                    for (int n = 0; n < NS; n += 4) {
                        float4 v = make_float4(fmaf(dq, Y[n], Pd[n]), fmaf(dq, Y[n + 1], Pd[n + 1]),
                                               fmaf(dq, Y[n + 2], Pd[n + 2]), fmaf(dq, Y[n + 3], Pd[n + 3]));
                        if (out_mode == kOutPartial) {
                            *reinterpret_cast<float4 *>(part + off + n) = v;
                        } else {
                            if (out_mode == kOutAddPartial) {
                                const float4 p = *reinterpret_cast<const float4 *>(part + off + n);
                                v.x += p.x; v.y += p.y; v.z += p.z; v.w += p.w;
                            }
                            o[off + n] = from_f32<Tout>(v.x);
                            o[off + n + 1] = from_f32<Tout>(v.y);
                            o[off + n + 2] = from_f32<Tout>(v.z);
                            o[off + n + 3] = from_f32<Tout>(v.w);
                        }
                    }
                }
            }
            const float dsv = *ds_s;
            unsigned char *St = smem + SM::kSt;
#pragma unroll
            for (int n = 0; n < NS; n += 4) {
                S[n] = fmaf(dsv, S[n], Sd[n]);
                S[n + 1] = fmaf(dsv, S[n + 1], Sd[n + 1]);
                S[n + 2] = fmaf(dsv, S[n + 2], Sd[n + 2]);
                S[n + 3] = fmaf(dsv, S[n + 3], Sd[n + 3]);
                *reinterpret_cast<float *>(St + kmaj<NS>(n, tid)) = to_tf32(S[n]);
                *reinterpret_cast<float *>(St + kmaj<NS>(n + 1, tid)) = to_tf32(S[n + 1]);
                *reinterpret_cast<float *>(St + kmaj<NS>(n + 2, tid)) = to_tf32(S[n + 2]);
                *reinterpret_cast<float *>(St + kmaj<NS>(n + 3, tid)) = to_tf32(S[n + 3]);
            }
        }
        fence_async_shared();
        tc_fence_before();
        __syncthreads();
    }

    if (*abort_s) {
        // a wait timed out: let any copy or MMA still in flight land (bounded)
        // before the shared memory and the TMEM of this CTA are released
        mbar_wait(tma_bar, tma_phase, 1u << 16);
        mbar_wait(mma_bar, mma_phase, 1u << 16);
    } else if (state_out) {
        float *dst = state_out + ((size_t)bh * kDK + tid) * DV + j0;
#pragma unroll
        for (int n = 0; n < NS; ++n) dst[n] = S[n];
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace tc
}  // namespace gdn
