// vda_tc.cuh -- the frame-wise operator's key Gram and key-value products on
// the tensor cores (bf16 inputs, d_k = 128):
//   A_f = K_f^T diag(beta) K_f   (128 x 128),   B_f = K_f^T diag(beta) V_f   (128 x DV)
// as one tcgen05 contraction over the frame's tokens, 64 at a time:
//   [D_A | D_B] += K_c^T [ (beta K_c)_hi | (beta K_c)_lo | (beta V_c)_hi | (beta V_c)_lo ]
// M = 128 (the key index, TMEM lanes), K = the chunk's tokens, N = 2*128 for
// A and 2*DV for B (two MMAs per 16 tokens).  K_c^T is the TMA tile of K read
// MN-major; the beta-scaled operands are formed in shared memory as bf16
// hi/lo pairs (x = hi + lo to about 2^-16), so the only rounding of the
// products is the fp32 accumulation.  Tokens past the frame's end enter with
// beta = 0.  Two stages: the TMA of chunk c+1 and the operand forming of
// chunk c overlap the MMAs of chunk c-1.  Every wait is bounded.
#pragma once

#include "tc_common.cuh"
#include "vda.cuh"

namespace gdn {
namespace vda {

using namespace gdn::sm100;
using gdn::tc2::bulk_load;
using gdn::tc2::kWaitTries;
using gdn::tc2::sdesc_sw128_mn;
using gdn::tc2::split2;
using gdn::tc2::swz128;

constexpr int kTcThreads = 256;
constexpr unsigned long long kTcWaitNs = 1000000000ull;   // a wait here gives up after 1 s

template <int DV>
struct GramTcSmem {
    static constexpr int kK = 0;                           // K tile: 2 x [64 tok][64] bf16, 128B swizzle
    static constexpr int kV = kK + 16384;                  // V tile: DV/64 blocks
    static constexpr int kBK = kV + DV * 128;              // [tok][256] operand: 4 groups of 64 columns
    static constexpr int kBV = kBK + 4 * 8192;             // [tok][2*DV] operand
    static constexpr int kStage = kBV + (2 * DV / 64) * 8192;
    static constexpr int kBeta = 2 * kStage;               // [2][64] fp32
    static constexpr int kBar = kBeta + 2 * 64 * 4;        // full[2], free[2], done
    static constexpr int kCtl = kBar + 64;                 // tmem base, abort
    static constexpr int kBytes = kCtl + 16;
    static constexpr int kAlloc = kBytes + 1024;
    static_assert(kStage % 1024 == 0, "stages stay 1024-aligned");
};

template <int DV>
__global__ void __launch_bounds__(kTcThreads, 1)
vda_gram_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const float *__restrict__ beta, float *__restrict__ A, float *__restrict__ Bm, int F, int U,
                   int H, unsigned int *__restrict__ err)
{
    using SM = GramTcSmem<DV>;
    constexpr int NB = 2 * DV;                             // columns of the B part
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + SM::kBar);
    uint64_t *freeb = full + 2;
    uint64_t *done = full + 4;
    uint32_t *tmem_s = reinterpret_cast<uint32_t *>(smem + SM::kCtl);
    volatile int *abort_s = reinterpret_cast<volatile int *>(smem + SM::kCtl + 4);
    float *beta_s = reinterpret_cast<float *>(smem + SM::kBeta);
    const int f = blockIdx.x, bh = blockIdx.y, b = bh / H, h = bh % H;
    const int T = F * U, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nch = (U + 63) / 64;
    const uint32_t sbase = smem_u32(smem);

    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(&freeb[0], 1);
        mbar_init(&freeb[1], 1);
        mbar_init(done, 1);
        fence_mbar_init();
        *abort_s = 0;
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(tmem_s, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_s;

    auto wait_ok = [&](uint64_t *bar, uint32_t parity) {
        if (!mbar_wait_ns(bar, parity, kTcWaitNs)) {
            *abort_s = 1;
            if (err) atomicAdd(err, 1u);
            return false;
        }
        return true;
    };
    auto issue = [&](int c) {   // TMA of chunk c into stage c & 1
        unsigned char *st = smem + (c & 1) * SM::kStage;
        uint64_t *bar = &full[c & 1];
        mbar_arrive_expect_tx(bar, 16384 + DV * 128);
        const int t0 = f * U + c * 64;
        tma_load_4d(st + SM::kK, &tm_k, bar, 0, h, t0, b);
        tma_load_4d(st + SM::kK + 8192, &tm_k, bar, 64, h, t0, b);
#pragma unroll
        for (int vb = 0; vb < DV / 64; ++vb) tma_load_4d(st + SM::kV + vb * 8192, &tm_v, bar, vb * 64, h, t0, b);
    };
    if (tid == 0) issue(0);
    constexpr uint32_t idA = idesc(128, 256, 1, 1, 1);     // A MN-major (K tile), B MN-major
    constexpr uint32_t idB = idesc(128, NB, 1, 1, 1);
    uint32_t full_ph = 0, free_ph = 0;

    for (int c = 0; c < nch; ++c) {
        const int s = c & 1;
        unsigned char *st = smem + s * SM::kStage;
        if (tid == 0 && c + 1 < nch) {
            if (c >= 1) {   // chunk c-1's MMAs are done with stage (c+1) & 1
                wait_ok(&freeb[(c + 1) & 1], (free_ph >> ((c + 1) & 1)) & 1u);
                free_ph ^= 1u << ((c + 1) & 1);
            }
            if (!*abort_s) issue(c + 1);
        }
        // this chunk's write strengths (0 past the frame's end)
        if (tid < 64) {
            const int u = c * 64 + tid;
            beta_s[s * 64 + tid] = u < U ? beta[((size_t)b * T + (size_t)f * U + u) * H + h] : 0.f;
        }
        wait_ok(&full[s], (full_ph >> s) & 1u);
        full_ph ^= 1u << s;
        __syncthreads();                                   // beta_s visible; abort seen by all
        if (*abort_s) break;
        // ---- operands: (beta x)_hi | (beta x)_lo, 16 bytes (8 columns) per step
        for (int e = tid; e < 64 * (128 + DV) / 8; e += kTcThreads) {
            const int k = e / ((128 + DV) / 8), col = (e % ((128 + DV) / 8)) * 8;   // token, column of [K | V]
            const bool isk = col < 128;
            const int n = isk ? col : col - 128;
            const unsigned char *src = st + (isk ? SM::kK : SM::kV) + (n >> 6) * 8192;
            const uint4 raw = *reinterpret_cast<const uint4 *>(src + swz128(k * 128 + (n & 63) * 2));
            const float bt = beta_s[s * 64 + k];
            const __nv_bfloat162 *pr = reinterpret_cast<const __nv_bfloat162 *>(&raw);
            uint4 hi, lo;
            uint32_t *ph = reinterpret_cast<uint32_t *>(&hi), *pl = reinterpret_cast<uint32_t *>(&lo);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 x = __bfloat1622float2(pr[q]);
                split2(bt * x.x, bt * x.y, ph[q], pl[q]);
            }
            const int w = isk ? 128 : DV;                  // hi at column n, lo at n + w
            unsigned char *dst = st + (isk ? SM::kBK : SM::kBV);
            *reinterpret_cast<uint4 *>(dst + (n >> 6) * 8192 + swz128(k * 128 + (n & 63) * 2)) = hi;
            *reinterpret_cast<uint4 *>(dst + ((n + w) >> 6) * 8192 + swz128(k * 128 + ((n + w) & 63) * 2)) = lo;
        }
        fence_async_shared();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t sa = sbase + s * SM::kStage;
            const uint64_t dK = sdesc_sw128_mn(sa + SM::kK, 8192);
            const uint64_t dBK = sdesc_sw128_mn(sa + SM::kBK, 8192);
            const uint64_t dBV = sdesc_sw128_mn(sa + SM::kBV, 8192);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {               // 16 tokens per MMA
                const uint32_t acc = (c > 0 || ks > 0) ? 1u : 0u;
                const uint64_t a = dK + (uint64_t)((ks * 2048) >> 4);
                mma_bf16(tmem, a, dBK + (uint64_t)((ks * 2048) >> 4), idA, acc);
                mma_bf16(tmem + 256, a, dBV + (uint64_t)((ks * 2048) >> 4), idB, acc);
            }
            mma_commit(&freeb[s]);
            if (c + 1 == nch) mma_commit(done);
        }
    }
    // ---- epilogue: A = D[:, 0:128] + D[:, 128:256], B = D[:, 256:256+DV] + D[:, 256+DV:256+2DV]
    if (!*abort_s) {
        if (tid == 0) wait_ok(done, 0);
        __syncthreads();
    }
    tc_fence_after();
    if (!*abort_s) {
        const int quarter = warp & 3, half = warp >> 2;    // half 0: A, half 1: B
        const int row = quarter * 32 + lane;
        const uint32_t lb = (uint32_t)(quarter * 32) << 16;
        const size_t fh = (size_t)f * gridDim.y + bh;
        const int ncol = half ? DV : 128;
        const uint32_t base = half ? 256u : 0u;
        float *dst = half ? Bm + (fh * 128 + row) * DV : A + (fh * 128 + row) * 128;
        for (int n0 = 0; n0 < ncol; n0 += 16) {
            float hi[16], lo[16];
            tmem_ld16(tmem + lb + base + n0, hi);
            tmem_ld16(tmem + lb + base + ncol + n0, lo);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 16; q += 4)
                *reinterpret_cast<float4 *>(dst + n0 + q) =
                    make_float4(hi[q] + lo[q], hi[q + 1] + lo[q + 1], hi[q + 2] + lo[q + 2], hi[q + 3] + lo[q + 3]);
        }
    } else if (tid == 0) {
        // a wait gave up: let MMAs and copies in flight land before shared memory and TMEM go
        mbar_wait(&full[0], 0, 64);
        mbar_wait(&full[1], 0, 64);
        mbar_wait(done, 0, 64);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace vda
}  // namespace gdn

namespace gdn {
namespace vda {

// ---------------------------------------------------------------------------
// Readout on the tensor cores: 128 tokens of one frame per CTA,
//   D = Q [S_hi | S_lo] (+ Q [R_hi | R_lo]),   o = D[:, :DV] + D[:, DV:]
// M = 128 tokens (TMEM lanes), K = d_k = 128, N = 2*DV.  Q is four TMA tiles
// (two token halves x two key halves) read K-major; the state images are
// the chain's operand images (img_off), fetched by bulk copies.  Rows past
// the frame's end are computed but not stored.
// ---------------------------------------------------------------------------
// Four consecutive outputs with one vector store (16 B fp32, 8 B bf16).
__device__ __forceinline__ void store4(float *p, float a, float b, float c, float d) {
    *reinterpret_cast<float4 *>(p) = make_float4(a, b, c, d);
}
__device__ __forceinline__ void store4(__nv_bfloat16 *p, float a, float b, float c, float d) {
    uint2 v;
    v.x = gdn::tc2::pack_bf16(a, b);
    v.y = gdn::tc2::pack_bf16(c, d);
    *reinterpret_cast<uint2 *>(p) = v;
}

template <int DV>
struct ReadTcSmem {
    static constexpr int kQ = 0;                           // 2 key halves x [128 tok][64] bf16
    static constexpr int kImg = 32768;                     // [ndir] images of 128 x 2*DV bf16
    static constexpr int kImgBytes = 128 * DV * 4;
    static constexpr int kBar = kImg + 2 * kImgBytes;      // loaded, done
    static constexpr int kCtl = kBar + 16;                 // tmem base, abort
    static constexpr int kBytes = kCtl + 16;
    static constexpr int kAlloc = kBytes + 1024;
};

template <int DV, typename Tout>
__global__ void __launch_bounds__(128, 1)
vda_readout_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const unsigned char *__restrict__ img,
                      Tout *__restrict__ o, int F, int U, int H, int ndir, unsigned int *__restrict__ err)
{
    using SM = ReadTcSmem<DV>;
    constexpr int NB = 2 * DV;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *loaded = reinterpret_cast<uint64_t *>(smem + SM::kBar);
    uint64_t *done = loaded + 1;
    uint32_t *tmem_s = reinterpret_cast<uint32_t *>(smem + SM::kCtl);
    volatile int *abort_s = reinterpret_cast<volatile int *>(smem + SM::kCtl + 4);
    const int nblk = (U + 127) / 128;
    const int f = blockIdx.x / nblk, u0 = (blockIdx.x % nblk) * 128;
    const int bh = blockIdx.y, nbh = gridDim.y, b = bh / H, h = bh % H;
    const int T = F * U, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t sbase = smem_u32(smem);
    const size_t ibytes = SM::kImgBytes;

    if (tid == 0) {
        mbar_init(loaded, 1);
        mbar_init(done, 1);
        fence_mbar_init();
        *abort_s = 0;
        prefetch_tensormap(&tm_q);
        // a token half that starts past the end of the sequence is not fetched
        // (its rows are past the frame too and never stored): it stays as is
        const int t0 = f * U + u0;
        const int halves = t0 + 64 < T ? 2 : 1;
        mbar_arrive_expect_tx(loaded, halves * 16384 + ndir * SM::kImgBytes);
#pragma unroll
        for (int kh = 0; kh < 2; ++kh)
            for (int th = 0; th < halves; ++th)
                tma_load_4d(smem + SM::kQ + kh * 16384 + th * 8192, &tm_q, loaded, kh * 64, h, t0 + th * 64, b);
        for (int d = 0; d < ndir; ++d) {
            const unsigned char *src = img + ((size_t)d * F * nbh + (size_t)f * nbh + bh) * ibytes;
            for (int piece = 0; piece < SM::kImgBytes; piece += 16384)
                bulk_load(smem + SM::kImg + d * ibytes + piece, src + piece, 16384, loaded);
        }
    }
    if (warp == 0) {
        tmem_alloc(tmem_s, NB);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_s;
    if (tid == 0) {
        if (!mbar_wait_ns(loaded, 0, kTcWaitNs)) {
            *abort_s = 1;
            if (err) atomicAdd(err, 1u);
        } else {
            tc_fence_after();
            constexpr uint32_t id = idesc(128, NB, 1, 0, 1);   // A K-major (Q), B MN-major (image)
            int n = 0;
            for (int d = 0; d < ndir; ++d) {
                const uint64_t dI = sdesc_sw128_mn(sbase + SM::kImg + d * (uint32_t)ibytes, 16384);
#pragma unroll
                for (int s = 0; s < 8; ++s, ++n) {          // 16 keys per MMA
                    const uint64_t a = sdesc_sw128(sbase + SM::kQ + (s >> 2) * 16384 + (s & 3) * 32);
                    mma_bf16(tmem, a, dI + (uint64_t)((s * 2048) >> 4), id, n > 0 ? 1u : 0u);
                }
            }
            mma_commit(done);
        }
    }
    __syncthreads();
    if (!*abort_s) {
        if (!mbar_wait_ns(done, 0, kTcWaitNs)) {
            *abort_s = 1;
            if (err) atomicAdd(err, 1u);
        }
    }
    tc_fence_after();
    // thread = token row (warp w reads TMEM lanes 32w .. 32w+31)
    // (the TMEM loads are warp-wide: every lane takes part, rows past the frame
    // only skip the stores)
    const int row = warp * 32 + lane, u = u0 + row;
    if (!*abort_s) {
        const uint32_t lb = (uint32_t)(warp * 32) << 16;
        Tout *dst = o + (((size_t)b * T + (size_t)f * U + u) * H + h) * DV;
        for (int n0 = 0; n0 < DV; n0 += 16) {
            float hi[16], lo[16];
            tmem_ld16(tmem + lb + n0, hi);
            tmem_ld16(tmem + lb + DV + n0, lo);
            tmem_wait_ld();
            if (u < U) {
#pragma unroll
                for (int q = 0; q < 16; q += 4)
                    store4(dst + n0 + q, hi[q] + lo[q], hi[q + 1] + lo[q + 1], hi[q + 2] + lo[q + 2],
                           hi[q + 3] + lo[q + 3]);
            }
        }
    } else if (tid == 0) {
        mbar_wait(loaded, 0, 64);
        mbar_wait(done, 0, 64);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, NB);
}

}  // namespace vda
}  // namespace gdn
