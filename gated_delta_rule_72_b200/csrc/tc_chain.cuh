// tc_chain.cuh -- the inter-chunk state chain on the tensor cores.
//
// One CTA of 128 threads owns one (b, h), one direction and a slice of NS
// columns of the d_k x d_v state (the columns evolve independently).  It
// walks the chunks in order (the reverse direction from the last chunk to
// the first) keeping its state slice on chip: an fp32 master copy in
// registers (thread d holds row d) and a bf16 hi/lo copy in shared memory as
// the B operand of the tensor-core products.  Per chunk, from the prep
// record (rows in forward token order) and the bf16 Q and K tiles:
//   X = W S,  Y = Q S                        (S as hi + lo)
//   Delta = U - X
//   O = diag(dq) Y + P Delta                 (P and Delta as hi/lo, 3 products)
//   S <- ds S + K^T (diag(dkk) Delta)        (Delta as hi + lo)
// Operands of the next chunk (TMA tiles and the record images) are fetched
// while the current chunk is computed.
#pragma once

#include "tc_common.cuh"

namespace gdn {
namespace tc2 {

template <int NS>
struct ChainSmem {
    static constexpr int kKQ = 32768;                      // [K|Q] x 2 column blocks, 128B swizzle
    static constexpr int kWimg = kKQ;                      // W image 16384
    static constexpr int kPh = kWimg + 16384;              // P hi image 8192
    static constexpr int kPl = kPh + 8192;                 // P lo image 8192
    static constexpr int kStage = kPl + 8192;              // 65536
    static constexpr int kStage0 = 0;
    static constexpr int kStage1 = kStage;
    static constexpr int kSh = 2 * kStage;                 // S hi, MN-major, K = 128
    static constexpr int kSl = kSh + 128 * NS * 2;
    static constexpr int kDh = kSl + 128 * NS * 2;         // Delta hi, MN-major, K = 64
    static constexpr int kDl = kDh + 64 * NS * 2;
    static constexpr int kEh = kDl + 64 * NS * 2;          // (dkk Delta) hi
    static constexpr int kEl = kEh + 64 * NS * 2;
    static constexpr int kBar = kEl + 64 * NS * 2;         // tma[2], mma
    static constexpr int kCtl = kBar + 32;
    static constexpr int kBytes = kCtl + 16;
    static constexpr int kAlloc = kBytes + 1024;
    static_assert(kAlloc <= 232448, "shared memory budget");
};

constexpr int kChainThreads = 128;

enum OutMode { kOutStore = 0, kOutPartial = 1, kOutAddPartial = 2 };

template <typename Tout>
__device__ __forceinline__ void store4(Tout *p, float4 v);
template <>
__device__ __forceinline__ void store4<float>(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16 *p, float4 v) {
    uint2 u;
    u.x = pack_bf16(v.x, v.y);
    u.y = pack_bf16(v.z, v.w);
    *reinterpret_cast<uint2 *>(p) = u;
}

// grid (DV/NS, B*H), block 128.
template <int DV, int NS, typename Tout>
__global__ void __launch_bounds__(kChainThreads, 1)
chain_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
             const unsigned char *__restrict__ recs, const float *__restrict__ state_in,
             float *__restrict__ state_out, Tout *__restrict__ o, float *__restrict__ part,
             int T, int H, int nC, int dir, int out_mode, unsigned int *__restrict__ err)
{
    using SM = ChainSmem<NS>;
    using RC = Rec<DV>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *tma_bar = reinterpret_cast<uint64_t *>(smem + SM::kBar);   // [2]
    uint64_t *mma_bar = tma_bar + 2;
    uint32_t *tmem_base_s = reinterpret_cast<uint32_t *>(smem + SM::kCtl);
    volatile int *abort_s = reinterpret_cast<volatile int *>(smem + SM::kCtl + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slice = blockIdx.x, bh = blockIdx.y;
    const int b = bh / H, h = bh % H;
    const int j0 = slice * NS;
    const int nbh = gridDim.y;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const bool row_lane = lane < 16;                    // M=64 accumulators: row 16*warp+lane
    const int f = warp * 16 + (lane & 15);              // forward row of a row lane
    constexpr uint32_t kColX = 0, kColY = NS, kColP = 2 * NS, kColS = 3 * NS;
    constexpr uint32_t kCols = (4 * NS <= 32) ? 32 : (4 * NS <= 64) ? 64 : (4 * NS <= 128) ? 128 : 256;
    const unsigned char *rec_base = recs + (size_t)(dir * nbh + bh) * nC * RC::kBytes;

    if (tid == 0) {
        mbar_init(&tma_bar[0], 1);
        mbar_init(&tma_bar[1], 1);
        mbar_init(mma_bar, 1);
        fence_mbar_init();
        *abort_s = 0;
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_q);
    }
    if (warp == 0) {
        tmem_alloc(tmem_base_s, kCols);
        tmem_relinquish();
    }

    // state slice: thread d owns row d (fp32) and writes its hi/lo operand row
    float S[NS];
    {
        const float *src = state_in ? state_in + ((size_t)bh * kDK + tid) * DV + j0 : nullptr;
#pragma unroll
        for (int n = 0; n < NS; ++n) S[n] = src ? src[n] : 0.f;
#pragma unroll
        for (int n = 0; n < NS; n += 8) {
            uint4 hi, lo;
            split2(S[n], S[n + 1], hi.x, lo.x); split2(S[n + 2], S[n + 3], hi.y, lo.y);
            split2(S[n + 4], S[n + 5], hi.z, lo.z); split2(S[n + 6], S[n + 7], hi.w, lo.w);
            *reinterpret_cast<uint4 *>(smem + SM::kSh + mnmaj<128>(n, tid)) = hi;
            *reinterpret_cast<uint4 *>(smem + SM::kSl + mnmaj<128>(n, tid)) = lo;
        }
    }
    fence_async_shared();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_s;

    auto chunk_of = [&](int step) { return dir == 0 ? step : nC - 1 - step; };
    auto issue_loads = [&](int step, int buf) {
        const int c = chunk_of(step);
        unsigned char *st = smem + (buf ? SM::kStage1 : SM::kStage0);
        const unsigned char *rec = rec_base + (size_t)c * RC::kBytes;
        uint64_t *bar = &tma_bar[buf];
        mbar_arrive_expect_tx(bar, SM::kStage);
        const int t0 = c * 64;
        tma_load_4d(st, &tm_k, bar, 0, h, t0, b);
        tma_load_4d(st + 16384, &tm_k, bar, 64, h, t0, b);
        tma_load_4d(st + 8192, &tm_q, bar, 0, h, t0, b);
        tma_load_4d(st + 16384 + 8192, &tm_q, bar, 64, h, t0, b);
        bulk_load(st + SM::kWimg, rec + RC::kW, 16384, bar);
        bulk_load(st + SM::kPh, rec + RC::kPh, 8192, bar);
        bulk_load(st + SM::kPl, rec + RC::kPl, 8192, bar);
    };
    auto wait_all = [&](uint64_t *bar, uint32_t parity) {
        if (!mbar_wait(bar, parity, kWaitTries)) {
            *abort_s = 1;
            if (err) atomicAdd(err, 1u);
        }
    };
    // per-row record values of a chunk: U slice, dq, dkk (row lanes) and ds
    auto load_rows = [&](int step, float *U, float &dq, float &dkk, float &ds) {
        const unsigned char *rec = rec_base + (size_t)chunk_of(step) * RC::kBytes;
        const float *gate = reinterpret_cast<const float *>(rec + RC::kGate);
        ds = gate[128];
        if (row_lane) {
            const float4 *u = reinterpret_cast<const float4 *>(rec + RC::kU + ((size_t)f * DV + j0) * 4);
#pragma unroll
            for (int q = 0; q < NS / 4; ++q) {
                const float4 v = u[q];
                U[4 * q] = v.x; U[4 * q + 1] = v.y; U[4 * q + 2] = v.z; U[4 * q + 3] = v.w;
            }
            dq = gate[f];
            dkk = gate[64 + f];
        }
    };

    if (tid == 0) issue_loads(0, 0);
    float Un[NS], dqn = 0.f, dkkn = 0.f, dsn = 0.f;
    load_rows(0, Un, dqn, dkkn, dsn);
    uint32_t tma_phases = 0, mma_phase = 0;   // bit b: parity of tma_bar[b]

    for (int step = 0; step < nC; ++step) {
        const int buf = step & 1;
        const int c = chunk_of(step);
        const uint32_t st_addr = sbase + (buf ? SM::kStage1 : SM::kStage0);
        float U[NS];
#pragma unroll
        for (int n = 0; n < NS; ++n) U[n] = Un[n];
        const float dq = dqn, dkk = dkkn, ds = dsn;

        wait_all(&tma_bar[buf], (tma_phases >> buf) & 1u);
        tma_phases ^= 1u << buf;
        __syncthreads();
        if (*abort_s) break;
        // ---- X = W S and Y = Q S ------------------------------------------------------
        if (tid == 0) {
            if (step + 1 < nC) issue_loads(step + 1, buf ^ 1);
            tc_fence_after();
            constexpr uint32_t id = idesc(64, NS, 1, 0, 1);
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                const uint32_t sb = sbase + (part ? SM::kSl : SM::kSh);
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const uint64_t bd = sdesc_noswz(sb + s * 256, 128, 128 * 16);
                    const uint32_t acc = (part | s) != 0;
                    mma_bf16(tmem + kColX, sdesc_noswz(st_addr + SM::kWimg + 2 * s * 1024, 1024, 128),
                             bd, id, acc);
                    mma_bf16(tmem + kColY,
                             sdesc_sw128(st_addr + 8192 + (s >> 2) * 16384 + (s & 3) * 32), bd, id, acc);
                }
            }
            mma_commit(mma_bar);
        }
        // the next chunk's row values travel while the tensor cores work
        if (step + 1 < nC) load_rows(step + 1, Un, dqn, dkkn, dsn);
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
            if (row_lane) {
#pragma unroll
                for (int n = 0; n < NS; n += 8) {
                    float d[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) d[e] = U[n + e] - X[n + e];
                    uint4 dh, dl, eh, el;
                    split2(d[0], d[1], dh.x, dl.x); split2(d[2], d[3], dh.y, dl.y);
                    split2(d[4], d[5], dh.z, dl.z); split2(d[6], d[7], dh.w, dl.w);
                    split2(dkk * d[0], dkk * d[1], eh.x, el.x); split2(dkk * d[2], dkk * d[3], eh.y, el.y);
                    split2(dkk * d[4], dkk * d[5], eh.z, el.z); split2(dkk * d[6], dkk * d[7], eh.w, el.w);
                    const int off = mnmaj<64>(n, f);
                    *reinterpret_cast<uint4 *>(smem + SM::kDh + off) = dh;
                    *reinterpret_cast<uint4 *>(smem + SM::kDl + off) = dl;
                    *reinterpret_cast<uint4 *>(smem + SM::kEh + off) = eh;
                    *reinterpret_cast<uint4 *>(smem + SM::kEl + off) = el;
                }
            }
        }
        fence_async_shared();
        tc_fence_before();
        __syncthreads();
        // ---- P Delta (3 products) and K^T (dkk Delta) (2 products) ------------------------
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idp = idesc(64, NS, 1, 0, 1);
            constexpr uint32_t ids = idesc(128, NS, 1, 1, 1);
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const uint64_t dh = sdesc_noswz(sbase + SM::kDh + s * 256, 128, 64 * 16);
                const uint64_t dl = sdesc_noswz(sbase + SM::kDl + s * 256, 128, 64 * 16);
                const uint64_t ph = sdesc_noswz(st_addr + SM::kPh + 2 * s * 1024, 1024, 128);
                const uint64_t pl = sdesc_noswz(st_addr + SM::kPl + 2 * s * 1024, 1024, 128);
                mma_bf16(tmem + kColP, ph, dh, idp, s > 0);
                mma_bf16(tmem + kColP, ph, dl, idp, 1);
                mma_bf16(tmem + kColP, pl, dh, idp, 1);
                const uint64_t ka = sdesc_sw128_mn(st_addr + s * 2048, 16384);
                mma_bf16(tmem + kColS, ka, sdesc_noswz(sbase + SM::kEh + s * 256, 128, 64 * 16), ids, s > 0);
                mma_bf16(tmem + kColS, ka, sdesc_noswz(sbase + SM::kEl + s * 256, 128, 64 * 16), ids, 1);
            }
            mma_commit(mma_bar);
        }
        wait_all(mma_bar, mma_phase);
        mma_phase ^= 1;
        tc_fence_after();
        {
            float Pd[NS], Sd[NS];
#pragma unroll
            for (int q = 0; q < NS / 16; ++q) {
                tmem_ld16(tmem + lane_base + kColP + q * 16, Pd + q * 16);
                tmem_ld16(tmem + lane_base + kColS + q * 16, Sd + q * 16);
            }
            tmem_wait_ld();
            const int t = c * 64 + f;
            if (row_lane && t < T) {
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
                        store4<Tout>(o + off + n, v);
                    }
                }
            }
#pragma unroll
            for (int n = 0; n < NS; n += 8) {
#pragma unroll
                for (int e = 0; e < 8; ++e) S[n + e] = fmaf(ds, S[n + e], Sd[n + e]);
                uint4 hi, lo;
                split2(S[n], S[n + 1], hi.x, lo.x); split2(S[n + 2], S[n + 3], hi.y, lo.y);
                split2(S[n + 4], S[n + 5], hi.z, lo.z); split2(S[n + 6], S[n + 7], hi.w, lo.w);
                *reinterpret_cast<uint4 *>(smem + SM::kSh + mnmaj<128>(n, tid)) = hi;
                *reinterpret_cast<uint4 *>(smem + SM::kSl + mnmaj<128>(n, tid)) = lo;
            }
        }
        fence_async_shared();
        tc_fence_before();
        __syncthreads();
    }

    if (*abort_s) {
        mbar_wait(&tma_bar[0], tma_phases & 1u, 1u << 16);
        mbar_wait(&tma_bar[1], (tma_phases >> 1) & 1u, 1u << 16);
        mbar_wait(mma_bar, mma_phase, 1u << 16);
    } else if (state_out) {
        float *dst = state_out + ((size_t)bh * kDK + tid) * DV + j0;
#pragma unroll
        for (int n = 0; n < NS; n += 4)
            *reinterpret_cast<float4 *>(dst + n) = make_float4(S[n], S[n + 1], S[n + 2], S[n + 3]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kCols);
}

}  // namespace tc2
}  // namespace gdn
