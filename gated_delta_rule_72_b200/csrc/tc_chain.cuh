// tc_chain.cuh -- the inter-chunk state chain on the tensor cores.
//
// One CTA owns one (b, h), one direction and a slice of NS columns of the
// d_k x d_v state (the columns evolve independently).  It walks the chunks in
// order (the reverse direction from the last chunk to the first) keeping its
// state slice on chip: an fp32 master copy in registers (thread d of the
// chain warps holds row d) and a bf16 hi/lo copy in shared memory as the B
// operand of the tensor-core products.  Per chunk, from the prep record
// (rows in forward token order) and the bf16 Q and K tiles:
//   X = W S                                  (S as hi + lo)      -- chain
//   Delta = U - X
//   S <- ds S + K^T (diag(dkk) Delta)        (Delta as hi + lo)  -- chain
//   Y = Q S,  O = diag(dq) Y + P Delta       (P, Delta hi/lo)    -- output
// The hi and lo halves of a split operand sit side by side along N, so one
// MMA instruction of width 2*NS yields both partial products (tcgen05.mma
// issue, not tensor throughput, bounds these small products).
// Roles (16 warps).  Warps 0-7 run the chain (the sequential dependency
// S -> X -> Delta -> S'), two warps per TMEM lane quarter, each owning half of
// the slice's columns.  Warps 8-11 drain the output products from
// double-buffered TMEM accumulators while the chain moves on.  A tcgen05.mma
// costs its issuing thread tens of cycles whatever its size, so the products
// are issued by several threads at once: warps 12 and 13 each issue half of
// the K-steps of the chain's two products (X and K^T E, into separate
// accumulators the chain adds), warp 14 the output products (Y and P Delta),
// warp 15 the loads.  The roles meet on mbarriers, each of which can only
// advance again after all of its waiters have seen its previous phase.
#pragma once

#include "tc_common.cuh"

namespace gdn {
namespace tc2 {

#ifdef GDN_CHAIN_TIMING
// Development aid (not built into the library): cycle stamps of CTA (0,0),
// steps 10..19, issuing lane (slots 0..9) and chain thread 0 (slots 10..14).
__device__ long long g_chain_ts[10][24];
#define CHAIN_TS(slot) do { if (blockIdx.x == 0 && blockIdx.y == 0 && step >= 10 && step < 20) \
    g_chain_ts[step - 10][slot] = clock64(); } while (0)
#else
#define CHAIN_TS(slot) do { } while (0)
#endif

template <int NS>
struct ChainSmem {
    static constexpr int kKQ = 32768;                      // [K|Q] x 2 column blocks, 128B swizzle
    static constexpr int kWimg = kKQ;                      // W image 16384
    static constexpr int kPh = kWimg + 16384;              // P hi image 8192
    static constexpr int kPl = kPh + 8192;                 // P lo image 8192
    static constexpr int kU = kPl + 8192;                  // U slice [64][NS] fp32
    static constexpr int kG = kU + 64 * NS * 4;            // dq[64], dkk[64], ds
    static constexpr int kStage = kG + 1024;
    static constexpr int kStage0 = 0;
    static constexpr int kStage1 = kStage;
    static constexpr int kSh = 2 * kStage;                 // S hi, MN-major, K = 128
    static constexpr int kSl = kSh + 128 * NS * 2;
    static constexpr int kDh = kSl + 128 * NS * 2;         // Delta hi, MN-major, K = 64
    static constexpr int kDl = kDh + 64 * NS * 2;
    static constexpr int kEh = kDl + 64 * NS * 2;          // (dkk Delta) hi
    static constexpr int kEl = kEh + 64 * NS * 2;
    static constexpr int kBar = kEl + 64 * NS * 2;         // mbarriers
    static constexpr int kCtl = kBar + 256;
    static constexpr int kBytes = kCtl + 16;
    static constexpr int kAlloc = kBytes + 1024;
    static_assert(kAlloc <= 232448, "shared memory budget");
};

constexpr int kChainThreads = 512;     // 8 chain, 4 output, 3 MMA-issuing and 1 load warp

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

// grid (DV/NS, B*H), block 256.
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
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::kBar);
    uint64_t *tma_bar = bars + 0;      // [2] stage loaded              (load warp -> issuers)
    uint64_t *free_st = bars + 2;      // [2] stage consumed: 3 MMA commits + 12 warps (-> load warp)
    uint64_t *xa_bar = bars + 4;       // X, first K half               (issuer A -> chain)
    uint64_t *xb_bar = bars + 5;       // X, second K half              (issuer B -> chain)
    uint64_t *sa_bar = bars + 6;       // K^T E, first half             (issuer A -> chain)
    uint64_t *sb_bar = bars + 7;       // K^T E, second half            (issuer B -> chain)
    uint64_t *y_bar = bars + 8;        // Y done reading S              (issuer C -> chain)
    uint64_t *out_bar = bars + 9;      // [2] Y and P Delta of a slot   (issuer C -> output, chain)
    uint64_t *free_bar = bars + 11;    // [2] slot drained, 4 warps     (output -> issuer C)
    uint64_t *d_bar = bars + 13;       // Delta and E written, 8 warps  (chain -> issuers)
    uint64_t *r_bar = bars + 14;       // S rewritten, 8 warps          (chain -> issuers)
    uint32_t *tmem_base_s = reinterpret_cast<uint32_t *>(smem + SM::kCtl);
    volatile int *abort_s = reinterpret_cast<volatile int *>(smem + SM::kCtl + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3;
    const int slice = blockIdx.x, bh = blockIdx.y;
    const int b = bh / H, h = bh % H;
    const int j0 = slice * NS;
    const int nbh = gridDim.y;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const bool row_lane = lane < 16;                    // M=64 accumulators: row 16*quarter+lane
    const int f = quarter * 16 + (lane & 15);           // forward row of a row lane
    constexpr int NH = NS / 2;                          // columns per chain warp
    // TMEM columns (each accumulator 2*NS wide: the hi and lo partial products)
    constexpr uint32_t kColXA = 0, kColXB = 2 * NS, kColSA = 4 * NS, kColSB = 6 * NS;
    constexpr uint32_t kColY = 8 * NS, kColP = 12 * NS;
    constexpr uint32_t kCols = 512;
    static_assert(16 * NS <= 512, "TMEM budget");
    static_assert(NS == kSliceCols, "the record stores U in slices of kSliceCols columns");
    const unsigned char *rec_base = recs + (size_t)(dir * nbh + bh) * nC * RC::kBytes;

    if (tid == 0) {
        mbar_init(&tma_bar[0], 1);
        mbar_init(&tma_bar[1], 1);
        mbar_init(&free_st[0], 15);    // issuers A, B, C + 8 chain + 4 output warps
        mbar_init(&free_st[1], 15);
        mbar_init(xa_bar, 1);
        mbar_init(xb_bar, 1);
        mbar_init(sa_bar, 1);
        mbar_init(sb_bar, 1);
        mbar_init(y_bar, 1);
        mbar_init(&out_bar[0], 1);
        mbar_init(&out_bar[1], 1);
        mbar_init(&free_bar[0], 4);     // one arrival per warp
        mbar_init(&free_bar[1], 4);
        mbar_init(d_bar, 8);
        mbar_init(r_bar, 8);
        fence_mbar_init();
        *abort_s = 0;
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_q);
    }
    if (warp == 0) {
        tmem_alloc(tmem_base_s, kCols);
        tmem_relinquish();
    }
    // state slice: chain thread (quarter, column half) owns row d, columns c0 .. c0+NH-1
    const int d_row = quarter * 32 + lane;
    const int c0 = (warp >> 2) * NH;
    float S[NH];
    if (warp < 8) {
        const float *src = state_in ? state_in + ((size_t)bh * kDK + d_row) * DV + j0 + c0 : nullptr;
#pragma unroll
        for (int n = 0; n < NH; ++n) S[n] = src ? src[n] : 0.f;
#pragma unroll
        for (int n = 0; n < NH; n += 8) {
            uint4 hi, lo;
            split2(S[n], S[n + 1], hi.x, lo.x); split2(S[n + 2], S[n + 3], hi.y, lo.y);
            split2(S[n + 4], S[n + 5], hi.z, lo.z); split2(S[n + 6], S[n + 7], hi.w, lo.w);
            *reinterpret_cast<uint4 *>(smem + SM::kSh + mnmaj<128>(c0 + n, d_row)) = hi;
            *reinterpret_cast<uint4 *>(smem + SM::kSl + mnmaj<128>(c0 + n, d_row)) = lo;
        }
    }
    fence_async_shared();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_s;

    auto chunk_of = [&](int step) { return dir == 0 ? step : nC - 1 - step; };
    auto rec_of = [&](int step) { return rec_base + (size_t)chunk_of(step) * RC::kBytes; };
    auto wait_on = [&](uint64_t *bar, uint32_t parity) {
        if (!mbar_wait(bar, parity, kWaitTries)) {
            *abort_s = 1;
            if (err) atomicAdd(err, 1u);
        }
    };
    constexpr uint32_t idX = idesc(64, 2 * NS, 1, 0, 1);    // X, Y, P Delta: A K-major, B MN-major
    constexpr uint32_t idS = idesc(128, 2 * NS, 1, 1, 1);   // K^T E: A MN-major (K tile), B MN-major
    const uint64_t dSh = sdesc_noswz(sbase + SM::kSh, 128, 128 * 16);
    const uint64_t dDh = sdesc_noswz(sbase + SM::kDh, 128, 64 * 16);
    const uint64_t dEh = sdesc_noswz(sbase + SM::kEh, 128, 64 * 16);
    auto adv = [](uint64_t d, uint32_t bytes) { return d + (uint64_t)(bytes >> 4); };
    auto stage_of = [&](int step) { return sbase + ((step & 1) ? SM::kStage1 : SM::kStage0); };

    if (warp == 15) {
        // ============================ load warp ====================================
        if (lane == 0) {
            uint32_t free_phases = 0;
            for (int step = 0; step < nC; ++step) {
                const int buf = step & 1;
                if (step >= 2) {   // this stage's previous use has been consumed by all issuers
                    wait_on(&free_st[buf], (free_phases >> buf) & 1u);
                    free_phases ^= 1u << buf;
                }
                if (*abort_s) break;
                const int c = chunk_of(step);
                unsigned char *st = smem + (buf ? SM::kStage1 : SM::kStage0);
                const unsigned char *rec = rec_of(step);
                uint64_t *bar = &tma_bar[buf];
                mbar_arrive_expect_tx(bar, SM::kKQ + 16384 + 16384 + RC::kUSlice + RC::kGateCopy);
                const int t0 = c * 64;
                tma_load_4d(st, &tm_k, bar, 0, h, t0, b);
                tma_load_4d(st + 16384, &tm_k, bar, 64, h, t0, b);
                tma_load_4d(st + 8192, &tm_q, bar, 0, h, t0, b);
                tma_load_4d(st + 16384 + 8192, &tm_q, bar, 64, h, t0, b);
                bulk_load(st + SM::kWimg, rec + RC::kW, 16384, bar);
                bulk_load(st + SM::kPh, rec + RC::kPh, 8192, bar);
                bulk_load(st + SM::kPl, rec + RC::kPl, 8192, bar);
                bulk_load(st + SM::kU, rec + RC::kU + slice * RC::kUSlice, RC::kUSlice, bar);
                bulk_load(st + SM::kG, rec + RC::kGate, RC::kGateCopy, bar);
            }
        }
        __syncwarp();
    } else if (warp == 12 || warp == 13) {
        // ===================== chain issuers A (warp 12) and B (warp 13) =============
        if (lane == 0) {
            const int part = warp - 12;
            uint64_t *xbar = part ? xb_bar : xa_bar;
            uint64_t *sbar = part ? sb_bar : sa_bar;
            const uint32_t colX = part ? kColXB : kColXA, colS = part ? kColSB : kColSA;
            uint32_t tma_phases = 0, d_phase = 0, r_phase = 0;
            for (int step = 0; step < nC; ++step) {
                const int buf = step & 1;
                const uint32_t st = stage_of(step);
                if (part == 0) CHAIN_TS(0);
                wait_on(&tma_bar[buf], (tma_phases >> buf) & 1u);
                tma_phases ^= 1u << buf;
                if (part == 0) CHAIN_TS(1);
                if (step > 0) { wait_on(r_bar, r_phase); r_phase ^= 1; }
                if (part == 0) CHAIN_TS(2);
                if (*abort_s) break;
                tc_fence_after();
                // X = W [S_hi | S_lo], K-steps 4*part .. 4*part+3
                const uint64_t dW = sdesc_noswz(st + SM::kWimg, 1024, 128);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int s = part * 4 + k;
                    mma_bf16(tmem + colX, adv(dW, 2 * s * 1024), adv(dSh, s * 256), idX, k > 0);
                }
                mma_commit(xbar);
                if (part == 0) CHAIN_TS(3);
                wait_on(d_bar, d_phase);
                d_phase ^= 1;
                if (part == 0) CHAIN_TS(4);
                if (*abort_s) break;
                tc_fence_after();
                // K^T [E_hi | E_lo], K-steps 2*part .. 2*part+1 (tokens 32*part .. +31)
                const uint64_t dK = sdesc_sw128_mn(st, 16384);
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int s = part * 2 + k;
                    mma_bf16(tmem + colS, adv(dK, s * 2048), adv(dEh, s * 256), idS, k > 0);
                }
                mma_commit(sbar);
                if (part == 0) CHAIN_TS(5);
                mma_commit(&free_st[buf]);
            }
        }
        __syncwarp();
    } else if (warp == 14) {
        // ============================ output issuer C ==============================
        if (lane == 0) {
            uint32_t tma_phases = 0, d_phase = 0, r_phase = 0, free_phases = 0;
            for (int step = 0; step < nC; ++step) {
                const int buf = step & 1, slot = step & 1;
                const uint32_t st = stage_of(step);
                wait_on(&tma_bar[buf], (tma_phases >> buf) & 1u);
                tma_phases ^= 1u << buf;
                if (step > 0) { wait_on(r_bar, r_phase); r_phase ^= 1; }
                if (step >= 2) {   // the output warps have drained this slot's last use
                    wait_on(&free_bar[slot], (free_phases >> slot) & 1u);
                    free_phases ^= 1u << slot;
                }
                if (*abort_s) break;
                tc_fence_after();
                // Y = Q [S_hi | S_lo]
                const uint64_t dQ = sdesc_sw128(st + 8192);
                const uint32_t colY = kColY + slot * 2 * NS;
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_bf16(tmem + colY, adv(dQ, (s >> 2) * 16384 + (s & 3) * 32), adv(dSh, s * 256), idX,
                             s > 0);
                mma_commit(y_bar);
                wait_on(d_bar, d_phase);
                d_phase ^= 1;
                if (*abort_s) break;
                tc_fence_after();
                // P [Delta_hi | Delta_lo] with P = P_hi + P_lo
                const uint64_t dPh = sdesc_noswz(st + SM::kPh, 1024, 128);
                const uint64_t dPl = sdesc_noswz(st + SM::kPl, 1024, 128);
                const uint32_t colP = kColP + slot * 2 * NS;
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    mma_bf16(tmem + colP, adv(dPh, 2 * s * 1024), adv(dDh, s * 256), idX, s > 0);
                    mma_bf16(tmem + colP, adv(dPl, 2 * s * 1024), adv(dDh, s * 256), idX, 1);
                }
                mma_commit(&out_bar[slot]);
                mma_commit(&free_st[buf]);
            }
        }
        __syncwarp();
    } else if (warp < 8) {
        // ============================ chain warps ===================================
        uint32_t x_phase = 0, s_phase = 0, y_phase = 0, out_phases = 0, tma_phases = 0;
        for (int step = 0; step < nC; ++step) {
            const int buf = step & 1;
            const unsigned char *stg = smem + (buf ? SM::kStage1 : SM::kStage0);
            // this chunk's U slice and gates arrive with the stage
            wait_on(&tma_bar[buf], (tma_phases >> buf) & 1u);
            tma_phases ^= 1u << buf;
            float U[NH];
            float dkk = 0.f;
            {
                const float *us = reinterpret_cast<const float *>(stg + SM::kU) + f * NS + c0;
#pragma unroll
                for (int q = 0; q < NH / 4; ++q) {
                    const float4 v = reinterpret_cast<const float4 *>(us)[q];
                    U[4 * q] = v.x; U[4 * q + 1] = v.y; U[4 * q + 2] = v.z; U[4 * q + 3] = v.w;
                }
                dkk = reinterpret_cast<const float *>(stg + SM::kG)[64 + f];
            }
            const float ds = reinterpret_cast<const float *>(stg + SM::kG)[128];
            __syncwarp();
            if (lane == 0) mbar_arrive(&free_st[buf]);   // this warp is done reading the stage
            if (tid == 0) CHAIN_TS(10);
            wait_on(xa_bar, x_phase);
            if (tid == 0) CHAIN_TS(17);
            wait_on(xb_bar, x_phase);
            x_phase ^= 1;
            if (step > 0) {   // P Delta of the previous step has read the Delta buffers
                const int ps = (step - 1) & 1;
                wait_on(&out_bar[ps], (out_phases >> ps) & 1u);
                out_phases ^= 1u << ps;
            }
            CHAIN_TS(11);
            tc_fence_after();
#pragma unroll
            for (int q = 0; q < NH / 16; ++q) {   // 16 columns: X = (A hi + A lo) + (B hi + B lo)
                const int n0 = c0 + q * 16;
                float x0[16], x1[16], x2[16], x3[16];
                tmem_ld16(tmem + lane_base + kColXA + n0, x0);
                tmem_ld16(tmem + lane_base + kColXA + NS + n0, x1);
                tmem_ld16(tmem + lane_base + kColXB + n0, x2);
                tmem_ld16(tmem + lane_base + kColXB + NS + n0, x3);
                tmem_wait_ld();
                if (tid == 0) CHAIN_TS(15);
                if (row_lane) {
#pragma unroll
                    for (int h8 = 0; h8 < 16; h8 += 8) {
                        const int n = n0 + h8;
                        float d[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            d[e] = U[q * 16 + h8 + e] - ((x0[h8 + e] + x1[h8 + e]) + (x2[h8 + e] + x3[h8 + e]));
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
            if (tid == 0) CHAIN_TS(12);
            __syncwarp();
            if (lane == 0) mbar_arrive(d_bar);
            wait_on(sa_bar, s_phase);
            wait_on(sb_bar, s_phase);
            s_phase ^= 1;
            wait_on(y_bar, y_phase);   // Y has read this step's S
            y_phase ^= 1;
            if (tid == 0) CHAIN_TS(13);
            if (*abort_s) break;
            tc_fence_after();
#pragma unroll
            for (int q = 0; q < NH / 16; ++q) {   // S <- ds S + (A hi + A lo) + (B hi + B lo)
                const int n0 = c0 + q * 16;
                float s0[16], s1[16], s2[16], s3[16];
                tmem_ld16(tmem + lane_base + kColSA + n0, s0);
                tmem_ld16(tmem + lane_base + kColSA + NS + n0, s1);
                tmem_ld16(tmem + lane_base + kColSB + n0, s2);
                tmem_ld16(tmem + lane_base + kColSB + NS + n0, s3);
                tmem_wait_ld();
                if (tid == 0) CHAIN_TS(16);
#pragma unroll
                for (int h8 = 0; h8 < 16; h8 += 8) {
                    const int n = q * 16 + h8;
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        S[n + e] = fmaf(ds, S[n + e], (s0[h8 + e] + s1[h8 + e]) + (s2[h8 + e] + s3[h8 + e]));
                    uint4 hi, lo;
                    split2(S[n], S[n + 1], hi.x, lo.x); split2(S[n + 2], S[n + 3], hi.y, lo.y);
                    split2(S[n + 4], S[n + 5], hi.z, lo.z); split2(S[n + 6], S[n + 7], hi.w, lo.w);
                    *reinterpret_cast<uint4 *>(smem + SM::kSh + mnmaj<128>(c0 + n, d_row)) = hi;
                    *reinterpret_cast<uint4 *>(smem + SM::kSl + mnmaj<128>(c0 + n, d_row)) = lo;
                }
            }
            fence_async_shared();
            tc_fence_before();
            if (tid == 0) CHAIN_TS(14);
            __syncwarp();
            if (lane == 0) mbar_arrive(r_bar);
        }
        if (!*abort_s && state_out) {
            float *dst = state_out + ((size_t)bh * kDK + d_row) * DV + j0 + c0;
#pragma unroll
            for (int n = 0; n < NH; n += 4)
                *reinterpret_cast<float4 *>(dst + n) = make_float4(S[n], S[n + 1], S[n + 2], S[n + 3]);
        }
    } else {
        // ============================ output warps (8..11) ===========================
        uint32_t out_phases = 0, tma_phases = 0;
        for (int step = 0; step < nC; ++step) {
            const int slot = step & 1, buf = step & 1;
            const int c = chunk_of(step);
            wait_on(&tma_bar[buf], (tma_phases >> buf) & 1u);
            tma_phases ^= 1u << buf;
            const float dq = reinterpret_cast<const float *>(smem + (buf ? SM::kStage1 : SM::kStage0) +
                                                             SM::kG)[f];
            __syncwarp();
            if (lane == 0) mbar_arrive(&free_st[buf]);   // done reading the stage
            const int t = c * 64 + f;
            const size_t off = (((size_t)b * T + (t < T ? t : 0)) * H + h) * DV + j0;
            float4 prev[NS / 4];
            if (out_mode == kOutAddPartial && row_lane && t < T) {
#pragma unroll
                for (int q = 0; q < NS / 4; ++q) prev[q] = *reinterpret_cast<const float4 *>(part + off + 4 * q);
            }
            wait_on(&out_bar[slot], (out_phases >> slot) & 1u);
            out_phases ^= 1u << slot;
            tc_fence_after();
            const uint32_t cy = kColY + slot * 2 * NS, cp = kColP + slot * 2 * NS;
#pragma unroll
            for (int q = 0; q < NS / 16; ++q) {   // 16 columns at a time: hi part + lo part
                float Y[16], Y2[16], Pd[16], P2[16];
                tmem_ld16(tmem + lane_base + cy + q * 16, Y);
                tmem_ld16(tmem + lane_base + cy + NS + q * 16, Y2);
                tmem_ld16(tmem + lane_base + cp + q * 16, Pd);
                tmem_ld16(tmem + lane_base + cp + NS + q * 16, P2);
                tmem_wait_ld();
                if (q == NS / 16 - 1) {   // the slot is drained: hand it back to issuer C
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&free_bar[slot]);
                }
                if (row_lane && t < T) {
#pragma unroll
                    for (int e = 0; e < 16; e += 4) {
                        const int n = q * 16 + e;
                        float4 v;
                        v.x = fmaf(dq, Y[e] + Y2[e], Pd[e] + P2[e]);
                        v.y = fmaf(dq, Y[e + 1] + Y2[e + 1], Pd[e + 1] + P2[e + 1]);
                        v.z = fmaf(dq, Y[e + 2] + Y2[e + 2], Pd[e + 2] + P2[e + 2]);
                        v.w = fmaf(dq, Y[e + 3] + Y2[e + 3], Pd[e + 3] + P2[e + 3]);
                        if (out_mode == kOutPartial) {
                            *reinterpret_cast<float4 *>(part + off + n) = v;
                        } else {
                            if (out_mode == kOutAddPartial) {
                                const float4 p = prev[n / 4];
                                v.x += p.x; v.y += p.y; v.z += p.z; v.w += p.w;
                            }
                            store4<Tout>(o + off + n, v);
                        }
                    }
                }
            }
            if (*abort_s) break;
        }
    }

    __syncthreads();
    if (*abort_s && tid == 0) {
        // a wait timed out: let copies and MMAs in flight land (bounded) before
        // shared memory and TMEM are released
        mbar_wait(&tma_bar[0], 0, 64);
        mbar_wait(&tma_bar[1], 0, 64);
        mbar_wait(sa_bar, 0, 64);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kCols);
}

}  // namespace tc2
}  // namespace gdn
