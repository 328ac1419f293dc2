// tc_chain.cuh -- the inter-chunk state chain on the tensor cores.
//
// One CTA owns one (b, h), one direction and a slice of NS = 64 columns of
// the d_k x d_v state (the columns evolve independently).  It walks the
// chunks in order (the reverse direction from the last chunk to the first)
// keeping its state slice on chip: an fp32 master copy in registers and a
// bf16 hi/lo copy in shared memory as the B operand of the tensor-core
// products.  Per chunk, from the prep record (rows in forward token order)
// and the bf16 Q and K tiles:
//   [Y; X] = [Q; W] [S_hi | S_lo]            one M=128 product
//   Delta = U - X
//   S <- ds S + K^T [E_hi | E_lo],  E = diag(dkk) Delta
//   O = diag(dq) Y + [P_hi | P_lo] [D; D],  D = [Delta_hi | Delta_lo]
// The hi and lo halves of a split operand sit side by side along N, so one
// MMA of width 2*NS yields both partial products; P's halves are stacked
// along K instead, so the tensor core adds P_hi D + P_lo D itself.  Stacking
// Q over W makes Y and X one instruction stream (a tcgen05.mma costs its
// issuing thread tens of cycles whatever its size, so fewer, wider products
// are faster); Y then lands in TMEM lanes 0-63 and X in lanes 64-127.
//
// Roles (20 warps).  The 16 epilogue warps cover the 128 TMEM lanes four
// times (warp w reads lane quarter w % 4, columns 16 * (w / 4) .. +15):
//   quarters 2, 3 (X rows)  form Delta and E           (critical path)
//   quarters 0, 1 (Y rows)  form and store the output   (off the chain)
//   all                     S <- ds S + K^T E, thread = one row of S
// Warps 16 and 17 issue [Q;W] S, one K half each (A then also K^T E), warp 19
// issues P D and warp 18 loads the stages.  A thread that has just queued a
// batch of MMAs is slow to see barriers complete, so the off-chain product
// gets an issuing thread of its own.
// The roles meet on mbarriers; each of them can only complete its next phase
// after every waiter has observed the previous one.
//
// Bidirectional mode runs both directions in one launch (grid.z = 2).  Each
// direction writes its 32 x 16 output pieces to its own fp32 buffer; of the
// two CTAs that produce the same piece, the one that finishes second (an
// atomic counter per piece decides) adds the other's piece and writes o.
#pragma once

#include "tc_common.cuh"

namespace gdn {
namespace tc2 {

#ifdef GDN_CHAIN_TIMING
// Development aid (not built into the library): cycle stamps of CTA (0,0,0),
// steps 10..19.
__device__ long long g_chain_ts[10][32];
#define CHAIN_TS(slot) do { if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && \
    step >= 10 && step < 20) g_chain_ts[step - 10][slot] = clock64(); } while (0)
#else
#define CHAIN_TS(slot) do { } while (0)
#endif

constexpr int kChainNS = 64;           // state columns per CTA

struct ChainSmem {
    static constexpr int NS = kChainNS;
    // one stage (1024-aligned): [Q;W] 2 x 16 KB column blocks (Q rows 0-63,
    // W rows 64-127), K 2 x 8 KB, P_hi | P_lo 2 x 8 KB (all 128B-swizzled,
    // K-major), U 64 x 64 fp32 (rows swizzled, u_off).  The operands the epilogues write,
    // [S_hi | S_lo], [D_hi | D_lo] and [E_hi | E_lo], are 128B-swizzled
    // MN-major (one 128-byte row per K index), like a tile load would write
    // them: the unswizzled layouts cost the tensor core several times the
    // shared-memory wavefronts.
    static constexpr int kQW = 0;
    static constexpr int kK = 32768;
    static constexpr int kP = kK + 16384;
    static constexpr int kU = kP + 16384;
    static constexpr int kStage = kU + 64 * NS * 4;
    static constexpr int kSL = 2 * kStage;                 // [S_hi | S_lo], K = 128: 2 x 16 KB
    static constexpr int kD = kSL + 128 * 2 * NS * 2;      // [D_hi | D_lo], K = 64: 2 x 8 KB
    static constexpr int kE = kD + 64 * 2 * NS * 2;        // [E_hi | E_lo]
    static constexpr int kG = kE + 64 * 2 * NS * 2;        // 2 x gates (dq, dkk, ds)
    static constexpr int kGate = 528;
    static constexpr int kBar = kG + 2 * kGate;            // mbarriers
    static constexpr int kCtl = kBar + 128;
    static constexpr int kBytes = kCtl + 16;
    static constexpr int kAlloc = kBytes + 1024;
    static_assert(kStage % 1024 == 0 && kSL % 1024 == 0 && kD % 1024 == 0 && kE % 1024 == 0,
                  "swizzled operands must stay 1024-aligned");
    static_assert(NS == 64, "one 64-element MN group per hi / lo half");
    static_assert(kAlloc <= 232448, "shared memory budget");
};

constexpr int kChainWarps = 20;
constexpr int kChainThreads = kChainWarps * 32;

enum OutMode { kOutStore = 0, kOutPair = 1 };

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

// Output of a chain: where each direction's pieces go and how they combine.
template <typename Tout>
struct ChainOut {
    Tout *o;                 // [B, T, H, DV]
    float *part[2];          // kOutPair: fp32 [B, T, H, DV] per direction (part[0] may be o)
    unsigned int *cnt;       // kOutPair: one counter per 32 x 16 piece, zero on entry
    int mode;
};

// grid (DV/NS, B*H, directions), block kChainThreads.  blockIdx.z + dir0 is
// the direction (0 causal, 1 reverse).
template <int DV, typename Tout>
__global__ void __launch_bounds__(kChainThreads, 1)
chain_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
             const __grid_constant__ CUtensorMap tm_o, const unsigned char *__restrict__ recs, const float *__restrict__ state_in,
             float *__restrict__ state_out, const ChainOut<Tout> out, int T, int H, int nC,
             int dir0, unsigned int *__restrict__ err)
{
    using SM = ChainSmem;
    using RC = Rec<DV>;
    constexpr int NS = kChainNS;
    constexpr int N2 = 2 * NS;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::kBar);
    uint64_t *full = bars + 0;         // [2] stage loaded                        (loader -> all)
    uint64_t *free_st = bars + 2;      // [2] stage consumed: 16 warps, A, B, C x 2  (-> loader)
    uint64_t *xy_bar = bars + 4;       // [Y; X] complete, 2 commits              (A, B -> warps)
    uint64_t *delta_bar = bars + 5;    // Delta (fp32) in the stage, 8 X warps    (-> Y warps)
    uint64_t *e_bar = bars + 6;        // E written (and Y read), 8 Y warps       (-> A, B)
    uint64_t *dd_bar = bars + 7;       // D written, 8 X warps                    (-> C)
    uint64_t *s_bar = bars + 8;        // K^T E complete, 2 commits               (A, B -> warps, C)
    uint64_t *r_bar = bars + 9;        // S rewritten, 16 warps                   (-> A, B)
    uint64_t *pd_bar = bars + 10;      // P D complete                            (C -> warps)
    uint64_t *pd_free = bars + 11;     // P D read, 8 Y warps                     (-> C)
    uint64_t *o_bar = bars + 12;       // output tile staged, 8 Y warps           (-> C)
    uint32_t *tmem_base_s = reinterpret_cast<uint32_t *>(smem + SM::kCtl);
    volatile int *abort_s = reinterpret_cast<volatile int *>(smem + SM::kCtl + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, cg = (warp >> 2) & 3;
    const int slice = blockIdx.x, bh = blockIdx.y, dir = dir0 + blockIdx.z;
    const int b = bh / H, h = bh % H;
    const int j0 = slice * NS;
    const int nbh = gridDim.y;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int n0 = cg * 16;                                 // this warp's 16 columns of the slice
    // TMEM columns, each accumulator 2*NS wide (hi | lo): [Y;X] in two K halves
    // (XA, XB), K^T E in two token halves (S, and XB again once [Y;X] is read), P D
    constexpr uint32_t kColXA = 0, kColXB = N2, kColS = 2 * N2, kColPD = 3 * N2;
    constexpr uint32_t kCols = 512;
    static_assert(4 * N2 <= 512, "TMEM budget");
    static_assert(NS == kSliceCols, "the record stores U in slices of the chain's width");
    const unsigned char *rec_base = recs + (size_t)(dir * nbh + bh) * nC * RC::kBytes;

    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(&free_st[0], 20);
        mbar_init(&free_st[1], 20);
        mbar_init(xy_bar, 2);
        mbar_init(delta_bar, 8);
        mbar_init(e_bar, 8);
        mbar_init(dd_bar, 8);
        mbar_init(s_bar, 2);
        mbar_init(r_bar, 16);
        mbar_init(pd_bar, 1);
        mbar_init(pd_free, 8);
        mbar_init(o_bar, 8);
        fence_mbar_init();
        *abort_s = 0;
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_q);
        if (out.mode == kOutStore) prefetch_tensormap(&tm_o);
    }
    if (warp == 0) {
        tmem_alloc(tmem_base_s, kCols);
        tmem_relinquish();
    }
    // state: epilogue thread (quarter, cg, lane) owns row d_row, columns n0 .. n0+15
    const int d_row = quarter * 32 + lane;
    float S[16];
    if (warp < 16) {
        const float *src = state_in ? state_in + ((size_t)bh * kDK + d_row) * DV + j0 + n0 : nullptr;
#pragma unroll
        for (int n = 0; n < 16; ++n) S[n] = src ? src[n] : 0.f;
#pragma unroll
        for (int n = 0; n < 16; n += 8) {
            uint4 hi, lo;
            split2(S[n], S[n + 1], hi.x, lo.x); split2(S[n + 2], S[n + 3], hi.y, lo.y);
            split2(S[n + 4], S[n + 5], hi.z, lo.z); split2(S[n + 6], S[n + 7], hi.w, lo.w);
            *reinterpret_cast<uint4 *>(smem + SM::kSL + swz_mn(n0 + n, d_row, 16384)) = hi;
            *reinterpret_cast<uint4 *>(smem + SM::kSL + swz_mn(NS + n0 + n, d_row, 16384)) = lo;
        }
    }
    fence_async_shared();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_s;

    auto chunk_of = [&](int step) { return dir == 0 ? step : nC - 1 - step; };
    auto wait_on = [&](uint64_t *bar, uint32_t parity) {
        if (!mbar_wait(bar, parity, kWaitTries)) {
            *abort_s = 1;
            if (err) atomicAdd(err, 1u);
        }
    };
    auto stage_addr = [&](int step) { return sbase + (step & 1) * SM::kStage; };
    auto gates = [&](int step) { return reinterpret_cast<const float *>(smem + SM::kG + (step & 1) * SM::kGate); };
    auto adv = [](uint64_t d, uint32_t bytes) { return d + (uint64_t)(bytes >> 4); };
    constexpr uint32_t idQW = idesc(128, N2, 1, 0, 1);   // [Q;W] S and P D: A K-major, B MN-major
    constexpr uint32_t idKE = idesc(128, N2, 1, 1, 1);   // K^T E: A MN-major (the K tile), B MN-major
    const uint64_t dK0 = sdesc_sw128_mn(sbase + SM::kK, 8192);
    // MN-major swizzled B operands; a K-step of 16 rows advances 2048 bytes
    const uint64_t dSL = sdesc_sw128_mn(sbase + SM::kSL, 16384);
    const uint64_t dD = sdesc_sw128_mn(sbase + SM::kD, 8192);
    const uint64_t dE = sdesc_sw128_mn(sbase + SM::kE, 8192);

    if (warp == 18) {
        // ============================ loader ========================================
        if (lane == 0) {
            uint32_t free_phases = 0;
            for (int step = 0; step < nC; ++step) {
                const int buf = step & 1;
                if (step >= 2) {   // the stage's previous chunk has been consumed
                    wait_on(&free_st[buf], (free_phases >> buf) & 1u);
                    free_phases ^= 1u << buf;
                }
                CHAIN_TS(24);
                if (*abort_s) break;
                const int c = chunk_of(step);
                unsigned char *st = smem + buf * SM::kStage;
                const unsigned char *rec = rec_base + (size_t)c * RC::kBytes;
                uint64_t *bar = &full[buf];
                mbar_arrive_expect_tx(bar, 4 * 16384 + 64 * NS * 4 + SM::kGate);
                const int t0 = c * 64;
                tma_load_4d(st + SM::kQW, &tm_q, bar, 0, h, t0, b);
                tma_load_4d(st + SM::kQW + 16384, &tm_q, bar, 64, h, t0, b);
                bulk_load(st + SM::kQW + 8192, rec + RC::kW, 8192, bar);
                bulk_load(st + SM::kQW + 16384 + 8192, rec + RC::kW + 8192, 8192, bar);
                tma_load_4d(st + SM::kK, &tm_k, bar, 0, h, t0, b);
                tma_load_4d(st + SM::kK + 8192, &tm_k, bar, 64, h, t0, b);
                bulk_load(st + SM::kP, rec + RC::kPh, 16384, bar);
                bulk_load(st + SM::kU, rec + RC::kU + slice * RC::kUSlice, RC::kUSlice, bar);
                bulk_load(smem + SM::kG + buf * SM::kGate, rec + RC::kGate, SM::kGate, bar);
            }
        }
        __syncwarp();
    } else if (warp == 16 || warp == 17) {
        // ===== issuers A (warp 16) and B (warp 17): half of [Q;W] S each (d_k 0-63 /
        // 64-127), then half of K^T E each (tokens 0-31 / 32-63; B accumulates into
        // its [Y;X] columns, which every reader has drained by the time E is ready)
        if (lane == 0) {
            const int part = warp - 16;
            const uint32_t colXY = part ? kColXB : kColXA;
            const uint32_t colS = part ? kColXB : kColS;
            uint32_t full_phases = 0, e_phase = 0, r_phase = 0;
            for (int step = 0; step < nC; ++step) {
                const int buf = step & 1;
                const uint32_t st = stage_addr(step);
                if (part == 0) CHAIN_TS(0);
                wait_on(&full[buf], (full_phases >> buf) & 1u);
                full_phases ^= 1u << buf;
                if (step > 0) { wait_on(r_bar, r_phase); r_phase ^= 1; }
                if (part == 0) CHAIN_TS(1); else CHAIN_TS(23);
                if (*abort_s) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint64_t a = sdesc_sw128(st + SM::kQW + part * 16384 + k * 32);
                    mma_bf16(tmem + colXY, a, adv(dSL, (part * 4 + k) * 2048), idQW, k > 0);
                }
                if (part == 0) CHAIN_TS(6); else CHAIN_TS(8);
                mma_commit(xy_bar);
#ifdef GDN_CHAIN_TIMING
                if (part == 0) { mbar_wait(xy_bar, step & 1, kWaitTries); CHAIN_TS(7); }
#endif
                wait_on(e_bar, e_phase);
                e_phase ^= 1;
                if (part == 0) CHAIN_TS(2);
                if (*abort_s) break;
                tc_fence_after();
                const uint64_t dK = sdesc_sw128_mn(st + SM::kK, 8192);   // this stage's K tile
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int s = part * 2 + k;
                    mma_bf16(tmem + colS, adv(dK, s * 2048), adv(dE, s * 2048), idKE, k > 0);
                }
                mma_commit(s_bar);
                if (part == 0) CHAIN_TS(3);
                mma_commit(&free_st[buf]);
            }
        }
        __syncwarp();
    } else if (warp == 19) {
        // ===== issuer C: P D once D is written and K^T E is done (the chain's
        // product goes first) and the output warps have drained the previous P D;
        // then the TMA store of the staged output tile
        if (lane == 0) {
            uint32_t full_phases = 0, dd_phase = 0, s_phase = 0, pf_phase = 0, o_phase = 0;
            for (int step = 0; step < nC; ++step) {
                const int buf = step & 1;
                const int c = chunk_of(step);
                const uint32_t st = stage_addr(step);
                wait_on(&full[buf], (full_phases >> buf) & 1u);
                full_phases ^= 1u << buf;
                wait_on(dd_bar, dd_phase);
                dd_phase ^= 1;
                wait_on(s_bar, s_phase);
                s_phase ^= 1;
                CHAIN_TS(4);
                if (step > 0) { wait_on(pd_free, pf_phase); pf_phase ^= 1; }
                if (*abort_s) break;
                tc_fence_after();
                // [P_hi | P_lo] [D; D]: K-steps 0-3 read P_hi, 4-7 P_lo, both with D.
                // M = 128: rows 64-127 of A run on into the next 8 KB (P_lo, then U;
                // junk rows whose accumulator lanes are never read).
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const uint64_t a = sdesc_sw128(st + SM::kP + (s >> 2) * 8192 + (s & 3) * 32);
                    mma_bf16(tmem + kColPD, a, adv(dD, (s & 3) * 2048), idQW, s > 0);
                }
                mma_commit(pd_bar);
                CHAIN_TS(5);
                mma_commit(&free_st[buf]);
                if (out.mode == kOutStore) {
                    // the output warps staged the tile in this stage's U region
                    wait_on(o_bar, o_phase);
                    o_phase ^= 1;
                    if (*abort_s) break;
                    const unsigned char *ob = smem + buf * SM::kStage + SM::kU;
                    if (sizeof(Tout) == 4) {
                        tma_store_4d(&tm_o, ob, j0, h, c * 64, b);
                        tma_store_4d(&tm_o, ob + 8192, j0 + 32, h, c * 64, b);
                    } else {
                        tma_store_4d(&tm_o, ob, j0, h, c * 64, b);
                    }
                    bulk_commit_group();
                    bulk_wait_read_all();   // the stage may be reloaded after this
                    CHAIN_TS(24);
                }
                mbar_arrive(&free_st[buf]);
            }
            if (out.mode == kOutStore) bulk_wait_all();   // the output stores have landed
        }
        __syncwarp();
    } else {
        // ============================ epilogue warps (0..15) ========================
        // Lane quarter 2, 3 warps (X rows) and quarter 0, 1 warps (Y rows) pair up:
        // X warp (q + 2, cg) and Y warp (q, cg) cover the same 32 token rows and 16
        // columns.  X forms Delta (into the stage's U region, in place) and D; Y
        // forms E from that Delta, so both halves of the lane-quarter <-> SM
        // sub-partition binding share the Delta epilogue.
        const bool xrows = quarter >= 2;                 // TMEM lanes 64-127 hold X
        const int r = xrows ? d_row - 64 : d_row;        // token row (forward order) of this lane
        int uo[4], so[4], oo[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uo[q] = u_off(r, n0 + 4 * q);
            // output staging: fp32 boxes of 32 columns, or one bf16 box of 64
            oo[q] = sizeof(Tout) == 4 ? ((n0 + 4 * q) >> 5) * 8192 + sw128(r, ((n0 + 4 * q) & 31) * 2, 0)
                                      : sw128(r, n0 + 4 * q, 0);   // q = 0, 2 used
        }
        const int dof[4] = {swz_mn(n0, r, 8192), swz_mn(n0 + 8, r, 8192), swz_mn(NS + n0, r, 8192),
                            swz_mn(NS + n0 + 8, r, 8192)};
        so[0] = swz_mn(n0, d_row, 16384);
        so[1] = swz_mn(n0 + 8, d_row, 16384);
        so[2] = swz_mn(NS + n0, d_row, 16384);
        so[3] = swz_mn(NS + n0 + 8, d_row, 16384);
        uint32_t full_phases = 0, xy_phase = 0, dl_phase = 0, s_phase = 0, pd_phase = 0;
        for (int step = 0; step < nC; ++step) {
            const int buf = step & 1;
            const int c = chunk_of(step);
            unsigned char *ureg = smem + buf * SM::kStage + SM::kU;
            wait_on(&full[buf], (full_phases >> buf) & 1u);
            full_phases ^= 1u << buf;
            if (tid == 64) CHAIN_TS(9);
            if (tid == 0) CHAIN_TS(14);
            const float *gt = gates(step);
            const float ds = gt[128];
            const float dq = gt[r], dkk = gt[64 + r];
            // X rows overwrite D below: the previous P D must have read it
            if (xrows && step > 0) { wait_on(pd_bar, pd_phase); pd_phase ^= 1; }
            wait_on(xy_bar, xy_phase);
            xy_phase ^= 1;
            if (*abort_s) break;
            tc_fence_after();
            float acc[16];   // X (or Y) = (A hi + A lo) + (B hi + B lo)
            {
                float a0[16], a1[16], a2[16], a3[16];
                tmem_ld16(tmem + lane_base + kColXA + n0, a0);
                tmem_ld16(tmem + lane_base + kColXA + NS + n0, a1);
                tmem_ld16(tmem + lane_base + kColXB + n0, a2);
                tmem_ld16(tmem + lane_base + kColXB + NS + n0, a3);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) acc[e] = (a0[e] + a1[e]) + (a2[e] + a3[e]);
            }
            tc_fence_before();
            if (tid == 0) CHAIN_TS(15);
            if (xrows) {
                if (tid == 64) CHAIN_TS(10);
                // Delta = U - X, written back over U for the Y warps
                float d[16];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float4 u = *reinterpret_cast<const float4 *>(ureg + uo[q]);
                    u.x -= acc[4 * q]; u.y -= acc[4 * q + 1]; u.z -= acc[4 * q + 2]; u.w -= acc[4 * q + 3];
                    *reinterpret_cast<float4 *>(ureg + uo[q]) = u;
                    d[4 * q] = u.x; d[4 * q + 1] = u.y; d[4 * q + 2] = u.z; d[4 * q + 3] = u.w;
                }
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(delta_bar);
                    mbar_arrive(&free_st[buf]);   // done with the stage (Y warps hold it)
                }
                if (tid == 64) CHAIN_TS(21);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const float *x = d + 8 * hh;
                    uint4 dh, dl;
                    split2(x[0], x[1], dh.x, dl.x); split2(x[2], x[3], dh.y, dl.y);
                    split2(x[4], x[5], dh.z, dl.z); split2(x[6], x[7], dh.w, dl.w);
                    *reinterpret_cast<uint4 *>(smem + SM::kD + dof[hh]) = dh;
                    *reinterpret_cast<uint4 *>(smem + SM::kD + dof[2 + hh]) = dl;
                }
                fence_async_shared();
                __syncwarp();
                if (lane == 0) mbar_arrive(dd_bar);
                if (tid == 64) CHAIN_TS(11);
            } else {
                // E = dkk Delta from the X warps' Delta
                wait_on(delta_bar, dl_phase);
                dl_phase ^= 1;
                if (tid == 0) CHAIN_TS(20);
                if (*abort_s) break;
                float d[16];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 u = *reinterpret_cast<const float4 *>(ureg + uo[q]);
                    d[4 * q] = dkk * u.x; d[4 * q + 1] = dkk * u.y; d[4 * q + 2] = dkk * u.z; d[4 * q + 3] = dkk * u.w;
                }
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const float *x = d + 8 * hh;
                    uint4 eh, el;
                    split2(x[0], x[1], eh.x, el.x); split2(x[2], x[3], eh.y, el.y);
                    split2(x[4], x[5], eh.z, el.z); split2(x[6], x[7], eh.w, el.w);
                    *reinterpret_cast<uint4 *>(smem + SM::kE + dof[hh]) = eh;
                    *reinterpret_cast<uint4 *>(smem + SM::kE + dof[2 + hh]) = el;
                }
                fence_async_shared();
                __syncwarp();
                if (lane == 0) mbar_arrive(e_bar);
                if (tid == 0) CHAIN_TS(22);
            }
            // ---- S <- ds S + K^T E (two token halves, hi + lo each) -------------------
            wait_on(s_bar, s_phase);
            s_phase ^= 1;
            if (tid == 64) CHAIN_TS(12);
            if (tid == 0) CHAIN_TS(16);
            if (*abort_s) break;
            tc_fence_after();
            {
                float s0[16], s1[16], s2[16], s3[16];
                tmem_ld16(tmem + lane_base + kColS + n0, s0);
                tmem_ld16(tmem + lane_base + kColS + NS + n0, s1);
                tmem_ld16(tmem + lane_base + kColXB + n0, s2);
                tmem_ld16(tmem + lane_base + kColXB + NS + n0, s3);
                tmem_wait_ld();
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int n = 8 * hh;
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        S[n + e] = fmaf(ds, S[n + e], (s0[n + e] + s1[n + e]) + (s2[n + e] + s3[n + e]));
                    uint4 hi, lo;
                    split2(S[n], S[n + 1], hi.x, lo.x); split2(S[n + 2], S[n + 3], hi.y, lo.y);
                    split2(S[n + 4], S[n + 5], hi.z, lo.z); split2(S[n + 6], S[n + 7], hi.w, lo.w);
                    *reinterpret_cast<uint4 *>(smem + SM::kSL + so[hh]) = hi;
                    *reinterpret_cast<uint4 *>(smem + SM::kSL + so[2 + hh]) = lo;
                }
            }
            fence_async_shared();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(r_bar);
            if (tid == 64) CHAIN_TS(13);
            if (tid == 0) CHAIN_TS(17);
            if (xrows) continue;
            // ---- output rows: o = dq Y + P D ----------------------------------------
            wait_on(pd_bar, pd_phase);
            pd_phase ^= 1;
            if (*abort_s) break;
            tc_fence_after();
            float p0[16], p1[16];
            tmem_ld16(tmem + lane_base + kColPD + n0, p0);
            tmem_ld16(tmem + lane_base + kColPD + NS + n0, p1);
            tmem_wait_ld();
            if (tid == 0) CHAIN_TS(18);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(pd_free);
            float4 v[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                v[q].x = fmaf(dq, acc[4 * q], p0[4 * q] + p1[4 * q]);
                v[q].y = fmaf(dq, acc[4 * q + 1], p0[4 * q + 1] + p1[4 * q + 1]);
                v[q].z = fmaf(dq, acc[4 * q + 2], p0[4 * q + 2] + p1[4 * q + 2]);
                v[q].w = fmaf(dq, acc[4 * q + 3], p0[4 * q + 3] + p1[4 * q + 3]);
            }
            if (out.mode == kOutStore) {
                // stage the tile over this stage's U region (its Delta has been read)
                // as 128B-swizzled boxes of 128-byte rows; issuer C stores it
                if (sizeof(Tout) == 4) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) *reinterpret_cast<float4 *>(ureg + oo[q]) = v[q];
                } else {
#pragma unroll
                    for (int q = 0; q < 4; q += 2) {
                        uint4 w;
                        w.x = pack_bf16(v[q].x, v[q].y); w.y = pack_bf16(v[q].z, v[q].w);
                        w.z = pack_bf16(v[q + 1].x, v[q + 1].y); w.w = pack_bf16(v[q + 1].z, v[q + 1].w);
                        *reinterpret_cast<uint4 *>(ureg + oo[q]) = w;
                    }
                }
                fence_async_shared();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(o_bar);
                    mbar_arrive(&free_st[buf]);
                }
            } else {
                __syncwarp();
                if (lane == 0) mbar_arrive(&free_st[buf]);
                // pair mode: publish this direction's piece; the second finisher combines
                const int t = c * 64 + r;
                const size_t off = (((size_t)b * T + (t < T ? t : 0)) * H + h) * DV + j0 + n0;
                float *mine = dir ? out.part[1] : out.part[0];
                float *other = dir ? out.part[0] : out.part[1];
                if (t < T) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) *reinterpret_cast<float4 *>(mine + off + 4 * q) = v[q];
                }
                __threadfence();
                __syncwarp();
                unsigned int prior = 0;
                if (lane == 0) {
                    const size_t piece = (((size_t)bh * nC + c) * gridDim.x + slice) * 8 + quarter * 4 + cg;
                    prior = atomicAdd(out.cnt + piece, 1u);
                }
                prior = __shfl_sync(0xffffffffu, prior, 0);
                if (prior == 1u) {
                    __threadfence();
                    if (t < T) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float4 w = __ldcg(reinterpret_cast<const float4 *>(other + off + 4 * q));
                            float4 sum = v[q];
                            sum.x += w.x; sum.y += w.y; sum.z += w.z; sum.w += w.w;
                            store4<Tout>(out.o + off + 4 * q, sum);
                        }
                    }
                }
            }
            if (tid == 0) CHAIN_TS(19);
        }
        if (!*abort_s && state_out) {
            float *dst = state_out + ((size_t)bh * kDK + d_row) * DV + j0 + n0;
#pragma unroll
            for (int n = 0; n < 16; n += 4)
                *reinterpret_cast<float4 *>(dst + n) = make_float4(S[n], S[n + 1], S[n + 2], S[n + 3]);
        }
    }

    __syncthreads();
    if (*abort_s && tid == 0) {
        // a wait timed out: give copies and MMAs in flight a bounded chance to
        // land before shared memory and TMEM are released
        mbar_wait(&full[0], 0, 64);
        mbar_wait(&full[1], 0, 64);
        mbar_wait(s_bar, 0, 64);
        mbar_wait(pd_bar, 0, 64);
        mbar_wait(xy_bar, 0, 64);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kCols);
}

}  // namespace tc2
}  // namespace gdn
