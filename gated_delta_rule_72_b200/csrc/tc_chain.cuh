// tc_chain.cuh -- the inter-chunk state chain on the tensor cores.
//
// One CTA owns one (b, h), one direction and a slice of NS columns (32 or 64)
// of the d_k x d_v state (the columns evolve independently).  It walks the
// chunks in order (the reverse direction from the last chunk to the first)
// keeping its state slice on chip: an fp32 master copy in registers and a
// bf16 hi/lo copy in shared memory as the B operand of the tensor-core
// products.  Per chunk, from the prep record (rows in forward token order)
// and the bf16 Q and K tiles:
//   [Y; X] = [Q; W] [S_hi | S_lo]            one M=128 product
//   Delta = U - X,  E = diag(dkk) Delta
//   S <- ds S + K^T [E_hi | E_lo]
//   O = diag(dq) Y + [P_hi | P_lo] [D; D],  D = [Delta_hi | Delta_lo]
// The hi and lo halves of a split operand sit side by side along N, so one
// MMA of width 2*NS yields both partial products; P's halves are stacked
// along K instead, so the tensor core adds P_hi D + P_lo D itself.  Stacking
// Q over W makes Y and X one instruction stream; Y then lands in TMEM lanes
// 0-63 and X in lanes 64-127.
//
// What bounds a step.  An MMA stream (one issuing thread, one accumulator)
// completes one K=16 instruction per ~130 cycles whatever N is, so each
// product is split over two streams where TMEM has room.  The epilogues are
// bound by instruction issue (splitting a value into bf16 hi/lo costs about
// three instructions), and a TMEM lane quarter can only be read by the warps
// of the matching SM sub-partition, so the X rows' epilogue runs on two of
// the four.  NS = 32 halves the epilogues at the same MMA count; NS = 64
// halves the CTAs (and the record traffic) for a given head count.
//
// Roles (21 warps).  The 16 epilogue warps cover the 128 TMEM lanes four
// times (warp w reads lane quarter w % 4, columns NS/4 * (w / 4) .. +NS/4-1):
//   quarters 2, 3 (X rows)  form Delta, D and E        (critical path)
//   quarters 0, 1 (Y rows)  form and stage the output   (off the chain)
//   all                     S <- ds S + K^T E, thread = one row of S
// Warps 16 and 17 issue [Q;W] S, one K half each, and K^T E (one token half
// each when TMEM holds two accumulators for it, else warp 16 alone); warp 19
// issues P D, warp 20 stores the output tiles and warp 18 loads the stages.
// (Four streams for [Q;W] S, where TMEM has room, measured slower: the extra
// TMEM loads in the critical epilogue cost more than the shorter chains save.)  The
// roles meet on mbarriers, each of which can only complete its next phase
// after every waiter has observed the previous one.
//
// Bidirectional mode runs both directions in one launch (grid.z = 2), and
// both write the same fp32 output tiles.  An atomic counter per tile decides
// the order: the first of the two CTAs TMA-stores its tile and then marks it
// landed; the second waits for that mark (the two directions reach a given
// tile at very different times, so it seldom waits) and TMA-reduce-adds its
// own tile onto it.  The first one's mark does not depend on any other CTA,
// and the second only waits on a CTA that is already running.
#pragma once

#include "tc_common.cuh"

namespace gdn {
namespace tc2 {

#ifdef GDN_CHAIN_TIMING
// Development aid (not built into the library): cycle stamps of CTA (0,0,0),
// steps 10..19.
__device__ long long g_chain_ts[10][32];
__device__ long long g_chain_rarr[10][20];   // per-warp arrival on the S-rewritten barrier
#define CHAIN_TS(slot) do { if (slice == 0 && bh == 0 && dir == 0 && \
    step >= 10 && step < 20) g_chain_ts[step - 10][slot] = clock64(); } while (0)
#else
#define CHAIN_TS(slot) do { } while (0)
#endif

template <int NS>
struct ChainSmem {
    static_assert(NS == 32 || NS == 64, "slice width");
    // One stage (1024-aligned): [Q;W] 2 x 16 KB column blocks (Q rows 0-63,
    // W rows 64-127), K 2 x 8 KB, P_hi | P_lo 2 x 8 KB (all 128B-swizzled,
    // K-major), U as NS/32 granules of 64 x 32 fp32 (rows swizzled, u_off).
    // The operands the epilogues write, [S_hi | S_lo], [D_hi | D_lo] and
    // [E_hi | E_lo], are 128B-swizzled MN-major (one 128-byte row of 64 MN
    // elements per K index, hi and lo halves in separate 64-element groups when
    // NS = 64), as a tile load would write them: unswizzled layouts cost the
    // tensor core several times the shared-memory wavefronts.
    static constexpr int kQW = 0;
    static constexpr int kK = 32768;
    static constexpr int kP = kK + 16384;
    static constexpr int kU = kP + 16384;
    static constexpr int kStage = kU + 64 * NS * 4;
    static constexpr int kSL = 2 * kStage;                 // [S_hi | S_lo], K = 128
    static constexpr int kD = kSL + 128 * 2 * NS * 2;      // [D_hi | D_lo], K = 64
    static constexpr int kE = kD + 64 * 2 * NS * 2;        // [E_hi | E_lo], K = 64
    // Output staging: two dedicated buffers where there is room (NS = 32), so
    // that a stage is free for the next load as soon as its operands are used;
    // else (NS = 64) the tile is staged over the stage's U area once U is read.
    static constexpr bool kOwnOut = NS == 32;
    static constexpr int kOBytes = 64 * NS * 4;
    static constexpr int kO = kE + 64 * 2 * NS * 2;        // [2] output tiles (kOwnOut)
    static constexpr int kG = kO + (kOwnOut ? 2 * kOBytes : 0);   // 2 x gates (dq, dkk, ds)
    static constexpr int kGate = 528;
    static constexpr int kBar = kG + 2 * kGate;            // mbarriers
    static constexpr int kCtl = kBar + 128;
    static constexpr int kBytes = kCtl + 16;
    static constexpr int kAlloc = kBytes + 1024;
    // MN-group strides of the swizzled B operands (used when 2 * NS > 64)
    static constexpr int kGrpSL = 128 * 128, kGrpDE = 64 * 128;
    static_assert(kStage % 1024 == 0 && kSL % 1024 == 0 && kD % 1024 == 0 && kE % 1024 == 0,
                  "swizzled operands must stay 1024-aligned");
    static_assert(kAlloc <= 232448, "shared memory budget");
};

template <int NS>
__host__ __device__ constexpr int chain_threads() { return 21 * 32; }

enum OutMode { kOutStore = 0, kOutPair = 1 };

// Initial and final states per direction ([B, H, d_k, d_v] fp32 each; null:
// zero / not written).  Direction 0 is the causal scan, 1 the reverse one.
struct ChainStates {
    const float *in[2];
    float *out[2];
};

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

// Output of a chain.  kOutStore: tm_o maps o ([B, T, H, DV], Tout).  kOutPair
// (both directions): tm_o maps an fp32 [B, T, H, DV] sum (o itself when Tout
// is float), cnt holds one counter per output tile, zero on entry.
template <typename Tout>
struct ChainOut {
    unsigned int *cnt;
    int mode;
};

// Staging of one output tile (64 rows x NS columns) for its TMA store: byte
// offset of the 16-byte chunk that starts at column `col` of row `row`.
// fp32: boxes of 32 columns (128-byte rows, 8 KB each, 128B swizzle); bf16:
// one box of NS columns (128B swizzle for 128-byte rows, 64B for 64-byte rows).
template <int NS, typename Tout>
__device__ __forceinline__ int out_stage_off(int row, int col) {
    if (sizeof(Tout) == 4) return (col >> 5) * 8192 + swz128(row * 128 + (col & 31) * 4);
    return NS == 64 ? swz128(row * 128 + col * 2) : swz64(row * 64 + col * 2);
}

// NC consecutive TMEM columns (8 or 16) of this warp's lane quarter.
template <int NC>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float *v) {
    if (NC == 16) {
        tmem_ld16(taddr, v);
    } else {
        uint32_t r[8];
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                     : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                       "=r"(r[6]), "=r"(r[7])
                     : "r"(taddr));
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
    }
}

// The chain of one (slice, bh, dir): block chain_threads<NS>(), `smem` its
// 1024-aligned shared memory (ChainSmem<NS>); nslices = DV / NS, nbh = B * H.
// With `ready` non-null the prep records are produced alongside (by other CTAs
// of a cooperative launch) and each record's flag is waited for (bounded)
// before the record is loaded.
template <int DV, int NS, typename Tout>
__device__ __forceinline__ void chain_body(
    const CUtensorMap *tm_k, const CUtensorMap *tm_q, const CUtensorMap *tm_o,
    const unsigned char *__restrict__ recs, const ChainStates &states,
    const ChainOut<Tout> &out, const unsigned int *__restrict__ ready, int T, int H, int nC, int slice,
    int bh, int dir, int nslices, int nbh, unsigned char *smem, unsigned int *__restrict__ err)
{
    using SM = ChainSmem<NS>;
    using RC = Rec<DV>;
    constexpr int N2 = 2 * NS;          // accumulator width: hi | lo
    constexpr int NC = NS / 4;          // columns per epilogue warp
    constexpr bool kSplitS = 5 * N2 <= 512;   // K^T E in two streams (own TMEM columns)
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::kBar);
    uint64_t *full = bars + 0;         // [2] stage loaded                          (loader -> all)
    uint64_t *free_st = bars + 2;      // [2] stage consumed: 16 warps, A, B, C, storer (-> loader)
    uint64_t *xy_bar = bars + 4;       // [Y; X] complete, 2 commits                (A, B -> warps)
    uint64_t *d_bar = bars + 5;        // D and E written, 8 X warps                (-> A, B, C)
    uint64_t *s_bar = bars + 6;        // K^T E complete, 1 or 2 commits            (-> warps, C)
    uint64_t *r_bar = bars + 7;        // S rewritten, 16 warps                     (-> A, B)
    uint64_t *pd_bar = bars + 8;       // P D complete                              (C -> warps)
    uint64_t *pd_free = bars + 9;      // P D read, 8 Y warps                       (-> C)
    uint64_t *o_bar = bars + 10;       // output tile staged, 8 Y warps             (-> storer)
    uint64_t *o_seen = bars + 11;      // storer has seen o_bar's phase             (-> Y warps)
    uint64_t *o_free = bars + 12;      // [2] output buffer read by its store (kOwnOut, -> Y warps)
    uint32_t *tmem_base_s = reinterpret_cast<uint32_t *>(smem + SM::kCtl);
    volatile int *abort_s = reinterpret_cast<volatile int *>(smem + SM::kCtl + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, cg = (warp >> 2) & 3;
    const int b = bh / H, h = bh % H;
    const int j0 = slice * NS;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int n0 = cg * NC;                                 // this warp's columns of the slice
    // TMEM columns, each accumulator 2*NS wide (hi | lo): [Y;X] in two K halves,
    // K^T E (two token halves when kSplitS), P D
    constexpr uint32_t kColXA = 0, kColXB = N2, kColS = 2 * N2, kColPD = 3 * N2, kColSB = 4 * N2;
    constexpr uint32_t kCols = 512;
    static_assert(4 * N2 <= 512, "TMEM budget");
    static_assert(NS % kSliceCols == 0, "the record stores U in granules of kSliceCols columns");
    const unsigned char *rec_base = recs + (size_t)(dir * nbh + bh) * nC * RC::kBytes;

    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        // 16 warps and the commits of A, B, C; the storer too when the output
        // tile is staged inside the stage
        mbar_init(&free_st[0], SM::kOwnOut ? 19 : 20);
        mbar_init(&free_st[1], SM::kOwnOut ? 19 : 20);
        mbar_init(&o_free[0], 1);
        mbar_init(&o_free[1], 1);
        mbar_init(xy_bar, 2);
        mbar_init(d_bar, 8);
        mbar_init(s_bar, kSplitS ? 2 : 1);
        mbar_init(r_bar, 16);
        mbar_init(pd_bar, 1);
        mbar_init(pd_free, 8);
        mbar_init(o_bar, 8);
        mbar_init(o_seen, 1);
        fence_mbar_init();
        *abort_s = 0;
        prefetch_tensormap(tm_k);
        prefetch_tensormap(tm_q);
        prefetch_tensormap(tm_o);
    }
    if (warp == 0) {
        tmem_alloc(tmem_base_s, kCols);
        tmem_relinquish();
    }
    // Offsets of this thread's pieces of the split operands.  State: epilogue
    // thread (quarter, cg, lane) owns row d_row, columns n0 .. n0+NC-1.
    const int d_row = quarter * 32 + lane;
    auto sl_off = [&](int n, int k) { return (N2 > 64 ? (n >> 6) * SM::kGrpSL : 0) + swz128(k * 128 + (n & 63) * 2); };
    auto de_off = [&](int n, int k) { return (N2 > 64 ? (n >> 6) * SM::kGrpDE : 0) + swz128(k * 128 + (n & 63) * 2); };
    float S[NC];
    if (warp < 16) {
        const float *state_in = dir ? states.in[1] : states.in[0];   // (a select: no local copy)
        const float *src = state_in ? state_in + ((size_t)bh * kDK + d_row) * DV + j0 + n0 : nullptr;
#pragma unroll
        for (int n = 0; n < NC; ++n) S[n] = src ? src[n] : 0.f;
#pragma unroll
        for (int n = 0; n < NC; n += 8) {
            uint4 hi, lo;
            split2(S[n], S[n + 1], hi.x, lo.x); split2(S[n + 2], S[n + 3], hi.y, lo.y);
            split2(S[n + 4], S[n + 5], hi.z, lo.z); split2(S[n + 6], S[n + 7], hi.w, lo.w);
            *reinterpret_cast<uint4 *>(smem + SM::kSL + sl_off(n0 + n, d_row)) = hi;
            *reinterpret_cast<uint4 *>(smem + SM::kSL + sl_off(NS + n0 + n, d_row)) = lo;
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
    // MN-major swizzled B operands; a K-step of 16 rows advances 2048 bytes
    const uint64_t dSL = sdesc_sw128_mn(sbase + SM::kSL, SM::kGrpSL);
    const uint64_t dD = sdesc_sw128_mn(sbase + SM::kD, SM::kGrpDE);
    const uint64_t dE = sdesc_sw128_mn(sbase + SM::kE, SM::kGrpDE);

    if (warp == 18) {
        // ============================ loader ========================================
        if (lane == 0) {
            uint32_t free_phases = 0;
            for (int step = 0; step < nC; ++step) {
                const int buf = step & 1;
                const int c = chunk_of(step);
                // the record is prepared alongside: wait until it has landed (polled
                // before the stage wait, which it then overlaps)
                if (ready && !spin_until_geq(ready + (size_t)(dir * nbh + bh) * nC + c, 1u, kFlagWaitNs)) {
                    *abort_s = 1;
                    if (err) atomicAdd(err, 1u);
                    break;
                }
                if (step >= 2) {   // the stage's previous chunk has been consumed
                    wait_on(&free_st[buf], (free_phases >> buf) & 1u);
                    free_phases ^= 1u << buf;
                }
                if (*abort_s) break;
                if (ready) fence_proxy_async_global();
                unsigned char *st = smem + buf * SM::kStage;
                const unsigned char *rec = rec_base + (size_t)c * RC::kBytes;
                uint64_t *bar = &full[buf];
                mbar_arrive_expect_tx(bar, 4 * 16384 + 64 * NS * 4 + SM::kGate);
                const int t0 = c * 64;
                tma_load_4d(st + SM::kQW, tm_q, bar, 0, h, t0, b);
                tma_load_4d(st + SM::kQW + 16384, tm_q, bar, 64, h, t0, b);
                bulk_load(st + SM::kQW + 8192, rec + RC::kW, 8192, bar);
                bulk_load(st + SM::kQW + 16384 + 8192, rec + RC::kW + 8192, 8192, bar);
                tma_load_4d(st + SM::kK, tm_k, bar, 0, h, t0, b);
                tma_load_4d(st + SM::kK + 8192, tm_k, bar, 64, h, t0, b);
                bulk_load(st + SM::kP, rec + RC::kPh, 16384, bar);
                bulk_load(st + SM::kU, rec + RC::kU + j0 * 64 * 4, 64 * NS * 4, bar);
                bulk_load(smem + SM::kG + buf * SM::kGate, rec + RC::kGate, SM::kGate, bar);
            }
        }
        __syncwarp();
    } else if (warp == 16 || warp == 17) {
        // ===== issuers A (warp 16) and B (warp 17): half of [Q;W] S each (d_k 0-63 /
        // 64-127), then K^T E: tokens 0-31 / 32-63 into separate accumulators
        // when kSplitS, else all of it from A
        if (lane == 0) {
            const int part = warp - 16;
            const uint32_t colXY = part ? kColXB : kColXA;
            const uint32_t colS = part ? kColSB : kColS;
            uint32_t full_phases = 0, d_phase = 0, r_phase = 0;
            for (int step = 0; step < nC; ++step) {
                const int buf = step & 1;
                const uint32_t st = stage_addr(step);
                if (part == 0) CHAIN_TS(0);
                wait_on(&full[buf], (full_phases >> buf) & 1u);
                full_phases ^= 1u << buf;
                if (part == 0) CHAIN_TS(25);
                if (step > 0) { wait_on(r_bar, r_phase); r_phase ^= 1; }
                if (part == 0) CHAIN_TS(1); else CHAIN_TS(23);
                if (*abort_s) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int s = part * 4 + k;
                    const uint64_t a = sdesc_sw128(st + SM::kQW + (s >> 2) * 16384 + (s & 3) * 32);
                    mma_bf16(tmem + colXY, a, adv(dSL, s * 2048), idQW, k > 0);
                }
                if (part == 0) CHAIN_TS(6); else CHAIN_TS(8);
                mma_commit(xy_bar);
#ifdef GDN_CHAIN_TIMING
                if (part == 0) { mbar_wait(xy_bar, step & 1, kWaitTries); CHAIN_TS(7); }
#endif
                if (kSplitS || part == 0) {
                    wait_on(d_bar, d_phase);
                    d_phase ^= 1;
                    if (part == 0) CHAIN_TS(2);
                    if (*abort_s) break;
                    tc_fence_after();
                    const uint64_t dK = sdesc_sw128_mn(st + SM::kK, 8192);   // this stage's K tile
                    constexpr int kSteps = kSplitS ? 2 : 4;
#pragma unroll
                    for (int k = 0; k < kSteps; ++k) {
                        const int s = part * kSteps + k;
                        mma_bf16(tmem + colS, adv(dK, s * 2048), adv(dE, s * 2048), idKE, k > 0);
                    }
                    mma_commit(s_bar);
                    if (part == 0) CHAIN_TS(3);
                }
                mma_commit(&free_st[buf]);
            }
        }
        __syncwarp();
    } else if (warp == 19) {
        // ===== issuer C: P D once D is written and K^T E is done (the chain's
        // product goes first) and the output warps have drained the previous P D
        if (lane == 0) {
            uint32_t full_phases = 0, d_phase = 0, s_phase = 0, pf_phase = 0;
            for (int step = 0; step < nC; ++step) {
                const int buf = step & 1;
                const uint32_t st = stage_addr(step);
                wait_on(&full[buf], (full_phases >> buf) & 1u);
                full_phases ^= 1u << buf;
                wait_on(d_bar, d_phase);
                d_phase ^= 1;
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
            }
        }
        __syncwarp();
    } else if (warp == 20) {
        // ===== storer: the staged output tile leaves by TMA; in a bidirectional
        // scan the second of the two directions adds its tile onto the first's
        if (lane == 0) {
            uint32_t o_phase = 0;
            for (int step = 0; step < nC; ++step) {
                const int buf = step & 1;
                const int c = chunk_of(step);
                // the output warps staged the tile (own buffer, or the stage's U area)
                wait_on(o_bar, o_phase);
                o_phase ^= 1;
                mbar_arrive(o_seen);   // o_bar may complete its next phase
                if (*abort_s) break;
                const unsigned char *ob = SM::kOwnOut ? smem + SM::kO + buf * SM::kOBytes
                                                      : smem + buf * SM::kStage + SM::kU;
                bool add = false;      // TMA-reduce-add onto the other direction's tile
                size_t tile = 0;
                if (out.mode == kOutPair) {
                    tile = ((size_t)bh * nC + c) * nslices + slice;
                    if (atomicAdd(out.cnt + tile, 1u) != 0u) {
                        // second: wait for the first one's "landed" mark (+2)
                        if (!spin_until_geq(out.cnt + tile, 3u, kFlagWaitNs)) {
                            *abort_s = 1;
                            if (err) atomicAdd(err, 1u);
                            break;
                        }
                        fence_proxy_async_global();
                        add = true;
                    }
                }
                if (sizeof(Tout) == 4 || out.mode == kOutPair) {
#pragma unroll
                    for (int x = 0; x < NS / 32; ++x) {
                        if (add) tma_reduce_add_4d(tm_o, ob + x * 8192, j0 + 32 * x, h, c * 64, b);
                        else tma_store_4d(tm_o, ob + x * 8192, j0 + 32 * x, h, c * 64, b);
                    }
                } else {
                    tma_store_4d(tm_o, ob, j0, h, c * 64, b);
                }
                bulk_commit_group();
                bulk_wait_read_all();            // the staging buffer may be reused after this
                CHAIN_TS(27);
                mbar_arrive(SM::kOwnOut ? &o_free[buf] : &free_st[buf]);
                if (out.mode == kOutPair && !add) {
                    bulk_wait_all();             // landed in global memory: mark it (+2)
                    fence_proxy_async_global();
                    __threadfence();
                    atomicAdd(out.cnt + tile, 2u);
                }
            }
            bulk_wait_all();   // the output stores have landed
        }
        __syncwarp();
    } else {
        // ============================ epilogue warps (0..15) ========================
        const bool xrows = quarter >= 2;                 // TMEM lanes 64-127 hold X
        const int r = xrows ? d_row - 64 : d_row;        // token row (forward order) of this lane
        uint32_t full_phases = 0, xy_phase = 0, s_phase = 0, pd_phase = 0, os_phase = 0, of_phases = 0;
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
            const float dg = xrows ? gt[64 + r] : gt[r];   // dkk for X rows, dq for Y rows
            if (SM::kOwnOut && !xrows) {   // Y rows are done with the stage
                __syncwarp();
                if (lane == 0) mbar_arrive(&free_st[buf]);
            }
            // X rows overwrite D below: the previous P D must have read it
            if (xrows && step > 0) { wait_on(pd_bar, pd_phase); pd_phase ^= 1; }
            wait_on(xy_bar, xy_phase);
            xy_phase ^= 1;
            if (*abort_s) break;
            tc_fence_after();
            float acc[NC];   // X (or Y) = (A hi + A lo) + (B hi + B lo)
            {
                float a0[NC], a1[NC], a2[NC], a3[NC];
                tmem_ld_cols<NC>(tmem + lane_base + kColXA + n0, a0);
                tmem_ld_cols<NC>(tmem + lane_base + kColXA + NS + n0, a1);
                tmem_ld_cols<NC>(tmem + lane_base + kColXB + n0, a2);
                tmem_ld_cols<NC>(tmem + lane_base + kColXB + NS + n0, a3);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < NC; ++e) acc[e] = (a0[e] + a1[e]) + (a2[e] + a3[e]);
            }
            if (tid == 0) CHAIN_TS(15);
            if (xrows) {
                if (tid == 64) CHAIN_TS(10);
                float d[NC];
#pragma unroll
                for (int q = 0; q < NC / 4; ++q) {
                    const int col = n0 + 4 * q;
                    const float4 u = *reinterpret_cast<const float4 *>(ureg + (col >> 5) * RC::kUSlice + u_off(r, col & 31));
                    d[4 * q] = u.x - acc[4 * q];
                    d[4 * q + 1] = u.y - acc[4 * q + 1];
                    d[4 * q + 2] = u.z - acc[4 * q + 2];
                    d[4 * q + 3] = u.w - acc[4 * q + 3];
                }
                if (tid == 64) CHAIN_TS(21);
                __syncwarp();
                if (lane == 0) mbar_arrive(&free_st[buf]);   // done reading the stage
#pragma unroll
                for (int h8 = 0; h8 < NC; h8 += 8) {
                    const float *x = d + h8;
                    uint4 dh, dl, eh, el;
                    split2(x[0], x[1], dh.x, dl.x); split2(x[2], x[3], dh.y, dl.y);
                    split2(x[4], x[5], dh.z, dl.z); split2(x[6], x[7], dh.w, dl.w);
                    split2(dg * x[0], dg * x[1], eh.x, el.x); split2(dg * x[2], dg * x[3], eh.y, el.y);
                    split2(dg * x[4], dg * x[5], eh.z, el.z); split2(dg * x[6], dg * x[7], eh.w, el.w);
                    const int oh = de_off(n0 + h8, r), ol = de_off(NS + n0 + h8, r);
                    *reinterpret_cast<uint4 *>(smem + SM::kD + oh) = dh;
                    *reinterpret_cast<uint4 *>(smem + SM::kD + ol) = dl;
                    *reinterpret_cast<uint4 *>(smem + SM::kE + oh) = eh;
                    *reinterpret_cast<uint4 *>(smem + SM::kE + ol) = el;
                }
                if (tid == 64) CHAIN_TS(22);
                fence_async_shared();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(d_bar);
                if (tid == 64) CHAIN_TS(11);
            }
            // ---- S <- ds S + K^T E (hi + lo; two token halves when split) --------
            wait_on(s_bar, s_phase);
            s_phase ^= 1;
            if (tid == 64) CHAIN_TS(12);
            if (tid == 0) CHAIN_TS(16);
            if (*abort_s) break;
            tc_fence_after();
            {
                float s0[NC], s1[NC], s2[NC], s3[NC];
                tmem_ld_cols<NC>(tmem + lane_base + kColS + n0, s0);
                tmem_ld_cols<NC>(tmem + lane_base + kColS + NS + n0, s1);
                if (kSplitS) {
                    tmem_ld_cols<NC>(tmem + lane_base + kColSB + n0, s2);
                    tmem_ld_cols<NC>(tmem + lane_base + kColSB + NS + n0, s3);
                }
                tmem_wait_ld();
#pragma unroll
                for (int n = 0; n < NC; n += 8) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float dS = kSplitS ? (s0[n + e] + s1[n + e]) + (s2[n + e] + s3[n + e])
                                                 : s0[n + e] + s1[n + e];
                        S[n + e] = fmaf(ds, S[n + e], dS);
                    }
                    uint4 hi, lo;
                    split2(S[n], S[n + 1], hi.x, lo.x); split2(S[n + 2], S[n + 3], hi.y, lo.y);
                    split2(S[n + 4], S[n + 5], hi.z, lo.z); split2(S[n + 6], S[n + 7], hi.w, lo.w);
                    *reinterpret_cast<uint4 *>(smem + SM::kSL + sl_off(n0 + n, d_row)) = hi;
                    *reinterpret_cast<uint4 *>(smem + SM::kSL + sl_off(NS + n0 + n, d_row)) = lo;
                }
            }
            fence_async_shared();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(r_bar);
#ifdef GDN_CHAIN_TIMING
            if (lane == 0 && slice == 0 && bh == 0 && dir == 0 && step >= 10 && step < 20)
                g_chain_rarr[step - 10][warp] = clock64();
#endif
            if (tid == 64) CHAIN_TS(13);
            if (tid == 0) CHAIN_TS(17);
            if (xrows) continue;
            // ---- output rows: o = dq Y + P D ----------------------------------------
            wait_on(pd_bar, pd_phase);
            pd_phase ^= 1;
            if (*abort_s) break;
            tc_fence_after();
            float p0[NC], p1[NC];
            tmem_ld_cols<NC>(tmem + lane_base + kColPD + n0, p0);
            tmem_ld_cols<NC>(tmem + lane_base + kColPD + NS + n0, p1);
            tmem_wait_ld();
            if (tid == 0) CHAIN_TS(18);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(pd_free);
            float4 v[NC / 4];
#pragma unroll
            for (int q = 0; q < NC / 4; ++q) {
                v[q].x = fmaf(dg, acc[4 * q], p0[4 * q] + p1[4 * q]);
                v[q].y = fmaf(dg, acc[4 * q + 1], p0[4 * q + 1] + p1[4 * q + 1]);
                v[q].z = fmaf(dg, acc[4 * q + 2], p0[4 * q + 2] + p1[4 * q + 2]);
                v[q].w = fmaf(dg, acc[4 * q + 3], p0[4 * q + 3] + p1[4 * q + 3]);
            }
            // stage the tile for the storer (own double buffer, or over this stage's
            // U area, which is read by now); both directions of a bidirectional scan
            // add up in fp32
            unsigned char *ob = ureg;
            if (SM::kOwnOut) {
                ob = smem + SM::kO + buf * SM::kOBytes;
                if (step >= 2) {   // the store two tiles back has read this buffer
                    wait_on(&o_free[buf], (of_phases >> buf) & 1u);
                    of_phases ^= 1u << buf;
                }
            }
            if (sizeof(Tout) == 4 || out.mode == kOutPair) {
#pragma unroll
                for (int q = 0; q < NC / 4; ++q)
                    *reinterpret_cast<float4 *>(ob + out_stage_off<NS, float>(r, n0 + 4 * q)) = v[q];
            } else {
#pragma unroll
                for (int q = 0; q < NC / 4; q += 2) {
                    uint4 w;
                    w.x = pack_bf16(v[q].x, v[q].y); w.y = pack_bf16(v[q].z, v[q].w);
                    w.z = pack_bf16(v[q + 1].x, v[q + 1].y); w.w = pack_bf16(v[q + 1].z, v[q + 1].w);
                    *reinterpret_cast<uint4 *>(ob + out_stage_off<NS, Tout>(r, n0 + 4 * q)) = w;
                }
            }
            fence_async_shared();
            // o_bar completes one phase per tile: not before the storer has seen the last
            if (step > 0) { wait_on(o_seen, os_phase); os_phase ^= 1; }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(o_bar);
                if (!SM::kOwnOut) mbar_arrive(&free_st[buf]);
            }
            if (tid == 0) CHAIN_TS(19);
        }
        float *state_out = dir ? states.out[1] : states.out[0];
        if (!*abort_s && state_out) {
            float *dst = state_out + ((size_t)bh * kDK + d_row) * DV + j0 + n0;
#pragma unroll
            for (int n = 0; n < NC; n += 4)
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

// grid (DV/NS, B*H, directions), block chain_threads<NS>(); blockIdx.z is the
// direction (0 causal, 1 reverse).
template <int DV, int NS, typename Tout>
__global__ void __launch_bounds__(chain_threads<NS>(), 1)
chain_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
             const __grid_constant__ CUtensorMap tm_o, const unsigned char *__restrict__ recs,
             const ChainStates states, const ChainOut<Tout> out,
             int T, int H, int nC, unsigned int *__restrict__ err)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    chain_body<DV, NS, Tout>(&tm_k, &tm_q, &tm_o, recs, states, out, nullptr, T, H, nC, blockIdx.x,
                             blockIdx.y, blockIdx.z, gridDim.x, gridDim.y, smem, err);
}

}  // namespace tc2
}  // namespace gdn
