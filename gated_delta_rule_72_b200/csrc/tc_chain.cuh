// tc_chain.cuh -- the inter-chunk state chain on the tensor cores.
//
// One CTA owns one (b, h), one direction and one segment of the chunk walk
// (the reverse direction walks the chunks last to first), with all DV
// columns of the d_k x DV state on chip: an fp32 master copy in registers and
// an fp16 copy in shared memory as the B operand of the tensor-core products.
// Per chunk, from the prep record (rows in forward token order):
//   [Y; X] = [Q~; W] S                  one M=128 product, two K halves
//   Delta  = U - X                      (fp16 D)
//   S     <- ds S + K~^T D
//   O      = Y + P D
// with Q~ = diag(e^g) Q and K~ = diag(e^{g_last - g}) K prepared by the prep
// kernel, so no per-row gate enters the chain.  Stacking Q~ over W makes Y
// and X one instruction stream: Y lands in TMEM lanes 0-63, X in 64-127.
// The chain's own products are split over two MMA streams (two issuing
// threads, two accumulators): a dependent tcgen05 MMA completes about every
// 130 cycles whatever N is up to 256, so the halves run side by side.
//
// TMEM (4 x DV columns): XA, XB hold the two K halves of [Y; X]; KA and then
// XA (once its X rows are read) the two token halves of K~^T D; OY holds O: a
// second [Q~; W] S product (one stream, issued while the X rows form D) puts
// Y there and P D accumulates onto it.  So the next chunk's [Q~; W] S waits
// only for the state, and the output stays off the chain's critical path.
//
// Roles (20 warps).  The 16 epilogue warps cover the 128 TMEM lanes four
// times (warp w reads lane quarter w % 4, columns DV/4 * (w / 4) .. +DV/4-1):
//   quarters 2, 3 (X rows)  Delta = U - X -> D             (critical path)
//   quarters 0, 1 (Y rows)  O = OY -> staged output tile
//   all                     S <- ds S + K~^T D, thread = one row of S
// Warps 16 and 17 issue the two halves of the chain's products (16 also
// the output's Y and P D) and warp 18 loads the records (one bulk copy per chunk,
// double-buffered).  A stage is free again once both issuers' products are
// done and every epilogue warp has read it.  The Y rows write the output
// straight to global memory from registers.  Roles meet on mbarriers; every
// wait is bounded and a wait that gives up sets an error flag and lets the
// kernel wind down.  A
// tcgen05.commit covers every earlier MMA of its issuing thread, so the
// [Y; X] product of a chunk completing also means that thread's P D of the
// chunk before has completed (and no longer reads D), and K~^T D completing
// means the output's Y product has read S.
//
// Sequence parallelism.  A chain of n chunks is cut into G segments of L
// chunks of the walk; segment g emits the outputs of walk steps
// [gL, min(n, (g+1)L)).  It starts from a zero state at an earlier step
// w0 <= gL, chosen so that the skipped transitions cannot matter: the state
// map of a chunk, M = prod_t alpha_t (I - beta_t k_t k_t^T), has 2-norm at
// most prod_t alpha_t max(1, |1 - beta_t |k_t|^2|) (each factor is a rank-one
// update of the identity), and the prep kernel writes the log of that bound
// per chunk.  Walking back from gL, w0 is the first step at which the summed
// bounds reach ln(2^-30); the state dropped at w0 then reaches step gL scaled
// by at most 2^-30, four orders of magnitude below the fp16 operand rounding.
// A walk that reaches step 0 without meeting the bound starts from the true
// initial state instead (exact).  Only the last segment writes the final
// state.  With fast-forgetting gates the walk back is a few chunks; with
// alpha = 1 it is the whole prefix (correct, but no faster than one segment).
//
// Bidirectional mode runs both directions in one launch; both add their rows
// into one zeroed fp32 sum with 16-byte atomic adds (an fp32 add of two values
// does not depend on their order, so the sum is deterministic).
#pragma once

#include "tc_common.cuh"

namespace gdn {
namespace tc2 {

template <int DV>
struct ChainSmem {
    static_assert(DV == 64 || DV == 128, "state width");
    // Two stages, each one record image (Rec<DV>).  The operands the
    // epilogues write are 128B-swizzled MN-major, as a tile load would write
    // them: S (K = d_k = 128 rows per 64-column group) and D (K = 64 tokens).
    // The output tile is staged in its own buffer, so a stage is free for the
    // next record as soon as its products are done.
    static constexpr int kStage = Rec<DV>::kStage;
    static constexpr int kGrpS = 128 * 128;
    static constexpr int kGrpD = 64 * 128;
    static constexpr int kS = 2 * kStage;
    static constexpr int kD = kS + (DV / 64) * kGrpS;
    static constexpr int kO = kD + (DV / 64) * kGrpD;    // output tile, fp32 staging
    static constexpr int kOBytes = 64 * DV * 4;
    static constexpr int kBar = kO + kOBytes;
    static constexpr int kCtl = kBar + 256;
    static constexpr int kBytes = kCtl + 32;
    // the dynamic shared memory is declared 1024-aligned (and checked at run
    // time), so no alignment slack is allocated
    static constexpr int kAlloc = kBytes;
    static_assert(kStage % 1024 == 0 && kS % 1024 == 0 && kD % 1024 == 0, "swizzled operands stay 1024-aligned");
    static_assert(kAlloc <= 232448, "shared memory budget");
};

constexpr int kChainThreads = 20 * 32;

enum OutMode { kOutStore = 0, kOutPair = 1 };

// Initial and final states per direction ([B, H, dk, d_v] fp32 each; null:
// zero / not written).  Direction 0 is the causal scan, 1 the reverse one.
// dk is the caller's key dimension (64 or 128); the chain always runs 128
// rows, those past dk staying zero (the prep pads keys and queries with zero
// columns).
struct ChainStates {
    const float *in[2];
    float *out[2];
    int dk;
};

// Output of a chain.  kOutStore: tm_o maps o ([B, T, H, DV], Tout), each
// tile stored once.  kOutPair (both directions): tm_o maps an fp32
// [B, T, H, DV] sum (o itself when Tout is float), zero on entry, onto which
// each direction's tiles are reduce-added by TMA (an fp32 add of two values,
// so the order does not matter).
template <typename Tout>
struct ChainOut {
    int mode;
};

// Staging of one output tile (64 rows x DV columns) for its TMA store: byte
// offset of the 16-byte chunk that starts at column `col` of row `row`.
// fp32: boxes of 32 columns (128-byte rows, 8 KB each, 128B swizzle); bf16:
// boxes of 64 columns (128-byte rows, 128B swizzle).
template <typename Tout>
__device__ __forceinline__ int out_stage_off(int row, int col) {
    if (sizeof(Tout) == 4) return (col >> 5) * 8192 + swz128(row * 128 + (col & 31) * 4);
    return (col >> 6) * 8192 + swz128(row * 128 + (col & 63) * 2);
}

// Segmentation of the chunk walk: G segments of L chunks; lb holds the log
// norm bound of every chunk's state map, [dir][b*H+h][chunk].
struct ChainSeg {
    int G, L;
    const float *lb;
};

// The chain of one (segment, bh, dir): block kChainThreads, `smem` its
// 1024-aligned shared memory (ChainSmem<DV>), nbh = B * H.  With `ready`
// non-null the prep records are produced alongside (by other CTAs of a
// cooperative launch) and each record's flag (and its log bound) is waited
// for, bounded, before it is used.
template <int DV, typename Tout>
__device__ __forceinline__ void chain_body(
    const CUtensorMap *tm_o, const unsigned char *__restrict__ recs, const ChainStates &states,
    const ChainOut<Tout> &out, const ChainSeg &seg, const unsigned int *__restrict__ ready, int H, int nC,
    int g, int bh, int dir, int nbh, unsigned char *smem, unsigned int *__restrict__ err)
{
    using SM = ChainSmem<DV>;
    using RC = Rec<DV>;
    constexpr int NC = DV / 4;          // columns per epilogue warp
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::kBar);
    uint64_t *full = bars + 0;         // [2] stage loaded                         (loader -> all)
    uint64_t *free_st = bars + 2;      // [2] stage consumed: A, B, 16 warps     (-> loader)
    uint64_t *xy_bar = bars + 4;       // [Y; X] complete, 2 commits               (A, B -> X warps)
    uint64_t *d_bar = bars + 5;        // D written, 8 X warps                     (-> A, B)
    uint64_t *s_bar = bars + 6;        // K~^T D complete, 2 commits               (-> epilogue)
    uint64_t *r_bar = bars + 7;        // S rewritten, 16 warps                    (-> A, B)
    uint64_t *pd_bar = bars + 8;       // Y + P D complete in OY, 1 commit          (-> Y warps)
    uint64_t *y_bar = bars + 9;        // O read out of OY, 8 Y warps               (-> A)
    uint64_t *o_bar = bars + 10;       // output tile staged, 8 Y warps            (-> storer)
    uint64_t *o_free = bars + 11;      // output buffer read by its store          (storer -> Y warps)
    uint32_t *tmem_base_s = reinterpret_cast<uint32_t *>(smem + SM::kCtl);
    volatile int *abort_s = reinterpret_cast<volatile int *>(smem + SM::kCtl + 4);
    volatile int *w0_s = reinterpret_cast<volatile int *>(smem + SM::kCtl + 8);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, cg = (warp >> 2) & 3;
    const int b = bh / H, h = bh % H;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int n0 = cg * NC;                                 // this warp's columns
    constexpr uint32_t kColXA = 0, kColXB = DV, kColKA = 2 * DV, kColOY = 3 * DV;
    constexpr uint32_t kCols = 4 * DV;
    const unsigned char *rec_base = recs + (size_t)(dir * nbh + bh) * nC * RC::kStride;
    const size_t flag_base = (size_t)(dir * nbh + bh) * nC;
    // this segment's outputs: walk steps [wb, we)
    const int wb = g * seg.L;
    const int we = min(nC, wb + seg.L);
    auto chunk_of = [&](int w) { return dir == 0 ? w : nC - 1 - w; };

    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(&free_st[0], 18);
        mbar_init(&free_st[1], 18);
        mbar_init(xy_bar, 2);
        mbar_init(d_bar, 8);
        mbar_init(s_bar, 2);
        mbar_init(r_bar, 16);
        mbar_init(pd_bar, 1);
        mbar_init(y_bar, 8);
        mbar_init(o_bar, 8);
        mbar_init(o_free, 1);
        fence_mbar_init();
        *abort_s = 0;
        prefetch_tensormap(tm_o);
    }
    if (warp == 0) {
        tmem_alloc(tmem_base_s, kCols);
        tmem_relinquish();
    }
    if (warp == 18 && lane == 0) {
        // where the walk starts: back from wb until the skipped state maps are
        // negligible (or step 0)
        int w = wb;
        if (wb > 0) {
            float acc = 0.f;
            while (w > 0) {
                --w;
                const int c = chunk_of(w);
                if (ready && !spin_until_geq(ready + flag_base + c, 1u, kFlagWaitNs)) {
                    *abort_s = 1;
                    if (err) atomicAdd(err, 1u);
                    break;
                }
                acc += ld_cg(seg.lb + flag_base + c);
                if (acc <= kLogWindow) break;
            }
        }
        *w0_s = w;
    }
    __syncthreads();
    const int w0 = *w0_s;
    const int nsteps = *abort_s ? 0 : we - w0;   // steps walked
    const int out0 = wb - w0;       // first step with output

    // State: epilogue thread (quarter, cg, lane) owns row d_row, columns n0 .. n0+NC-1.
    const int d_row = quarter * 32 + lane;
    auto s_off = [&](int n, int k) { return SM::kS + swz_mn(n, k, SM::kGrpS); };
    auto d_off = [&](int n, int k) { return SM::kD + swz_mn(n, k, SM::kGrpD); };
    float S[NC];
    if (warp < 16) {
        const float *state_in = (w0 == 0) ? (dir ? states.in[1] : states.in[0]) : nullptr;
        const float *src = (state_in && d_row < states.dk) ? state_in + ((size_t)bh * states.dk + d_row) * DV + n0
                                                           : nullptr;
#pragma unroll
        for (int n = 0; n < NC; ++n) S[n] = src ? src[n] : 0.f;
#pragma unroll
        for (int n = 0; n < NC; n += 8) {
            uint4 v;
            v.x = pack_f16(S[n], S[n + 1]); v.y = pack_f16(S[n + 2], S[n + 3]);
            v.z = pack_f16(S[n + 4], S[n + 5]); v.w = pack_f16(S[n + 6], S[n + 7]);
            *reinterpret_cast<uint4 *>(smem + s_off(n0 + n, d_row)) = v;
        }
    }
    fence_async_shared();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_s;

    auto wait_on = [&](uint64_t *bar, uint32_t parity) {
        if (!mbar_wait(bar, parity, kWaitTries)) {
            *abort_s = 1;
            if (err) atomicAdd(err, 1u);
        }
    };
    auto adv = [](uint64_t d, uint32_t bytes) { return d + (uint64_t)(bytes >> 4); };
    constexpr uint32_t idXY = idesc(128, DV, 0, 0, 1);   // [Q~;W] S and P D: A K-major, B MN-major
    constexpr uint32_t idKD = idesc(128, DV, 0, 1, 1);   // K~^T D: A MN-major (the key tile), B MN-major
    const uint64_t dS = sdesc_sw128_mn(sbase + SM::kS, SM::kGrpS);
    const uint64_t dD = sdesc_sw128_mn(sbase + SM::kD, SM::kGrpD);

    if (warp == 18) {
        // ============================ loader ========================================
        if (lane == 0 && !*abort_s) {
            uint32_t free_phases = 0;
            for (int step = 0; step < nsteps; ++step) {
                const int buf = step & 1;
                const int c = chunk_of(w0 + step);
                // the record is prepared alongside: wait until it has landed (polled
                // before the stage wait, which it then overlaps)
                if (ready && !spin_until_geq(ready + flag_base + c, 1u, kFlagWaitNs)) {
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
                uint64_t *bar = &full[buf];
                mbar_arrive_expect_tx(bar, RC::kBytes);
                bulk_load(smem + buf * SM::kStage, rec_base + (size_t)c * RC::kStride, RC::kBytes, bar);
            }
        }
        __syncwarp();
    } else if (warp == 16 || warp == 17) {
        // ===== issuers A (warp 16) and B (warp 17): one half of each chain product;
        // A also the output's [Q~; W] S into OY and P D onto it
        if (lane == 0) {
            const int part = warp - 16;
            const uint32_t colX = part ? kColXB : kColXA;
            const uint32_t colK = part ? kColXA : kColKA;   // B's half of K~^T D reuses XA
            uint32_t full_phases = 0, d_phase = 0, r_phase = 0, y_phase = 0;
            for (int step = 0; step < nsteps; ++step) {
                const int buf = step & 1;
                const uint32_t st = sbase + buf * SM::kStage;
                wait_on(&full[buf], (full_phases >> buf) & 1u);
                full_phases ^= 1u << buf;
                // S rewritten (and K~^T D read out of KA and XA)
                if (step > 0) { wait_on(r_bar, r_phase); r_phase ^= 1; }
                if (*abort_s) break;
                tc_fence_after();
                // [Y; X] half: d_k rows 64*part .. +63 of S
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint64_t a = sdesc_sw128(st + RC::kQW + part * 16384 + k * 32);
                    mma_bf16(tmem + colX, a, adv(dS, (part * 4 + k) * 2048), idXY, k > 0);
                }
                mma_commit(xy_bar);
                if (part == 0 && step >= out0) {
                    // the output's Y = [Q~; W] S into OY (rows 64-127 unused), once the
                    // previous chunk's O has been read out of OY
                    if (step > out0) { wait_on(y_bar, y_phase); y_phase ^= 1; }
                    if (*abort_s) break;
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint64_t a = sdesc_sw128(st + RC::kQW + (k >> 2) * 16384 + (k & 3) * 32);
                        mma_bf16(tmem + kColOY, a, adv(dS, k * 2048), idXY, k > 0);
                    }
                }
                // D written (X rows of XA, XB read)
                wait_on(d_bar, d_phase);
                d_phase ^= 1;
                if (*abort_s) break;
                tc_fence_after();
                // K~^T D half: tokens 32*part .. +31
                const uint64_t dK = sdesc_sw128_mn(st + RC::kK, 8192);
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int s = part * 2 + k;
                    mma_bf16(tmem + colK, adv(dK, s * 2048), adv(dD, s * 2048), idKD, k > 0);
                }
                mma_commit(s_bar);
                if (part == 0 && step >= out0) {
                    // P D onto Y in OY.  M = 128: rows 64-127 of A run on into U (finite;
                    // their lanes of OY are never read)
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_bf16(tmem + kColOY, sdesc_sw128(st + RC::kP + k * 32), adv(dD, k * 2048), idXY, 1);
                    mma_commit(pd_bar);
                }
                mma_commit(&free_st[buf]);
            }
        }
        __syncwarp();
    } else if (warp == 19) {
        // ===== storer: the staged output tile leaves by TMA (a bidirectional scan
        // reduce-adds both directions' tiles onto the zeroed fp32 sum)
        if (lane == 0) {
            const bool f32t = sizeof(Tout) == 4 || out.mode == kOutPair;
            const unsigned char *ob = smem + SM::kO;
            uint32_t o_phase = 0;
            for (int step = out0; step < nsteps; ++step) {
                const int c = chunk_of(w0 + step);
                wait_on(o_bar, o_phase);
                o_phase ^= 1;
                if (*abort_s) break;
                if (f32t) {
#pragma unroll
                    for (int x = 0; x < DV / 32; ++x) {
                        if (out.mode == kOutPair) tma_reduce_add_4d(tm_o, ob + x * 8192, 32 * x, h, c * 64, b);
                        else tma_store_4d(tm_o, ob + x * 8192, 32 * x, h, c * 64, b);
                    }
                } else {
#pragma unroll
                    for (int x = 0; x < DV / 64; ++x) tma_store_4d(tm_o, ob + x * 8192, 64 * x, h, c * 64, b);
                }
                bulk_commit_group();
                bulk_wait_read_all();            // the buffer may be refilled after this
                mbar_arrive(o_free);
            }
            bulk_wait_all();   // the output stores have landed
        }
        __syncwarp();
    } else {
        // ============================ epilogue warps (0..15) ========================
        const bool xrows = quarter >= 2;                 // TMEM lanes 64-127 hold X
        const int r = xrows ? d_row - 64 : d_row;        // token row (forward order) of this lane
        uint32_t full_phases = 0, xy_phase = 0, s_phase = 0, pd_phase = 0;
        for (int step = 0; step < nsteps; ++step) {
            const int buf = step & 1;
            const bool out_step = step >= out0;
            unsigned char *stg = smem + buf * SM::kStage;
            wait_on(&full[buf], (full_phases >> buf) & 1u);
            full_phases ^= 1u << buf;
            const float ds = *reinterpret_cast<const float *>(stg + RC::kGate);
            if (!xrows) {   // the Y rows read nothing else of the stage
                __syncwarp();
                if (lane == 0) mbar_arrive(&free_st[buf]);
            }
            if (xrows) {
                wait_on(xy_bar, xy_phase);
                xy_phase ^= 1;
                if (*abort_s) break;
                tc_fence_after();
                // ---- Delta = U - X -> D (fp16); the previous chunk's P D, issued before
                //      this [Y; X] by the same thread, has read the old D --------------
#pragma unroll
                for (int h16 = 0; h16 < NC; h16 += 16) {
                    float xa[16], xb[16];
                    tmem_ld16(tmem + lane_base + kColXA + n0 + h16, xa);
                    tmem_ld16(tmem + lane_base + kColXB + n0 + h16, xb);
                    const uint4 u0 = *reinterpret_cast<const uint4 *>(stg + RC::kU + u16_off<DV>(r, n0 + h16));
                    const uint4 u1 = *reinterpret_cast<const uint4 *>(stg + RC::kU + u16_off<DV>(r, n0 + h16 + 8));
                    tmem_wait_ld();
                    const uint32_t uu[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
                    uint32_t dd[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float2 u = unpack_f16(uu[e]);
                        dd[e] = pack_f16(u.x - (xa[2 * e] + xb[2 * e]), u.y - (xa[2 * e + 1] + xb[2 * e + 1]));
                    }
                    *reinterpret_cast<uint4 *>(smem + d_off(n0 + h16, r)) = make_uint4(dd[0], dd[1], dd[2], dd[3]);
                    *reinterpret_cast<uint4 *>(smem + d_off(n0 + h16 + 8, r)) = make_uint4(dd[4], dd[5], dd[6], dd[7]);
                }
                fence_async_shared();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&free_st[buf]);   // done reading the stage
                    mbar_arrive(d_bar);
                }
            }
            // ---- S <- ds S + K~^T D (token halves in KA and XA) ----------------------
            wait_on(s_bar, s_phase);
            s_phase ^= 1;
            if (*abort_s) break;
            tc_fence_after();
#pragma unroll
            for (int h16 = 0; h16 < NC; h16 += 16) {
                float ka[16], kb[16];
                tmem_ld16(tmem + lane_base + kColKA + n0 + h16, ka);
                tmem_ld16(tmem + lane_base + kColXA + n0 + h16, kb);
                tmem_wait_ld();
                uint32_t ss[8];
#pragma unroll
                for (int e = 0; e < 16; ++e) S[h16 + e] = fmaf(ds, S[h16 + e], ka[e] + kb[e]);
#pragma unroll
                for (int e = 0; e < 8; ++e) ss[e] = pack_f16(S[h16 + 2 * e], S[h16 + 2 * e + 1]);
                *reinterpret_cast<uint4 *>(smem + s_off(n0 + h16, d_row)) = make_uint4(ss[0], ss[1], ss[2], ss[3]);
                *reinterpret_cast<uint4 *>(smem + s_off(n0 + h16 + 8, d_row)) = make_uint4(ss[4], ss[5], ss[6], ss[7]);
            }
            fence_async_shared();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(r_bar);
            if (xrows || !out_step) continue;
            // ---- output rows: O = Y + P D out of OY ----------------------------------
            wait_on(pd_bar, pd_phase);
            pd_phase ^= 1;
            if (*abort_s) break;
            tc_fence_after();
            float o[NC];
#pragma unroll
            for (int h16 = 0; h16 < NC; h16 += 16) tmem_ld16(tmem + lane_base + kColOY + n0 + h16, o + h16);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(y_bar);   // OY may take the next chunk's Y
            // stage the tile in the output buffer once the store of the tile before
            // has read it (o_free completes once per tile; the k-th output tile
            // waits for the (k-1)-th completion, so it is never two phases behind)
            {
                const int k = step - out0;
                if (k > 0) wait_on(o_free, (uint32_t)((k - 1) & 1));
                if (*abort_s) break;
                unsigned char *ob = smem + SM::kO;
                if (sizeof(Tout) == 4 || out.mode == kOutPair) {
#pragma unroll
                    for (int q = 0; q < NC / 4; ++q)
                        *reinterpret_cast<float4 *>(ob + out_stage_off<float>(r, n0 + 4 * q)) =
                            make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
                } else {
#pragma unroll
                    for (int q = 0; q < NC / 8; ++q) {
                        uint4 w;
                        w.x = pack_bf16(o[8 * q], o[8 * q + 1]); w.y = pack_bf16(o[8 * q + 2], o[8 * q + 3]);
                        w.z = pack_bf16(o[8 * q + 4], o[8 * q + 5]); w.w = pack_bf16(o[8 * q + 6], o[8 * q + 7]);
                        *reinterpret_cast<uint4 *>(ob + out_stage_off<Tout>(r, n0 + 8 * q)) = w;
                    }
                }
                fence_async_shared();
                __syncwarp();
                if (lane == 0) mbar_arrive(o_bar);
            }
        }
        float *state_out = dir ? states.out[1] : states.out[0];
        if (!*abort_s && state_out && we == nC && d_row < states.dk) {
            float *dst = state_out + ((size_t)bh * states.dk + d_row) * DV + n0;
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
        mbar_wait(y_bar, 0, 64);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kCols);
}

// grid (G, B*H, directions), block kChainThreads; blockIdx.z is the direction
// (0 causal, 1 reverse), blockIdx.x the segment.
template <int DV, typename Tout>
__global__ void __launch_bounds__(kChainThreads, 1)
chain_kernel(const __grid_constant__ CUtensorMap tm_o, const unsigned char *__restrict__ recs,
             const ChainStates states, const ChainOut<Tout> out, const ChainSeg seg, int H, int nC,
             unsigned int *__restrict__ err)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    if (smem_u32(smem_raw) & 1023u) {   // no slack was allocated for aligning it here
        if (threadIdx.x == 0 && err) atomicAdd(err, 1u);
        return;
    }
    unsigned char *smem = smem_raw;
    chain_body<DV, Tout>(&tm_o, recs, states, out, seg, nullptr, H, nC, blockIdx.x, blockIdx.y, blockIdx.z,
                         gridDim.y, smem, err);
}

}  // namespace tc2
}  // namespace gdn
