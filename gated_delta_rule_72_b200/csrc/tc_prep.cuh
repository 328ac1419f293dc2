// tc_prep.cuh -- chunk preparation on the tensor cores (tcgen05 + TMA).
//
// For every chunk of 64 tokens of every (b, h) and direction (fully
// parallel; a persistent grid of two pipelines per SM walks the tasks and
// fetches the next task's tiles with TMA while it finishes the current one)
// this kernel computes, in the chunk's processing order r = 0..63 (the
// reverse direction walks a chunk back to front):
//   g_r = sum_{m<=r} log alpha_m                          (prefix sum, fp32)
//   [K; Q] K^T                                            (kind::f16 bf16, M=128, exact)
//   L_rs = beta_r e^{g_r-g_s} (KK^T)_rs, s < r             (fp32)
//   P_rs = e^{g_r-g_s} (QK^T)_rs, s <= r   (forward)     | readout mask
//        = e^{g_{r-1}-g_s} (QK^T)_rs, s < r (reverse)    |
//   T = (I + L)^{-1}                                      (blocked 16x16, CUDA cores)
//   W = T diag(beta e^g) K,  U = T diag(beta) V           (kind::f16 bf16: T diag(beta e^g)
//                                                          single, T diag(beta) as a hi/lo pair)
//   Q~_r = dq_r q_r, dq_r = e^{g_r} (reverse: e^{g_{r-1}});  K~_r = e^{g_63 - g_r} k_r
//   ds = e^{g_63}
// and writes them as one fp16 record (tc_common.cuh) with rows in forward
// token order: for the reverse direction every row and column index is
// mirrored (r -> 63 - r), so that the chain kernel never needs to know the
// direction.  Beside the record it writes the log of a bound on the 2-norm of
// the chunk's state map, g_63 + sum_r ln max(1, |1 - beta_r |k_r|^2|), which
// the chain uses to decide where a segment may start from a zero state.
#pragma once

#include "tc_common.cuh"

namespace gdn {
namespace tc2 {

// Gate vectors of one task (fp32, processing order), computed one task ahead.
struct PrepGate {
    static constexpr int kG = 0;       // g_r, prefix sums of log alpha
    static constexpr int kBeta = 64;   // beta_r
    static constexpr int kDq = 128;    // e^{g_r} (reverse: e^{g_{r-1}}), the query scale
    static constexpr int kDkk = 192;   // e^{g_63 - g_r}, the key scale of the state update
    static constexpr int kBg = 256;    // beta_r e^{g_r}
    static constexpr int kFacs = 320;  // e^{g_16k - g_r}, k = r / 16 (mask decay factors)
    static constexpr int kFast = 384;  // (int) 1 if every 16-token block decays by less than 80
    static constexpr int kDs = 385;    // e^{g_63}
    static constexpr int kFloats = 392;
};

template <int DV>
struct PrepSmem {
    static constexpr int kKQ = 32768;                 // [K|Q] x 2 column blocks, 128B swizzle
    static constexpr int kVb = 64 * DV * 2;           // V, 64-column blocks of 8 KB
    static constexpr int kStage = kKQ + kVb;          // one stage, 1024-aligned
    static constexpr int kL = kStage;                 // [64][65] fp32
    static constexpr int kT = kL + 64 * 65 * 4;       // [64][65] fp32
    static constexpr int kX = kT + 64 * 65 * 4;       // 2 x [16][16] fp32 (level-2 scratch)
    static constexpr int kT1 = (kX + 2 * 256 * 4 + 1023) / 1024 * 1024;   // bf16 K-major 64 x 64
    static constexpr int kT2h = kT1 + 8192;           // T diag(beta), bf16 hi
    static constexpr int kT2l = kT2h + 8192;          // and lo
    static constexpr int kGate = kT2l + 8192;         // two gate buffers (PrepGate), by task parity
    static constexpr int kMisc = kGate + 2 * 4 * PrepGate::kFloats;   // key-norm partials [2], record gate [4], task [2][4]
    static constexpr int kBar = kMisc + 64;           // tma, mma, gram
    static constexpr int kCtl = kBar + 32;            // tmem base, abort, ds
    static constexpr int kBytes = kCtl + 16;
    static constexpr int kAlloc = kBytes + 1024;
    static_assert(kStage % 1024 == 0 && kT1 % 1024 == 0, "swizzled areas stay 1024-aligned");
    // record staging: P and W images over T1 | T2h, U over L
    static_assert(64 * DV * 2 <= 2 * 64 * 65 * 4, "record staging areas");
    static_assert(kAlloc <= 232448 / 2 - 1024, "two pipelines per SM");
};

constexpr int kPrepThreads = 256;
constexpr int kPrepCtasPerSm = 2;
constexpr uint32_t kPrepColG = 0;      // Gram [K; Q] K^T, 128 lanes x 64 (dead before W is written)
constexpr uint32_t kPrepColW = 0;      // M=64 x 128
constexpr uint32_t kPrepColU = 128;    // M=64 x DV
constexpr uint32_t kPrepTmemCols = 256;

// Order of the prep tasks.  The chains of a launch are cut into G segments
// of L chunks (walk order); a segment first walks back into the tail of the
// segment before it.  So the tasks come position by position within the
// segments, the last `tail` positions first (from the end backwards), then
// the rest from the front; within a position: segment, direction, (b, h).
struct PrepOrder {
    int G, L, tail;
};

__device__ __forceinline__ bool prep_task(const PrepOrder &po, int t, int nbh, int ndir, int nC, int &dir,
                                          int &c, int &bh) {
    const int per = nbh * ndir * po.G;
    const int j = t / per, rem = t - j * per;
    bh = rem % nbh;
    dir = (rem / nbh) % ndir;
    const int g = rem / (nbh * ndir);
    const int p = j < po.tail ? po.L - 1 - j : j - po.tail;
    const int w = g * po.L + p;
    c = dir == 0 ? w : nC - 1 - w;
    return w < nC;
}

// One prep pipeline: 256 threads (ptid 0..255) with their own 1024-aligned
// shared-memory area `smem` (PrepSmem<DV>), 256 TMEM columns from `tmem` and
// named barriers `bar_id` (all 256 threads) and `aux_id` (warps 0-3); it
// walks tasks first_task, first_task + stride, ...
// (po order).  With `ready` non-null, each record's flag is set (release) once
// its stores have landed, for a chain kernel that runs alongside.
template <int DV>
__device__ __forceinline__ void prep_pipeline(
    const CUtensorMap *tm_k, const CUtensorMap *tm_q, const CUtensorMap *tm_v,
    const float *__restrict__ alpha, const float *__restrict__ beta, unsigned char *__restrict__ recs,
    float *__restrict__ lb, unsigned int *__restrict__ ready, int T, int H, int nC, int nbh, int ndir,
    PrepOrder po, int first_task, int task_stride, unsigned char *smem, uint32_t tmem, int ptid, int bar_id, int aux_id,
    unsigned int *__restrict__ err)
{
    using SM = PrepSmem<DV>;
    using RC = Rec<DV>;
    float *Lsm = reinterpret_cast<float *>(smem + SM::kL);
    float *Tsm = reinterpret_cast<float *>(smem + SM::kT);
    float *Xsm = reinterpret_cast<float *>(smem + SM::kX);
    float *gate_s = reinterpret_cast<float *>(smem + SM::kGate);   // [2][PrepGate::kFloats]
    float *kf_s = reinterpret_cast<float *>(smem + SM::kMisc);        // [2] key-norm terms
    float *rgate_s = reinterpret_cast<float *>(smem + SM::kMisc + 16); // [4] record gate (ds)
    uint64_t *tma_bar = reinterpret_cast<uint64_t *>(smem + SM::kBar);
    uint64_t *mma_bar = tma_bar + 1;
    uint64_t *g_bar = tma_bar + 2;     // the Gram product
    volatile int *abort_s = reinterpret_cast<volatile int *>(smem + SM::kCtl + 4);

    const int tid = ptid, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3;                  // TMEM lane quarter of this warp
    const int half = warp >> 2;                    // column half handled by this warp
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t sbase = smem_u32(smem);
    const int ntasks = po.L * po.G * ndir * nbh;
    auto psync = [&]() { asm volatile("bar.sync %0, 256;" ::"r"(bar_id) : "memory"); };
    auto sync128 = [&]() { asm volatile("bar.sync %0, 128;" ::"r"(aux_id) : "memory"); };  // warps 0-3

    if (tid == 0) {
        mbar_init(tma_bar, 1);
        mbar_init(mma_bar, 1);
        mbar_init(g_bar, 1);
        fence_mbar_init();
        *abort_s = 0;
        prefetch_tensormap(tm_k);
        prefetch_tensormap(tm_q);
        prefetch_tensormap(tm_v);
    }
    psync();

    // the next task of this pipeline with a chunk to prepare (ntasks if none)
    auto next_valid = [&](int t) {
        int dir, c, bh;
        while (t < ntasks && !prep_task(po, t, nbh, ndir, nC, dir, c, bh)) t += task_stride;
        return t;
    };
    // Task descriptors, decoded once by thread 0 and read by every thread:
    // two slots (current, next) of {valid, dir, chunk, b*H+h}.
    int *desc = reinterpret_cast<int *>(smem + SM::kMisc + 32);
    auto put_desc = [&](int slot, int t) {
        int dir = 0, c = 0, bh = 0;
        const bool ok = t < ntasks && prep_task(po, t, nbh, ndir, nC, dir, c, bh);
        desc[slot * 4 + 0] = ok ? 1 : 0;
        desc[slot * 4 + 1] = dir;
        desc[slot * 4 + 2] = c;
        desc[slot * 4 + 3] = bh;
    };
    auto issue_tma = [&](int dir, int c, int bh) {
        (void)dir;
        const int b = bh / H, h = bh % H, t0 = c * 64;
        unsigned char *st = smem;
        mbar_arrive_expect_tx(tma_bar, SM::kStage);
        tma_load_4d(st, tm_k, tma_bar, 0, h, t0, b);
        tma_load_4d(st + 16384, tm_k, tma_bar, 64, h, t0, b);
        tma_load_4d(st + 8192, tm_q, tma_bar, 0, h, t0, b);
        tma_load_4d(st + 16384 + 8192, tm_q, tma_bar, 64, h, t0, b);
#pragma unroll
        for (int vb = 0; vb < DV / 64; ++vb)
            tma_load_4d(st + SM::kKQ + vb * 8192, tm_v, tma_bar, vb * 64, h, t0, b);
    };
    auto wait_all = [&](uint64_t *bar, uint32_t parity) {
        if (!mbar_wait(bar, parity, kWaitTries)) {
            *abort_s = 1;
            if (err) atomicAdd(err, 1u);
        }
    };
    // Gates of a task, by warp 4, one task ahead: lane l loads rows 2l and 2l+1
    // (processing order; raw values, so that the loads' latency is not waited
    // for here) ...
    auto load_gates = [&](int dir, int c, int bh, float2 &al, float2 &bt) {
        const int b = bh / H, h = bh % H;
        const int t0 = token_of_row(c, 2 * lane, dir), t1 = token_of_row(c, 2 * lane + 1, dir);
        const size_t o0 = ((size_t)b * T + t0) * H + h, o1 = ((size_t)b * T + t1) * H + h;
        al.x = t0 < T ? alpha[o0] : 1.f;
        bt.x = t0 < T ? beta[o0] : 0.f;
        al.y = t1 < T ? alpha[o1] : 1.f;
        bt.y = t1 < T ? beta[o1] : 0.f;
    };
    // ... and fills the task's gate buffer (PrepGate) from them.
    auto make_gates = [&](float *gb, float2 al, float2 bt, bool rv) {
        const float a0 = __logf(al.x), a1 = __logf(al.y);
        float s = a0 + a1;   // inclusive prefix sum over the lanes of the row-pair sums
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, s, d);
            if (lane >= d) s += y;
        }
        const float ex = s - (a0 + a1);
        const float g0 = ex + a0, g1 = ex + a0 + a1;                    // rows 2l, 2l+1
        const float gl = __shfl_sync(0xffffffffu, g1, 31);              // g_63
        const float gm = __shfl_up_sync(0xffffffffu, g1, 1);            // g_{2l-1}
        const float gb16 = __shfl_sync(0xffffffffu, g0, lane & ~7);     // g_16k of this row pair's block
        const int r0 = 2 * lane;
        gb[PrepGate::kG + r0] = g0;
        gb[PrepGate::kG + r0 + 1] = g1;
        gb[PrepGate::kBeta + r0] = bt.x;
        gb[PrepGate::kBeta + r0 + 1] = bt.y;
        gb[PrepGate::kDq + r0] = rv ? (lane > 0 ? __expf(gm) : 1.f) : __expf(g0);
        gb[PrepGate::kDq + r0 + 1] = rv ? __expf(g0) : __expf(g1);
        gb[PrepGate::kDkk + r0] = __expf(gl - g0);
        gb[PrepGate::kDkk + r0 + 1] = __expf(gl - g1);
        gb[PrepGate::kBg + r0] = bt.x * __expf(g0);
        gb[PrepGate::kBg + r0 + 1] = bt.y * __expf(g1);
        // Decay factors of the masks without an exponential per entry: for s in
        // the 16-token block k, e^{g_r - g_s} = e^{g_r - g_16k} e^{g_16k - g_s}.
        // On the entries the masks keep (16k <= s <= r) the first factor is at
        // most 1 and the second at most e^(decay over 16 tokens), so both are
        // finite whenever that decay stays below 80 (else: one exponential per
        // entry).
        gb[PrepGate::kFacs + r0] = __expf(gb16 - g0);
        gb[PrepGate::kFacs + r0 + 1] = __expf(gb16 - g1);
        const bool ok = (lane & 7) != 7 || gb16 - g1 < 80.f;            // g_16k - g_16k+15
        const bool fast = __all_sync(0xffffffffu, ok);
        if (lane == 0) {
            reinterpret_cast<int *>(gb)[PrepGate::kFast] = fast ? 1 : 0;
            gb[PrepGate::kDs] = __expf(gl);
        }
    };

    int t = 0;   // thread 0: index of the current task
    if (tid == 0) {
        t = next_valid(first_task);
        put_desc(0, t);
        if (desc[0]) issue_tma(desc[1], desc[2], desc[3]);
    }
    // the blocks of T above the block diagonal are zero for every task (nothing
    // writes them), so they are cleared once
    for (int e = tid; e < 64 * 64; e += kPrepThreads) {
        const int i = e >> 6, jj = e & 63;
        if ((jj >> 4) > (i >> 4)) Tsm[i * 65 + jj] = 0.f;
    }
    psync();   // (desc[0] is set)
    float2 al_n = make_float2(1.f, 1.f), bt_n = make_float2(0.f, 0.f);   // warp 4: the next task's raw gates
    if (warp == 4 && desc[0]) {
        load_gates(desc[1], desc[2], desc[3], al_n, bt_n);
        make_gates(gate_s, al_n, bt_n, desc[1] != 0);
    }
    uint32_t tma_phase = 0, mma_phase = 0, g_phase = 0;
    unsigned int *pending_flag = nullptr;   // thread 0: ready flag of the last record stored
    const uint32_t st_addr = sbase;
    int slot = 0;

    for (;;) {
        if (!desc[slot * 4]) break;
        const int dir = desc[slot * 4 + 1], c = desc[slot * 4 + 2], bh = desc[slot * 4 + 3];
        const int nxt = slot ^ 1;
        const bool rev = dir != 0;
        unsigned char *rec = recs + ((size_t)(dir * nbh + bh) * nC + c) * RC::kStride;
        int tn = 0;
        if (tid == 0) {
            tn = next_valid(t + task_stride);
            put_desc(nxt, tn);
        }

        const float *gb = gate_s + slot * PrepGate::kFloats;   // this task's gates (made one task ahead)
        const float *g_s = gb + PrepGate::kG, *beta_s = gb + PrepGate::kBeta, *dq_s = gb + PrepGate::kDq;
        const float *dkk_s = gb + PrepGate::kDkk, *bg_s = gb + PrepGate::kBg;
        wait_all(tma_bar, tma_phase);
        tma_phase ^= 1;
        psync();
        if (*abort_s) break;
        // ---- [K; Q] K^T (one accumulator, the two 64-column blocks of d_k in turn) ---
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t id = idesc(128, 64, 1, 0, 0);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t a = st_addr + (k >> 2) * 16384 + (k & 3) * 32;
                mma_bf16(tmem + kPrepColG, sdesc_sw128(a), sdesc_sw128(a), id, k > 0);
            }
            mma_commit(g_bar);
        }
        if (warp == 4 && desc[nxt * 4])   // the next task's gates, made during this task's level 2
            load_gates(desc[nxt * 4 + 1], desc[nxt * 4 + 2], desc[nxt * 4 + 3], al_n, bt_n);
        // the previous task's record stores must have read the staging areas; when
        // a chain runs alongside, wait for them to land and flag that record
        if (tid == 0) {
            if (ready && pending_flag) {
                bulk_wait_all();
                fence_proxy_async_global();
                __threadfence();
                st_release_gpu(pending_flag, 1u);
            } else {
                bulk_wait_read_all();
            }
            pending_flag = ready ? ready + (size_t)(dir * nbh + bh) * nC + c : nullptr;
        }
        wait_all(g_bar, g_phase);
        g_phase ^= 1;
        tc_fence_after();
        psync();
        // ---- L (fp32, to shared), P (fp16 image, staged for a bulk store) and the
        //      key-norm term of the state map's bound --------------------------------
        {
            float G[32];
            tmem_ld16(tmem + lane_base + kPrepColG + half * 32, G);
            tmem_ld16(tmem + lane_base + kPrepColG + half * 32 + 16, G + 16);
            tmem_wait_ld();
            // the mask code once per direction, so that the column order of every
            // entry (forward or mirrored) is a compile-time constant
            auto mask = [&](auto rv_c) {
                constexpr bool rev = decltype(rv_c)::value;   // (shadows the task flag)
                const int ln = quarter * 32 + lane;          // TMEM lane = Gram row
                const int fl = ln & 63;                      // forward row within the chunk
                const int r = rev ? 63 - fl : fl;            // processing row
                const int f0 = half * 32;                    // forward columns f0 .. f0+31
                const bool fast = reinterpret_cast<const int *>(gb)[PrepGate::kFast] != 0;   // task-uniform
                const float *facs = gb + PrepGate::kFacs;                                  // e^{g_16k - g_s}
                // the 16-token blocks of this thread's 32 columns: first 16, last 16
                const int kA = rev ? 3 - (f0 >> 4) : (f0 >> 4), kB = rev ? 2 - (f0 >> 4) : (f0 >> 4) + 1;
                if (ln < 64) {
                    const float br = beta_s[r], gr = g_s[r];
                    const float eA = br * __expf(gr - g_s[16 * kA]), eB = br * __expf(gr - g_s[16 * kB]);
                    // (the decay test is task-uniform: one loop or the other runs)
                    if (fast) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int s = rev ? 63 - (f0 + e) : f0 + e;
                            Lsm[r * 65 + s] = s < r ? (e < 16 ? eA : eB) * facs[s] * G[e] : 0.f;
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int s = rev ? 63 - (f0 + e) : f0 + e;
                            Lsm[r * 65 + s] = s < r ? br * __expf(gr - g_s[s]) * G[e] : 0.f;
                        }
                    }
                    if (half == (fl >> 5)) {   // warps 0 and 5 hold the diagonal of rows 0-31 / 32-63
                        float kk = 0.f;        // |k_r|^2: the Gram's diagonal, column fl - f0 = lane
#pragma unroll
                        for (int e = 0; e < 32; ++e) kk = e == lane ? G[e] : kk;
                        float term = __logf(fmaxf(1.f, fabsf(1.f - br * kk)));
#pragma unroll
                        for (int d = 16; d > 0; d >>= 1) term += __shfl_xor_sync(0xffffffffu, term, d);
                        if (lane == 0) kf_s[half] = term;
                    }
                } else {
                    const float gq = rev ? (r > 0 ? g_s[r - 1] : 0.f) : g_s[r];
                    const float eA = __expf(gq - g_s[16 * kA]), eB = __expf(gq - g_s[16 * kB]);
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        float v[8];
                        if (fast) {
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const int f = f0 + cc * 8 + e;
                                const int s = rev ? 63 - f : f;
                                const bool keep = rev ? (s < r) : (s <= r);
                                v[e] = keep ? (cc < 2 ? eA : eB) * facs[s] * G[cc * 8 + e] : 0.f;
                            }
                        } else {
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const int f = f0 + cc * 8 + e;
                                const int s = rev ? 63 - f : f;
                                const bool keep = rev ? (s < r) : (s <= r);
                                v[e] = keep ? __expf(gq - g_s[s]) * G[cc * 8 + e] : 0.f;
                            }
                        }
                        uint4 p;
                        p.x = pack_f16(v[0], v[1]); p.y = pack_f16(v[2], v[3]);
                        p.z = pack_f16(v[4], v[5]); p.w = pack_f16(v[6], v[7]);
                        *reinterpret_cast<uint4 *>(smem + SM::kT1 + sw128(fl, f0 + cc * 8, 0)) = p;
                    }
                    fence_async_shared();
                }
            };
            if (rev) mask(std::true_type{}); else mask(std::false_type{});
        }
        tc_fence_before();
        psync();
        if (tid == 0) {
            bulk_store(rec + RC::kP, smem + SM::kT1, 8192);
            bulk_commit_group();
            lb[(size_t)(dir * nbh + bh) * nC + c] = g_s[63] + kf_s[0] + kf_s[1];
            rgate_s[0] = gb[PrepGate::kDs];
            rgate_s[1] = rgate_s[2] = rgate_s[3] = 0.f;
        }
        // ---- T = (I + L)^{-1}, blocked 16 x 16 (processing order); meanwhile the
        //      other threads write the record's Q~ and K~ (fp16) from the tiles -------
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
            // 16-byte chunks of the record: K~ (2 blocks x 512), Q~ (2 blocks x 512)
            for (int i = tid - 64; i < 2048; i += kPrepThreads - 64) {
                const int blk = i >> 9, within = (i & 511) * 16, f = (i & 511) >> 3;
                const int rr = rev ? 63 - f : f;
                const bool is_k = blk < 2;
                const unsigned char *src = smem + (blk & 1) * 16384 + (is_k ? 0 : 8192) + within;
                const uint4 raw = *reinterpret_cast<const uint4 *>(src);
                const uint32_t in[4] = {raw.x, raw.y, raw.z, raw.w};
                const float scale = is_k ? dkk_s[rr] : dq_s[rr];
                uint32_t o16[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 x2 = unpack_bf16(in[e]);
                    o16[e] = pack_f16(scale * x2.x, scale * x2.y);
                }
                unsigned char *dst = rec + (is_k ? RC::kK + (blk & 1) * 8192 : RC::kQW + (blk & 1) * 16384) + within;
                *reinterpret_cast<uint4 *>(dst) = make_uint4(o16[0], o16[1], o16[2], o16[3]);
            }
        }
        psync();
        // off-diagonal blocks by recursive doubling (processing order):
        //   level 2, within each 32-block b: T_10 = -T_11 (L_10 T_00)   (16 x 16 blocks)
        //   level 3: T_[32:64, 0:32] = -T_[32:64, 32:64] (L_[32:64, 0:32] T_[0:32, 0:32])
        // T is stored lower-triangular with explicit zeros above the diagonal, so
        // the sums run over whole blocks (unrolled); each thread owns a 2 x 2 tile.
        if (tid < 128) {   // level 2, X = L_10 T_00 into Xsm[b][16][16]
            const int b2 = tid >> 6, ti = (tid >> 3) & 7, tj = tid & 7, base = 32 * b2;
            const int a = base + 16 + 2 * ti, bc = base + 2 * tj;
            float x00 = 0.f, x01 = 0.f, x10 = 0.f, x11 = 0.f;
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const float l0 = Lsm[a * 65 + base + m], l1 = Lsm[(a + 1) * 65 + base + m];
                const float t0 = Tsm[(base + m) * 65 + bc], t1 = Tsm[(base + m) * 65 + bc + 1];
                x00 = fmaf(l0, t0, x00); x01 = fmaf(l0, t1, x01);
                x10 = fmaf(l1, t0, x10); x11 = fmaf(l1, t1, x11);
            }
            float *xb = Xsm + b2 * 256 + (2 * ti) * 16 + 2 * tj;
            xb[0] = x00; xb[1] = x01; xb[16] = x10; xb[17] = x11;
            sync128();      // level 2 is warps 0-3 alone
        }
        if (tid < 128) {   // level 2, T_10 = -T_11 X
            const int b2 = tid >> 6, ti = (tid >> 3) & 7, tj = tid & 7, base = 32 * b2;
            const int a = base + 16 + 2 * ti, bc = base + 2 * tj;
            const float *xb = Xsm + b2 * 256 + 2 * tj;
            float y00 = 0.f, y01 = 0.f, y10 = 0.f, y11 = 0.f;
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const float t0 = Tsm[a * 65 + base + 16 + m], t1 = Tsm[(a + 1) * 65 + base + 16 + m];
                const float x0 = xb[m * 16], x1 = xb[m * 16 + 1];
                y00 = fmaf(t0, x0, y00); y01 = fmaf(t0, x1, y01);
                y10 = fmaf(t1, x0, y10); y11 = fmaf(t1, x1, y11);
            }
            Tsm[a * 65 + bc] = -y00; Tsm[a * 65 + bc + 1] = -y01;
            Tsm[(a + 1) * 65 + bc] = -y10; Tsm[(a + 1) * 65 + bc + 1] = -y11;
        } else if (warp == 4 && desc[nxt * 4]) {
            // the next task's gates, into the other buffer (the last task that
            // used it is done)
            make_gates(gate_s + nxt * PrepGate::kFloats, al_n, bt_n, desc[nxt * 4 + 1] != 0);
        }
        psync();
        // level 3, X = L_[32:64, 0:32] T_[0:32, 0:32] (32 x 32, fp32, stride 33) in the
        // T2 image area (free until the T images).  Thread tile rows 2*(tid & 15),
        // columns 2*(tid >> 4): a warp's columns are 4w .. 4w+3, so the rows of T
        // above 4w (zero) are skipped by whole 8-row steps.
        float *X3 = reinterpret_cast<float *>(smem + SM::kT2h);
        {
            const int ti = tid & 15, tj = tid >> 4;
            const int a = 32 + 2 * ti, bc = 2 * tj;
            const int m0 = (warp * 4) & ~7;
            float x00 = 0.f, x01 = 0.f, x10 = 0.f, x11 = 0.f;
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
                if (c8 * 8 + 8 <= m0) continue;    // warp-uniform
#pragma unroll
                for (int mm = 0; mm < 8; ++mm) {
                    const int m = c8 * 8 + mm;
                    const float l0 = Lsm[a * 65 + m], l1 = Lsm[(a + 1) * 65 + m];
                    const float t0 = Tsm[m * 65 + bc], t1 = Tsm[m * 65 + bc + 1];
                    x00 = fmaf(l0, t0, x00); x01 = fmaf(l0, t1, x01);
                    x10 = fmaf(l1, t0, x10); x11 = fmaf(l1, t1, x11);
                }
            }
            float *xb = X3 + (2 * ti) * 33 + bc;
            xb[0] = x00; xb[1] = x01; xb[33] = x10; xb[34] = x11;
        }
        psync();
        {   // level 3, T_[32:64, 0:32] = -T_[32:64, 32:64] X: tile rows 2*(tid >> 4) (a
            // warp's rows 4w .. 4w+3, so T's zero columns past them are skipped),
            // columns 2*(tid & 15)
            const int ti = tid >> 4, tj = tid & 15;
            const int a = 32 + 2 * ti, bc = 2 * tj;
            const int m1 = warp * 4 + 4;          // T_[a, 32+m] = 0 for m >= m1
            float y00 = 0.f, y01 = 0.f, y10 = 0.f, y11 = 0.f;
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
                if (c8 * 8 >= m1) continue;        // warp-uniform
#pragma unroll
                for (int mm = 0; mm < 8; ++mm) {
                    const int m = c8 * 8 + mm;
                    const float t0 = Tsm[a * 65 + 32 + m], t1 = Tsm[(a + 1) * 65 + 32 + m];
                    const float x0 = X3[m * 33 + bc], x1 = X3[m * 33 + bc + 1];
                    y00 = fmaf(t0, x0, y00); y01 = fmaf(t0, x1, y01);
                    y10 = fmaf(t1, x0, y10); y11 = fmaf(t1, x1, y11);
                }
            }
            Tsm[a * 65 + bc] = -y00; Tsm[a * 65 + bc + 1] = -y01;
            Tsm[(a + 1) * 65 + bc] = -y10; Tsm[(a + 1) * 65 + bc + 1] = -y11;
        }
        // the P store has read its staging area (the T images go there next)
        if (tid == 0) bulk_wait_read_all();
        psync();
        // ---- A operands T diag(beta e^g) (bf16) and T diag(beta) (bf16 hi/lo pair),
        //      in forward row/column order (mirrored for the reverse direction) -------
        for (int cell = tid; cell < 64 * 8; cell += kPrepThreads) {
            const int fr = cell & 63, fc0 = (cell >> 6) * 8;
            const int r = rev ? 63 - fr : fr;
            float a[8], bvals[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int s = rev ? 63 - (fc0 + e) : fc0 + e;
                const float tv = Tsm[r * 65 + s];
                a[e] = tv * bg_s[s];
                bvals[e] = tv * beta_s[s];
            }
            uint4 h1, h2, l2;
            h1.x = pack_bf16(a[0], a[1]); h1.y = pack_bf16(a[2], a[3]);
            h1.z = pack_bf16(a[4], a[5]); h1.w = pack_bf16(a[6], a[7]);
            split2(bvals[0], bvals[1], h2.x, l2.x); split2(bvals[2], bvals[3], h2.y, l2.y);
            split2(bvals[4], bvals[5], h2.z, l2.z); split2(bvals[6], bvals[7], h2.w, l2.w);
            const int off = kmaj64(fr, fc0);
            *reinterpret_cast<uint4 *>(smem + SM::kT1 + off) = h1;
            *reinterpret_cast<uint4 *>(smem + SM::kT2h + off) = h2;
            *reinterpret_cast<uint4 *>(smem + SM::kT2l + off) = l2;
        }
        fence_async_shared();
        psync();
        // ---- W = T1 K and U = T2 V on the tensor cores (K and V straight from the tiles)
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idw = idesc(64, 128, 1, 0, 1);
            constexpr uint32_t idu = idesc(64, DV, 1, 0, 1);
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                mma_bf16(tmem + kPrepColW, sdesc_noswz(sbase + SM::kT1 + 2 * s * 1024, 1024, 128),
                         sdesc_sw128_mn(st_addr + s * 2048, 16384), idw, s > 0);
                const uint64_t bv = sdesc_sw128_mn(st_addr + SM::kKQ + s * 2048, 8192);
                mma_bf16(tmem + kPrepColU, sdesc_noswz(sbase + SM::kT2h + 2 * s * 1024, 1024, 128), bv, idu, s > 0);
                mma_bf16(tmem + kPrepColU, sdesc_noswz(sbase + SM::kT2l + 2 * s * 1024, 1024, 128), bv, idu, 1);
            }
            mma_commit(mma_bar);
        }
        wait_all(mma_bar, mma_phase);
        mma_phase ^= 1;
        tc_fence_after();
        // the tiles are consumed: fetch the next task's while this one is written out
        if (tid == 0 && desc[nxt * 4]) issue_tma(desc[nxt * 4 + 1], desc[nxt * 4 + 2], desc[nxt * 4 + 3]);
        // ---- record: W image and U rows (fp16), staged in the areas the products
        //      are done with (T images, L/T) and written by bulk stores ---------------
        {
            const bool row_lane = lane < 16;
            const int f = quarter * 16 + lane;       // forward row (M=64 accumulator layout)
            {
                float w[64];                         // W columns half*64 .. +63
#pragma unroll
                for (int q = 0; q < 4; ++q) tmem_ld16(tmem + lane_base + kPrepColW + half * 64 + q * 16, w + 16 * q);
                tmem_wait_ld();
                if (row_lane) {
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        uint4 p;
                        p.x = pack_f16(w[8 * q], w[8 * q + 1]); p.y = pack_f16(w[8 * q + 2], w[8 * q + 3]);
                        p.z = pack_f16(w[8 * q + 4], w[8 * q + 5]); p.w = pack_f16(w[8 * q + 6], w[8 * q + 7]);
                        *reinterpret_cast<uint4 *>(smem + SM::kT1 + sw128(f, half * 64 + 8 * q, 8192)) = p;
                    }
                }
            }
#pragma unroll
            for (int q2 = 0; q2 < DV / 64; ++q2) {   // U columns half*DV/2 .. +DV/2-1, 32 at a time
                float u[32];
                const int col = half * (DV / 2) + q2 * 32;
                tmem_ld16(tmem + lane_base + kPrepColU + col, u);
                tmem_ld16(tmem + lane_base + kPrepColU + col + 16, u + 16);
                tmem_wait_ld();
                if (row_lane) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        uint4 p;
                        p.x = pack_f16(u[8 * i], u[8 * i + 1]); p.y = pack_f16(u[8 * i + 2], u[8 * i + 3]);
                        p.z = pack_f16(u[8 * i + 4], u[8 * i + 5]); p.w = pack_f16(u[8 * i + 6], u[8 * i + 7]);
                        *reinterpret_cast<uint4 *>(smem + SM::kL + u16_off<DV>(f, col + 8 * i)) = p;
                    }
                }
            }
            fence_async_shared();
            // With a chain alongside, the record's Q~ and K~ (plain stores of the
            // conversion threads) must be visible before its flag is set, at the
            // next task.  The fence sits here, long after those stores: right
            // after them it held up each thread's next shared-memory access until
            // they had drained (about 1.5 K cycles per task).  A standalone prep
            // needs no fence: the chain kernel starts after it.
            if (ready) __threadfence();
        }
        tc_fence_before();
        psync();
        if (tid == 0) {
            bulk_store(rec + RC::kQW + 8192, smem + SM::kT1, 8192);              // W, d_k 0-63
            bulk_store(rec + RC::kQW + 16384 + 8192, smem + SM::kT1 + 8192, 8192);   // W, d_k 64-127
            bulk_store(rec + RC::kU, smem + SM::kL, 64 * DV * 2);
            bulk_store(rec + RC::kGate, rgate_s, 16);
            bulk_commit_group();
        }
        if (tid == 0) t = tn;
        slot = nxt;
    }

    if (tid == 0) {
        bulk_wait_all();   // the record stores have landed
        if (pending_flag && !*abort_s) {
            fence_proxy_async_global();
            __threadfence();
            st_release_gpu(pending_flag, 1u);
        }
    }
    if (*abort_s) {
        mbar_wait(tma_bar, tma_phase, 64);
        mbar_wait(mma_bar, mma_phase, 64);
        mbar_wait(g_bar, g_phase, 64);
    }
    tc_fence_before();
    psync();
}

// Standalone prep: grid persistent (<= tasks), block 256, one pipeline per CTA.
template <int DV>
__global__ void __launch_bounds__(kPrepThreads, kPrepCtasPerSm)
prep_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
            const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ alpha,
            const float *__restrict__ beta, unsigned char *__restrict__ recs, float *__restrict__ lb, int T, int H,
            int nC, int nbh, int ndir, PrepOrder po, unsigned int *__restrict__ err)
{
    using SM = PrepSmem<DV>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint32_t *tmem_base_s = reinterpret_cast<uint32_t *>(smem + SM::kCtl);
    if ((threadIdx.x >> 5) == 0) {
        tmem_alloc(tmem_base_s, kPrepTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_s;
    prep_pipeline<DV>(&tm_k, &tm_q, &tm_v, alpha, beta, recs, lb, nullptr, T, H, nC, nbh, ndir, po, blockIdx.x,
                      gridDim.x, smem, tmem, threadIdx.x, 0, 1, err);
    __syncthreads();
    if ((threadIdx.x >> 5) == 0) tmem_dealloc(tmem, kPrepTmemCols);
}

}  // namespace tc2
}  // namespace gdn
