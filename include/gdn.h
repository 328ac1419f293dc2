/*
 * gdn.h -- C-ABI of the B200 (sm_100a) gated delta-net scan library, libgdn.so.
 *
 * The operator (per batch b and head h, t = 1..T, state S of d_k x d_v with
 * the key dimension as the row index):
 *
 *     S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *
 * This is gated delta-net linear attention with a matrix-valued recurrent
 * state per head.  The issue "[Research] Explore linear attention for the
 * streaming video models" (sections "We already ship a hybrid
 * linear-attention model" and "Open questions and risks") asks for its
 * causal, forward-only form with the state carried across calls.  The
 * bidirectional form follows "Video DeltaNet" (AI summary, "Methodology in
 * Plain English"): a forward and a backward state cover disjoint regions
 * and their readouts are added.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  Layout   q, k : [B, T, H, dk]   v : [B, T, H, dv]   element type `dt`
 *           o : [B, T, H, dv] element type `o_dt` (GDN_F32 or GDN_BF16)
 *           all contiguous, row-major
 *           alpha, beta : [B, T, H] fp32;  alpha in (0, 1], beta in [0, 1]
 *           state : [B, H, dk, dv] fp32, row index = key dimension
 *  Sizes    B >= 1, H >= 1, T >= 0; dk, dv in {64, 128}.
 *  Pointers All tensor pointers are DEVICE pointers, 16-byte aligned (alpha
 *           and beta: 4-byte aligned, so a token slice of them is valid).  The
 *           caller owns every buffer, including the workspace; the library
 *           never allocates, frees or synchronises.  Every call is
 *           asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *           stream) and performs no host synchronisation, so a call can be
 *           captured in a CUDA graph.
 *  Workspace `workspace` must hold at least gdn_workspace_size(...) bytes
 *           for the same arguments, 256-byte aligned; it may be NULL when
 *           that size is 0.  Its contents on entry do not matter.
 *  Errors   Arguments are checked on the host before any launch; a bad
 *           argument returns a negative gdn_status and launches nothing.
 *           A failed launch returns GDN_ERR_CUDA.  Kernels never trap.
 *  Inputs   alpha must be > 0 (the kernels use log alpha); values outside
 *           the stated ranges are not detected and give unspecified
 *           results, but never out-of-bounds accesses.
 *  Output   State and accumulation are fp32 whatever `dt` is.  With
 *           o_dt = GDN_F32 the output is the fp32 accumulator; with
 *           GDN_BF16 it is rounded once to bf16 (round to nearest even).
 *           Rounding to bf16 alone moves max|o|/rms(o) by up to 2^-8 times
 *           max|o|/rms(o), which on long sequences is several 1e-2, so the
 *           fp32 output is the one that carries the accuracy of the scan.
 *  Paths    fp32 inputs run on the CUDA cores in fp32 (max|o - exact| /
 *           rms(o) near 1e-6).  bf16 inputs (dk = 64 or 128; 64 runs as 128
 *           with zero columns) run on the tensor cores: the chunk algebra's
 *           products take fp16 operands (each computed operand rounded once;
 *           T diag(beta) as a bf16 hi/lo pair) with fp32 accumulation, about
 *           3e-3 .. 8e-3 of rms(o) on sequences of 16k to 262k tokens.  fp16
 *           holds magnitudes up to 65504: the state and the values must stay
 *           below that (they do for unit-norm keys and values of moderate
 *           size; the scan is linear in v and the state, so larger inputs can
 *           be scaled down and the output scaled back).  Long chunk walks are
 *           cut into segments that run in parallel (gdn_set_chain_segments),
 *           which drops contributions below 2^-30 of the state.
 */
#ifndef GDN_H
#define GDN_H

#include <stddef.h>

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_NULL = -1,        /* a required pointer is NULL */
    GDN_ERR_SHAPE = -2,       /* B < 1, H < 1, T < 0, or a size overflows */
    GDN_ERR_DTYPE = -3,       /* dt or o_dt is not a gdn_dtype */
    GDN_ERR_ALIGN = -4,       /* a pointer is not 16-byte (workspace: 256-byte) aligned */
    GDN_ERR_UNSUPPORTED = -5, /* dk or dv not in {64, 128} */
    GDN_ERR_WORKSPACE = -6,   /* ws_bytes < gdn_workspace_size(...) */
    GDN_ERR_CUDA = -7         /* a CUDA launch or copy failed */
} gdn_status;

typedef enum { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype;

/*
 * gdn_scan_causal -- causal scan over T tokens with optional state in/out.
 *   state_in   initial state S_0, or NULL for zero.
 *   state_out  receives S_T, or NULL (not written).  May equal state_in
 *              (in-place update); must not overlap it otherwise.
 *   o          receives o_1..o_T.
 * T = 0 writes state_out <- state_in (zero if state_in is NULL) and no o.
 */
GDN_API gdn_status gdn_scan_causal(const void *q, const void *k, const void *v,
                           const float *alpha, const float *beta,
                           const float *state_in, float *state_out, void *o,
                           int B, int T, int H, int dk, int dv, gdn_dtype dt, gdn_dtype o_dt,
                           void *workspace, size_t ws_bytes, void *stream);

/*
 * gdn_scan_bidir -- bidirectional scan:
 *     o_t = S_t^T q_t + R_{t+1}^T q_t,
 *     R_t = alpha_t (I - beta_t k_t k_t^T) R_{t+1} + beta_t k_t v_t^T,  R_{T+1} = 0,
 * i.e. the causal scan from zero plus the same recurrence run from T down
 * to 1, read before token t is written (token t is counted once, by the
 * causal part).  The two readouts are summed in fp32 (and, for a bf16
 * output, rounded once).
 */
GDN_API gdn_status gdn_scan_bidir(const void *q, const void *k, const void *v,
                          const float *alpha, const float *beta, void *o,
                          int B, int T, int H, int dk, int dv, gdn_dtype dt, gdn_dtype o_dt,
                          void *workspace, size_t ws_bytes, void *stream);

/*
 * gdn_scan_bidir_states -- gdn_scan_bidir with an initial and a final state
 * per direction (for instance a conditioning context folded into the states
 * a clip's two scans start from):
 *   causal half   S_0 = state_in (NULL: zero), S_t as in gdn_scan_causal;
 *                 state_out (NULL: not written) <- S_T
 *   reverse half  R_{T+1} = state_in_bwd (NULL: zero),
 *                 R_t = alpha_t (I - beta_t k_t k_t^T) R_{t+1} + beta_t k_t v_t^T;
 *                 state_out_bwd (NULL: not written) <- R_1
 *   o_t = S_t^T q_t + R_{t+1}^T q_t
 * Each state is [B, H, dk, dv] fp32, 16-byte aligned.  An output state may
 * be its own direction's input state (updated in place); no other two of the
 * four may overlap (GDN_ERR_SHAPE).  With T = 0 each output state receives
 * its input state.  Workspace: gdn_workspace_size(..., bidir = 1).  Sources:
 * as gdn_scan_bidir; the initial states of the two scans are the
 * bidirectional form's counterpart of the causal scan's state in and out.
 */
GDN_API gdn_status gdn_scan_bidir_states(const void *q, const void *k, const void *v,
                                         const float *alpha, const float *beta,
                                         const float *state_in, const float *state_in_bwd,
                                         float *state_out, float *state_out_bwd, void *o,
                                         int B, int T, int H, int dk, int dv, gdn_dtype dt,
                                         gdn_dtype o_dt, void *workspace, size_t ws_bytes,
                                         void *stream);

/*
 * gdn_step -- one streaming call: gdn_scan_causal with state_in == state_out
 * == state (required, updated in place).  A rollout is a sequence of
 * gdn_step calls on successive slices of the token stream; the result equals
 * one gdn_scan_causal over the concatenated tokens up to rounding.
 */
GDN_API gdn_status gdn_step(const void *q, const void *k, const void *v,
                    const float *alpha, const float *beta, float *state, void *o,
                    int B, int T, int H, int dk, int dv, gdn_dtype dt, gdn_dtype o_dt,
                    void *workspace, size_t ws_bytes, void *stream);

/*
 * gdn_step_noalloc -- gdn_step for callers that cannot allocate device
 * memory.  Some callers may not call cudaMalloc at all: code running inside
 * a host framework that owns every byte of device memory through its own
 * pool, or a real-time rollout loop where an allocation (which can
 * synchronise the device) would stall the pipeline.  This entry point takes
 * no workspace: its scratch is a file-scope __device__ array of
 * GDN_NOALLOC_SCRATCH_BYTES (64 MiB) inside libgdn.so, which every GPU that
 * loads the library holds until the process exits.  The caller still owns
 * q, k, v, alpha, beta, state and o.  (The pages have no counterpart of
 * this call; it exists for deployment only.)
 *   - It runs on the current device.  Its first call on a device looks up the
 *     array's device address (cudaGetSymbolAddress) with that device current;
 *     make that first call before any stream capture.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine.
 *   - Arguments whose gdn_workspace_size(..., bidir = 0) exceeds
 *     GDN_NOALLOC_SCRATCH_BYTES are rejected with GDN_ERR_WORKSPACE before
 *     any launch (for d_k = d_v = 128 and bf16 inputs, whose workspace is
 *     one 73,856-byte record, a flag and a bound per chunk-head, that is
 *     B*H*ceil(T/64) > 908).
 *   - All calls share the one array and it keeps the last call's contents;
 *     nothing in it needs to start at zero (every scratch byte a call reads
 *     was written earlier by the same call, in stream order).  Calls that
 *     overlap on the GPU (different streams, or several host threads) race
 *     on the array and give wrong results: serialise them.
 * Semantics, layout and status codes are otherwise those of gdn_step.
 */
#define GDN_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
GDN_API gdn_status gdn_step_noalloc(const void *q, const void *k, const void *v,
                                    const float *alpha, const float *beta, float *state, void *o,
                                    int B, int T, int H, int dk, int dv, gdn_dtype dt,
                                    gdn_dtype o_dt, void *stream);

/*
 * gdn_workspace_size -- bytes of device workspace a call with these
 * arguments needs (bidir != 0: gdn_scan_bidir; else gdn_scan_causal /
 * gdn_step).  Returns 0 for arguments that the call would reject.
 */
GDN_API size_t gdn_workspace_size(int B, int T, int H, int dk, int dv, gdn_dtype dt,
                                  gdn_dtype o_dt, int bidir);

/*
 * gdn_set_short_call_tokens -- which causal calls (gdn_scan_causal, gdn_step,
 * gdn_step_noalloc) walk their tokens one by one on the CUDA cores, state
 * slice in registers, in fp32 (the recurrence written out per token:
 * p = S^T k, S <- alpha S + k (beta (v - alpha p))^T, o = S^T q), instead of
 * the chunked path.  A short call's fixed cost is then a few microseconds
 * instead of a chunk prep plus a chain step.  max_t < 0: automatic (the
 * default): calls of T <= 64 tokens whose T times the number of waves of
 * their B*H*dv/32 CTAs over the SMs is at most 48 (the measured break-even);
 * 0: never; 1..64 (larger values clamp to 64): every call of T <= max_t.
 * Bidirectional calls always take the chunked path.  Returns the previous
 * setting (-1 for automatic).  The setting is process-wide and read at each
 * call; it changes which kernels run, not the workspace a call needs
 * (gdn_workspace_size does not depend on it).  Both paths meet the same
 * tolerances.
 */
GDN_API int gdn_set_short_call_tokens(int max_t);

/*
 * gdn_set_chain_segments -- how many segments the tensor-core path cuts each
 * (b, h, direction) chunk walk into (sequence parallelism; bf16 inputs).
 * g < 1: automatic (the default): enough segments to occupy the SMs with one
 * wave of chain CTAs, at least 4 chunks each; g >= 1: g segments (at most one
 * per chunk).
 * A segment other than the first starts from a zero state some chunks before
 * its first output, at the first chunk boundary where the 2-norm bound of the
 * skipped state maps, the product over the skipped tokens of
 * alpha_t max(1, |1 - beta_t |k_t|^2|), falls to 2^-30 (or from the true
 * initial state if the walk back reaches the start).  The state dropped there
 * reaches the segment's first output scaled by at most 2^-30, so results
 * agree with one segment up to rounding; only the speed depends on how fast
 * the gates forget.  Returns the previous setting (-1 for automatic).
 * Process-wide, read at each call; the workspace does not depend on it.
 */
GDN_API int gdn_set_chain_segments(int g);

/*
 * gdn_vda_scan -- the frame-wise delta operator: the sequence is F frames of
 * U consecutive tokens (T = F * U) and the state is written once per frame,
 * by all of the frame's tokens at once:
 *   A_f = K_f^T diag(beta) K_f,   B_f = K_f^T diag(beta) V_f
 *   S_f = (I + A_f)^{-1} (alpha_f S_{f-1} + B_f),   o_u = S_f^T q_u  (u in frame f)
 * S_f is the state closest to the decayed memory alpha_f S_{f-1} that fits
 * every key-value pair of the frame in the least-squares sense (weights
 * beta).  bidir != 0 adds the reverse scan R_f = (I + A_f)^{-1} (alpha_f
 * R_{f+1} + B_f) read strictly: o_u += R_{f+1}^T q_u (the frames after f).
 * Source: AI summary of "Video DeltaNet: A Video-Native Hybrid Attention for
 * Livestream Video Generation", "Key Contributions" 2 (the closed form, for
 * a state mapping keys to values, i.e. the transpose of this layout) and
 * "Methodology in Plain English" (the objective in words); A_f, B_f and the
 * decayed previous state are this library's reading of that objective.
 *   q, k [B, T, H, dk]; v, o [B, T, H, dv] (dtypes dt, o_dt); alpha_frame
 *   [B, F, H] fp32 in (0, 1]; beta [B, T, H] fp32 >= 0; states [B, H, dk, dv]
 *   fp32: state_in / state_out the causal S_0 / S_F, state_in_bwd /
 *   state_out_bwd the reverse R_{F+1} / R_1 (used only when bidir; NULL: zero /
 *   not written), with the overlap rules of gdn_scan_bidir_states.
 *   Workspace: gdn_vda_workspace_size bytes, 256-byte aligned.  F = 0 passes
 *   the states through.  Two paths: fp32 inputs (or dk = 64) run every step in
 *   fp32 on the CUDA cores; bf16 inputs with dk = 128 take the frame Gram
 *   [A_f | B_f] and the readout on the tensor cores (bf16 keys and queries
 *   exact, the beta-scaled keys and values and the states as bf16 hi/lo
 *   pairs, fp32 accumulation).  Either way (I + A_f)^{-1} comes from an fp32
 *   Cholesky factorisation per frame and head, and the state recurrence is
 *   fp32 on the CUDA cores.
 */
GDN_API gdn_status gdn_vda_scan(const void *q, const void *k, const void *v, const float *alpha_frame,
                                const float *beta, const float *state_in, const float *state_in_bwd,
                                float *state_out, float *state_out_bwd, void *o, int B, int F, int U,
                                int H, int dk, int dv, int bidir, gdn_dtype dt, gdn_dtype o_dt,
                                void *workspace, size_t ws_bytes, void *stream);
/* gdn_vda_workspace_size -- bytes of workspace gdn_vda_scan needs (0 for
 * arguments it would reject, or F = 0). */
GDN_API size_t gdn_vda_workspace_size(int B, int F, int U, int H, int dk, int dv, int bidir);

/*
 * gdn_readout_gate -- readout epilogue of the linear branch, one pass over o:
 *   y[b,t,h,:] = o[b,t,h,:] / sqrt(mean_j o[b,t,h,j]^2 + eps) * gamma * sigmoid(z[b,t,h,:])
 * i.e. an RMS norm over the head's dv channels of each token, a per-channel
 * gain gamma ([dv] fp32; NULL = ones) and the content-dependent sigmoid gate
 * z.  Source: AI summary of "Video DeltaNet: A Video-Native Hybrid Attention
 * for Livestream Video Generation", "Key Contributions" 1 (the linear branch
 * has its own sigmoid gate and an RMS-normalised readout; the axis and the
 * order, norm then gate, are this library's reading).
 *   o, z, y: [B, T, H, dv] contiguous, dtypes o_dt, z_dt, y_dt (GDN_F32 or
 *   GDN_BF16), 16-byte aligned; dv in {64, 128}; eps >= 0 and finite.  y may
 *   be o or z itself when its dtype matches (in place); any other overlap is
 *   GDN_ERR_SHAPE.  T = 0 is a no-op.  Asynchronous on `stream`; no
 *   workspace.  All arithmetic in fp32.
 */
GDN_API gdn_status gdn_readout_gate(const void *o, gdn_dtype o_dt, const void *z, gdn_dtype z_dt,
                                    const float *gamma, float eps, void *y, gdn_dtype y_dt,
                                    int B, int T, int H, int dv, void *stream);

/* gdn_status_string -- static, NUL-terminated description of a status. */
GDN_API const char *gdn_status_string(gdn_status s);

/* gdn_version -- static version string of the library build. */
GDN_API const char *gdn_version(void);

/*
 * Introspection (measurement support; not part of the scan itself).
 *
 * gdn_launch_count -- number of CUDA kernels this library has launched in
 *   this process so far (all devices, all threads).
 * gdn_set_kernel_timing -- on != 0: from now on, bracket every kernel launch
 *   with a pair of CUDA events recorded on the launch stream; 0: stop.  Use
 *   only on eager (not graph-captured) calls.  Creating the events is the
 *   only host-side work it adds; it never synchronises.
 * gdn_read_kernel_timing -- synchronise on the recorded events, then report
 *   per kernel name (at most `max` names): total device milliseconds and the
 *   number of launches since the previous read, and forget them.  `names`
 *   receives `max` NUL-terminated slots of `name_len` bytes.  Returns the
 *   number of kernel names written, or a negative gdn_status.
 */
GDN_API unsigned long long gdn_launch_count(void);
/* gdn_device_timeouts -- number of bounded device-side waits (on TMA or
 * tensor-core completion) that gave up on the current device since the
 * library was loaded; non-zero means a kernel stopped early and its results
 * are invalid.  Synchronous (reads a device word).  Returns a gdn_status. */
GDN_API int gdn_device_timeouts(unsigned int *count);
GDN_API void gdn_set_kernel_timing(int on);
GDN_API int gdn_read_kernel_timing(char *names, int name_len, double *total_ms, int *launches,
                                   int max);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */
