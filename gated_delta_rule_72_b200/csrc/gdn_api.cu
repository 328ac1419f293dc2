// gdn_api.cu -- the C-ABI entry points of libgdn.so: argument checks,
// workspace planning and kernel dispatch.  See include/gdn.h.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <type_traits>

#include "../../include/gdn.h"
#include "common.cuh"
#include "launch_stats.cuh"
#include "simt_kernels.cuh"
#include "tc_chain.cuh"
#include "tc_fused.cuh"
#include "tc_prep.cuh"
#include "readout.cuh"
#include "token_step.cuh"
#include "vda.cuh"
#include "vda_tc.cuh"

// Count of bounded device-side waits that gave up (see gdn_device_timeouts).
static __device__ unsigned int g_wait_timeouts;

namespace {

using gdn::kChunk;

struct Args {
    const void *q, *k, *v;
    const float *alpha, *beta;
    const float *state_in;
    float *state_out;
    void *o;
    int B, T, H, dk, dv;
    gdn_dtype dt, o_dt;
    void *ws;
    size_t ws_bytes;
    cudaStream_t stream;
    // bidirectional calls: the reverse direction's initial R_{T+1} and final R_1
    const float *state_in_bwd = nullptr;
    float *state_out_bwd = nullptr;
};

inline bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------------------
// Workspace plan of the CUDA-core path: one fp32 record per chunk, head and
// direction, then (bidirectional only) an fp32 partial output [B,T,H,dv].
// ---------------------------------------------------------------------------
size_t simt_record_floats(int dk, int dv) {
    return (size_t)3 * kChunk * dk + (size_t)kChunk * dv + (size_t)kChunk * kChunk + 4;
}

size_t simt_workspace(int B, int T, int H, int dk, int dv, int bidir) {
    const size_t nC = (size_t)(T + kChunk - 1) / kChunk;
    const size_t ndir = bidir ? 2 : 1;
    size_t bytes = round_up(ndir * B * H * nC * simt_record_floats(dk, dv) * sizeof(float), 256);
    if (bidir) bytes += round_up((size_t)B * T * H * dv * sizeof(float), 256);
    return bytes;
}

gdn_status check_common(const Args &a, bool need_inputs) {
    if (a.dt != GDN_F32 && a.dt != GDN_BF16) return GDN_ERR_DTYPE;
    if (a.o_dt != GDN_F32 && a.o_dt != GDN_BF16) return GDN_ERR_DTYPE;
    if (a.B < 1 || a.H < 1 || a.T < 0) return GDN_ERR_SHAPE;
    if (!((a.dk == 64 || a.dk == 128) && (a.dv == 64 || a.dv == 128))) return GDN_ERR_UNSUPPORTED;
    // index arithmetic is 64-bit, but the chunk count and grid dims are int
    if ((long long)a.B * a.H > 65535LL || a.T > (1 << 30)) return GDN_ERR_SHAPE;
    if (need_inputs) {
        if (!a.q || !a.k || !a.v || !a.alpha || !a.beta || !a.o) return GDN_ERR_NULL;
        const void *ps[] = {a.q, a.k, a.v, a.o};
        for (const void *p : ps)
            if (!aligned(p, 16)) return GDN_ERR_ALIGN;
        // the gates are read one float at a time
        if (!aligned(a.alpha, 4) || !aligned(a.beta, 4)) return GDN_ERR_ALIGN;
    }
    const void *st[4] = {a.state_in, a.state_out, a.state_in_bwd, a.state_out_bwd};
    for (const void *p : st)
        if (p && !aligned(p, 16)) return GDN_ERR_ALIGN;
    // An output state may be its own direction's input state exactly; no other
    // two of the four state buffers may overlap.
    const size_t n = (size_t)a.B * a.H * a.dk * a.dv * sizeof(float);
    auto overlap = [n](const void *x, const void *y) {
        const char *p = static_cast<const char *>(x), *q = static_cast<const char *>(y);
        return p && q && p < q + n && q < p + n;
    };
    for (int i = 0; i < 4; ++i)
        for (int j = i + 1; j < 4; ++j) {
            const bool own = (i == 0 && j == 1) || (i == 2 && j == 3);
            if (overlap(st[i], st[j]) && !(own && st[i] == st[j])) return GDN_ERR_SHAPE;
        }
    return GDN_OK;
}

gdn_status check_ws(const Args &a, size_t need) {
    if (need == 0) return GDN_OK;
    if (!a.ws) return GDN_ERR_NULL;
    if (!aligned(a.ws, 256)) return GDN_ERR_ALIGN;
    if (a.ws_bytes < need) return GDN_ERR_WORKSPACE;
    return GDN_OK;
}

gdn_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// T = 0: state_out <- state_in (or zero).
gdn_status copy_state(const Args &a, const float *in, float *out) {
    if (!out || out == in) return GDN_OK;
    const size_t n = (size_t)a.B * a.H * a.dk * a.dv * sizeof(float);
    cudaError_t e = in ? cudaMemcpyAsync(out, in, n, cudaMemcpyDeviceToDevice, a.stream)
                       : cudaMemsetAsync(out, 0, n, a.stream);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// T = 0: every final state is its initial state (zero if none).
gdn_status empty_scan(const Args &a, int bidir) {
    const gdn_status s = copy_state(a, a.state_in, a.state_out);
    if (s != GDN_OK || !bidir) return s;
    return copy_state(a, a.state_in_bwd, a.state_out_bwd);
}

// ---------------------------------------------------------------------------
// CUDA-core path
// ---------------------------------------------------------------------------
template <int DK, int DV, typename Tin, typename Tout>
gdn_status run_simt(const Args &a, int bidir) {
    using namespace gdn::simt;
    constexpr int NS = 32;
    const int nC = (a.T + kChunk - 1) / kChunk;
    const int nbh = a.B * a.H;
    float *rec = static_cast<float *>(a.ws);
    const size_t rec_bytes = round_up((size_t)(bidir ? 2 : 1) * nbh * nC *
                                      Record<DK, DV>::kFloats * sizeof(float), 256);
    float *part = bidir ? reinterpret_cast<float *>(static_cast<char *>(a.ws) + rec_bytes) : nullptr;

    auto prep = prep_kernel<DK, DV, Tin>;
    const size_t prep_smem = PrepSmem<DK, DV>::kBytes;
    if (cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)prep_smem) != cudaSuccess)
        return GDN_ERR_CUDA;
    {
        gdn::LaunchScope ls("simt_prep", a.stream);
        prep<<<dim3(nC, nbh, bidir ? 2 : 1), 256, prep_smem, a.stream>>>(
            static_cast<const Tin *>(a.q), static_cast<const Tin *>(a.k),
            static_cast<const Tin *>(a.v), a.alpha, a.beta, rec, a.T, a.H, nC, 0);
    }
    if (launch_status() != GDN_OK) return GDN_ERR_CUDA;

    auto chain = chain_kernel<DK, DV, NS, Tout>;
    const size_t chain_smem = ChainSmem<DK, NS>::kBytes;
    if (cudaFuncSetAttribute(chain, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)chain_smem) != cudaSuccess)
        return GDN_ERR_CUDA;
    const dim3 grid(DV / NS, nbh, 1);
    Tout *o = static_cast<Tout *>(a.o);
    if (!bidir) {
        gdn::LaunchScope ls("simt_chain", a.stream);
        chain<<<grid, 256, chain_smem, a.stream>>>(rec, a.state_in, a.state_out, o, nullptr,
                                                   a.T, a.H, nC, 0, kOutStore, nbh);
        return launch_status();
    }
    {
        gdn::LaunchScope ls("simt_chain", a.stream);
        chain<<<grid, 256, chain_smem, a.stream>>>(rec, a.state_in, a.state_out, o, part, a.T, a.H, nC,
                                                   0, kOutPartial, nbh);
    }
    if (launch_status() != GDN_OK) return GDN_ERR_CUDA;
    gdn::LaunchScope ls("simt_chain", a.stream);
    chain<<<grid, 256, chain_smem, a.stream>>>(rec, a.state_in_bwd, a.state_out_bwd, o, part, a.T, a.H, nC, 1,
                                               kOutAddPartial, nbh);
    return launch_status();
}

template <typename Tin, typename Tout>
gdn_status dispatch_dims(const Args &a, int bidir) {
    if (a.dk == 128 && a.dv == 128) return run_simt<128, 128, Tin, Tout>(a, bidir);
    if (a.dk == 128 && a.dv == 64) return run_simt<128, 64, Tin, Tout>(a, bidir);
    if (a.dk == 64 && a.dv == 128) return run_simt<64, 128, Tin, Tout>(a, bidir);
    return run_simt<64, 64, Tin, Tout>(a, bidir);
}

template <typename Tin>
gdn_status dispatch_out(const Args &a, int bidir) {
    return a.o_dt == GDN_F32 ? dispatch_dims<Tin, float>(a, bidir)
                             : dispatch_dims<Tin, __nv_bfloat16>(a, bidir);
}

// The tensor-core path takes bf16 inputs (d_k = 64 runs as 128 with zero
// columns: the key and query tiles are loaded past their width, which reads
// zeros); fp32 inputs run on the CUDA-core (fp32) path.
bool use_tc(gdn_dtype dt, int dk, int dv) {
    return dt == GDN_BF16 && (dk == 128 || dk == 64) && (dv == 128 || dv == 64);
}

size_t tc_record_bytes(int dv) {
    return dv == 128 ? gdn::tc2::Rec<128>::kStride : gdn::tc2::Rec<64>::kStride;
}

// Tensor-core path workspace: one record per chunk, head and direction, one
// ready flag and one log bound per record; then, bidirectional with a bf16
// o only, the fp32 sum of the two directions (an fp32 o is its own sum).

size_t plan_workspace(int B, int T, int H, int dk, int dv, gdn_dtype dt, gdn_dtype o_dt, int bidir) {
    if (T == 0) return 0;
    if (use_tc(dt, dk, dv)) {
        const size_t nC = (size_t)(T + kChunk - 1) / kChunk;
        const size_t nrec = (bidir ? 2 : 1) * (size_t)B * H * nC;
        size_t bytes = round_up(nrec * tc_record_bytes(dv), 256);
        bytes += round_up(nrec * sizeof(unsigned int), 256);   // ready flags
        bytes += round_up(nrec * sizeof(float), 256);          // log bounds of the chunk maps
        if (bidir && o_dt == GDN_BF16) bytes += round_up((size_t)B * T * H * dv * sizeof(float), 256);
        return bytes;
    }
    return simt_workspace(B, T, H, dk, dv, bidir);
}

// ---------------------------------------------------------------------------
// Tensor-core path
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Tile map over a [B, T, H, d] tensor of bf16 (esize 2) or fp32 (esize 4):
// boxes of (box_d columns, 1 head, 64 tokens, 1 batch); loads past T read as
// zero and stores past T are dropped.  swz: 0 none, 64 or 128 (bytes).
bool encode_map(CUtensorMap *m, const void *base, int B, int T, int H, int d, int box_d, int swz,
                int esize = 2) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t es = (cuuint64_t)esize;
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)d * es, (cuuint64_t)H * d * es, (cuuint64_t)T * H * d * es};
    const cuuint32_t box[4] = {(cuuint32_t)box_d, 1, 64, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUtensorMapSwizzle sw = swz == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : swz == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                              : CU_TENSOR_MAP_SWIZZLE_NONE;
    return enc(m, esize == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
               const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

std::mutex g_err_mu;
unsigned int *g_err_ptr[64] = {};

unsigned int *timeout_counter() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> g(g_err_mu);
    if (!g_err_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_wait_timeouts) != cudaSuccess) return nullptr;
        g_err_ptr[dev] = static_cast<unsigned int *>(p);
    }
    return g_err_ptr[dev];
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return 148;
    return n;
}

// Segmentation of the chunk walks and the split of the SMs.
//   G segments of L chunks per chain; fused: n_chain chain CTAs beside
//   n_prep CTAs of two prep pipelines (one cooperative launch); else prep on
//   every SM, then the chains.
struct TcPlan {
    bool fused;
    int G, L, n_chain, n_prep;
    gdn::tc2::PrepOrder po;
};

// < 0: automatic; else the segments per chain (clamped to the chunk count)
std::atomic<int> g_chain_segments{-1};

// Fewest prep CTAs (two pipelines each) worth a fused launch: below this the
// prep would lag the chains and two launches do better.
constexpr int kMinFusedPrepCtas = 32;
// Fewest chunks per segment (a segment also walks back a few chunks first).
constexpr int kMinSegChunks = 4;
// Tail positions of every segment the prep produces first (the next
// segment's walk back reads them before anything else).
constexpr int kTailFirst = 12;

// Automatic plan (from B200 timings of the d = 128 workloads): when the walks
// are long enough to cut, prep on every SM and then one wave of chain CTAs
// (G = SMs / chains, at least 4 chunks per segment: a 32k-token causal scan
// of 12 heads 0.37 ms against 0.49 ms fused with 4 segments; bidirectional
// 75k tokens of 20 heads 2.8 ms against 4.2 ms fused; 168 streaming calls of
// 1,560 tokens and 16 heads 11.8 ms with 5 segments of 5 chunks, 13.3 ms with
// 4 of 7, 12.6 ms with 9 of 3, 16.4 ms fused with one); when they are not
// (short calls, or chains that fill the GPU),
// one fused launch where the SMs allow it, whose prep runs beside the chains
// so that the first chunk's record is ready early.  A forced segment count
// takes the fused launch where the SMs allow it.
TcPlan plan_tc(int chains, int nC, bool coop) {
    const int sms = sm_count();
    TcPlan p{};
    const int forced = g_chain_segments.load(std::memory_order_relaxed);
    const int gmax = nC / kMinSegChunks > 1 ? nC / kMinSegChunks : 1;
    int G;
    if (forced > 0) {
        G = forced < nC ? forced : nC;
        p.fused = coop && (long long)chains * G + kMinFusedPrepCtas <= sms;
    } else {
        G = sms / chains;
        if (G > gmax) G = gmax;
        if (G < 1) G = 1;
        p.fused = G == 1 && coop && chains + kMinFusedPrepCtas <= sms;
    }
    p.L = (nC + G - 1) / G;
    p.G = (nC + p.L - 1) / p.L;
    p.n_chain = chains * p.G;
    p.n_prep = p.fused ? sms - p.n_chain : 0;
    p.po.G = p.G;
    p.po.L = p.L;
    p.po.tail = p.G > 1 ? (p.L < kTailFirst ? p.L : kTailFirst) : 0;
    return p;
}

// Output tile map: fp32 boxes of 32 columns, bf16 boxes of 64 (128-byte rows,
// 128B swizzle, as the chain stages them).
bool encode_out_map(CUtensorMap *m, const void *target, const Args &a, int dv, bool f32) {
    return encode_map(m, target, a.B, a.T, a.H, dv, f32 ? 32 : 64, 128, f32 ? 4 : 2);
}

template <int DV>
gdn_status launch_prep(const Args &a, const CUtensorMap &mk, const CUtensorMap &mq, const CUtensorMap &mv,
                       unsigned char *recs, float *lb, int nC, int ndir, const gdn::tc2::PrepOrder &po,
                       unsigned int *err) {
    using SM = gdn::tc2::PrepSmem<DV>;
    auto kern = gdn::tc2::prep_kernel<DV>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kAlloc) != cudaSuccess)
        return GDN_ERR_CUDA;
    const int nbh = a.B * a.H;
    const long long ntasks = (long long)ndir * nC * nbh;
    const long long slots = (long long)sm_count() * gdn::tc2::kPrepCtasPerSm;
    const int grid = (int)(ntasks < slots ? ntasks : slots);
    gdn::LaunchScope ls("tc_prep", a.stream);
    kern<<<grid, gdn::tc2::kPrepThreads, SM::kAlloc, a.stream>>>(mk, mq, mv, a.alpha, a.beta, recs, lb, a.T, a.H, nC,
                                                                 nbh, ndir, po, err);
    return launch_status();
}

// o (bf16) <- sum (fp32), n a multiple of 4 elements.
__global__ void cast_bf16_kernel(const float4 *__restrict__ sum, uint2 *__restrict__ o, size_t n4) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
        const float4 v = sum[i];
        uint2 u;
        u.x = gdn::tc2::pack_bf16(v.x, v.y);
        u.y = gdn::tc2::pack_bf16(v.z, v.w);
        o[i] = u;
    }
}

template <int DV, typename Tout>
gdn_status launch_chain(const Args &a, const CUtensorMap &mo, const unsigned char *recs, int nC, int ndir,
                        const gdn::tc2::ChainStates &states, const gdn::tc2::ChainOut<Tout> &out,
                        const gdn::tc2::ChainSeg &seg, unsigned int *err) {
    using SM = gdn::tc2::ChainSmem<DV>;
    auto kern = gdn::tc2::chain_kernel<DV, Tout>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kAlloc) != cudaSuccess)
        return GDN_ERR_CUDA;
    gdn::LaunchScope ls(ndir == 2 ? "tc_chain_bidir" : "tc_chain", a.stream);
    kern<<<dim3(seg.G, a.B * a.H, ndir), gdn::tc2::kChainThreads, SM::kAlloc, a.stream>>>(mo, recs, states, out,
                                                                                          seg, a.H, nC, err);
    return launch_status();
}

// Prep and chain in one cooperative launch (tc_fused.cuh).  Returns
// GDN_ERR_UNSUPPORTED (nothing launched) when the launch cannot be cooperative.
template <int DV, typename Tout>
gdn_status launch_fused(const Args &a, const CUtensorMap &mk, const CUtensorMap &mq, const CUtensorMap &mv,
                        const CUtensorMap &mo, unsigned char *recs, float *lb, unsigned int *ready, int nC, int ndir,
                        const TcPlan &p, const gdn::tc2::ChainStates &states, const gdn::tc2::ChainOut<Tout> &out,
                        const gdn::tc2::ChainSeg &seg, unsigned int *err) {
    auto kern = gdn::tc2::fused_kernel<DV, Tout>;
    constexpr int smem = gdn::tc2::fused_smem_alloc<DV>();
    constexpr int threads = gdn::tc2::kChainThreads;
    static_assert(smem <= 227 * 1024, "fused launch shared memory");
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return GDN_ERR_CUDA;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem) != cudaSuccess ||
        per_sm < 1 || p.n_chain + p.n_prep > per_sm * sm_count())
        return GDN_ERR_UNSUPPORTED;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.n_chain + p.n_prep);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    gdn::LaunchScope ls("tc_fused", a.stream);
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, mk, mq, mv, mo, a.alpha, a.beta, recs, lb, ready, states,
                                             out, seg, p.po, a.T, a.H, nC, a.B * a.H, ndir, p.n_chain, err);
    if (e == cudaErrorCooperativeLaunchTooLarge || e == cudaErrorNotSupported) {
        (void)cudaGetLastError();
        return GDN_ERR_UNSUPPORTED;
    }
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

bool cooperative_supported() {
    int dev = 0, v = 0;
    return cudaGetDevice(&dev) == cudaSuccess &&
           cudaDeviceGetAttribute(&v, cudaDevAttrCooperativeLaunch, dev) == cudaSuccess && v != 0;
}

template <int DV, typename Tout>
gdn_status run_tc(const Args &a, int bidir) {
    CUtensorMap mk, mq, mv;
    if (!encode_map(&mk, a.k, a.B, a.T, a.H, a.dk, 64, 128) ||
        !encode_map(&mq, a.q, a.B, a.T, a.H, a.dk, 64, 128) ||
        !encode_map(&mv, a.v, a.B, a.T, a.H, DV, 64, 128))
        return GDN_ERR_CUDA;
    unsigned int *err = timeout_counter();
    if (!err) return GDN_ERR_CUDA;
    const int nC = (a.T + kChunk - 1) / kChunk;
    const int ndir = bidir ? 2 : 1;
    const size_t nrec = (size_t)ndir * a.B * a.H * nC;
    unsigned char *recs = static_cast<unsigned char *>(a.ws);
    unsigned char *p = recs + round_up(nrec * tc_record_bytes(DV), 256);
    unsigned int *ready = reinterpret_cast<unsigned int *>(p);
    p += round_up(nrec * sizeof(unsigned int), 256);
    float *lb = reinterpret_cast<float *>(p);
    p += round_up(nrec * sizeof(float), 256);
    gdn::tc2::ChainOut<Tout> out{};
    constexpr bool f32_out = std::is_same<Tout, float>::value;
    void *target = a.o;
    const size_t n = (size_t)a.B * a.T * a.H * DV;
    if (bidir) {
        // both directions in one launch, adding up in fp32 (in o itself for an
        // fp32 o, else in a buffer that is then rounded into o), from zero
        if (!f32_out) {
            target = p;
            p += round_up(n * sizeof(float), 256);
        }
        out.mode = gdn::tc2::kOutPair;
        if (cudaMemsetAsync(target, 0, n * sizeof(float), a.stream) != cudaSuccess) return GDN_ERR_CUDA;
    } else {
        out.mode = gdn::tc2::kOutStore;
    }
    CUtensorMap mo;
    if (!encode_out_map(&mo, target, a, DV, f32_out || bidir)) return GDN_ERR_CUDA;
    gdn::tc2::ChainStates states{};
    states.dk = a.dk;
    states.in[0] = a.state_in;
    states.out[0] = a.state_out;
    if (bidir) {
        states.in[1] = a.state_in_bwd;
        states.out[1] = a.state_out_bwd;
    }

    // One cooperative launch (prep on the SMs the chains leave free) when the
    // chains leave room for it; else prep, then chain.
    TcPlan plan = plan_tc(a.B * a.H * ndir, nC, cooperative_supported());
    gdn::tc2::ChainSeg seg{plan.G, plan.L, lb};
    gdn_status s = GDN_ERR_UNSUPPORTED;
    if (plan.fused) {
        if (cudaMemsetAsync(ready, 0, nrec * sizeof(unsigned int), a.stream) != cudaSuccess) return GDN_ERR_CUDA;
        s = launch_fused<DV, Tout>(a, mk, mq, mv, mo, recs, lb, ready, nC, ndir, plan, states, out, seg, err);
    }
    if (s == GDN_ERR_UNSUPPORTED) {
        gdn::tc2::PrepOrder po{1, nC, 0};
        s = launch_prep<DV>(a, mk, mq, mv, recs, lb, nC, ndir, po, err);
        if (s != GDN_OK) return s;
        s = launch_chain<DV, Tout>(a, mo, recs, nC, ndir, states, out, seg, err);
    }
    if (s != GDN_OK || !bidir || f32_out) return s;
    gdn::LaunchScope ls("tc_bidir_cast", a.stream);
    const size_t n4 = n / 4;
    const int grid = (int)((n4 + 255) / 256 < (size_t)sm_count() * 8 ? (n4 + 255) / 256 : (size_t)sm_count() * 8);
    cast_bf16_kernel<<<grid, 256, 0, a.stream>>>(static_cast<const float4 *>(target), static_cast<uint2 *>(a.o), n4);
    return launch_status();
}

gdn_status dispatch_tc(const Args &a, int bidir) {
    if (a.dv == 128)
        return a.o_dt == GDN_F32 ? run_tc<128, float>(a, bidir) : run_tc<128, __nv_bfloat16>(a, bidir);
    return a.o_dt == GDN_F32 ? run_tc<64, float>(a, bidir) : run_tc<64, __nv_bfloat16>(a, bidir);
}

// ---------------------------------------------------------------------------
// Short causal calls: token by token (token_step.cuh)
// ---------------------------------------------------------------------------
// < 0: automatic (below); else calls of at most this many tokens
std::atomic<int> g_short_call_tokens{-1};

// Automatic choice, from B200 timings of single calls (d = 128): the token
// path costs about 2.5 us plus 0.37 us per token for each wave of CTAs
// (B*H*dv/32 CTAs over the SMs), a one-chunk call of the chunked path about
// 24 us; so the token path is taken while tokens x waves <= 48.
bool take_token_path(const Args &a) {
    const int lim = g_short_call_tokens.load(std::memory_order_relaxed);
    if (lim >= 0) return a.T <= lim;
    if (a.T > gdn::tok::kMaxT) return false;
    const long long ctas = (long long)a.B * a.H * (a.dv / gdn::tok::kCols);
    const long long waves = (ctas + sm_count() - 1) / sm_count();
    return (long long)a.T * waves <= 48;
}

template <int DK, int DV, typename Tin, typename Tout>
gdn_status run_token(const Args &a) {
    auto kern = gdn::tok::token_kernel<DK, DV, Tin, Tout>;
    constexpr int smem = gdn::tok::TokSmem<DK>::kBytes;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return GDN_ERR_CUDA;
    gdn::LaunchScope ls("token_step", a.stream);
    kern<<<dim3(DV / gdn::tok::kCols, a.B * a.H), gdn::tok::kThreads, smem, a.stream>>>(
        static_cast<const Tin *>(a.q), static_cast<const Tin *>(a.k), static_cast<const Tin *>(a.v), a.alpha,
        a.beta, a.state_in, a.state_out, static_cast<Tout *>(a.o), a.T, a.H);
    return launch_status();
}

template <typename Tin, typename Tout>
gdn_status token_dims(const Args &a) {
    if (a.dk == 128 && a.dv == 128) return run_token<128, 128, Tin, Tout>(a);
    if (a.dk == 128 && a.dv == 64) return run_token<128, 64, Tin, Tout>(a);
    if (a.dk == 64 && a.dv == 128) return run_token<64, 128, Tin, Tout>(a);
    return run_token<64, 64, Tin, Tout>(a);
}

gdn_status run_short(const Args &a) {
    if (a.dt == GDN_F32)
        return a.o_dt == GDN_F32 ? token_dims<float, float>(a) : token_dims<float, __nv_bfloat16>(a);
    return a.o_dt == GDN_F32 ? token_dims<__nv_bfloat16, float>(a) : token_dims<__nv_bfloat16, __nv_bfloat16>(a);
}

gdn_status run(const Args &a, int bidir) {
    const gdn_status s =
        check_ws(a, plan_workspace(a.B, a.T, a.H, a.dk, a.dv, a.dt, a.o_dt, bidir));
    if (s != GDN_OK) return s;
    if (a.T == 0) return empty_scan(a, bidir);
    if (!bidir && take_token_path(a)) return run_short(a);
    if (use_tc(a.dt, a.dk, a.dv)) return dispatch_tc(a, bidir);
    return a.dt == GDN_F32 ? dispatch_out<float>(a, bidir) : dispatch_out<__nv_bfloat16>(a, bidir);
}

// ---------------------------------------------------------------------------
// Readout epilogue (readout.cuh)
// ---------------------------------------------------------------------------
template <int DV, typename To, typename Tz, typename Ty>
gdn_status run_readout(const void *o, const void *z, const float *gamma, float eps, void *y, long long rows,
                       cudaStream_t stream) {
    const long long per_block = gdn::rd::kThreads / 32;
    long long blocks = (rows + per_block - 1) / per_block;
    const long long cap = (long long)sm_count() * 8;
    if (blocks > cap) blocks = cap;
    gdn::LaunchScope ls("readout", stream);
    gdn::rd::readout_kernel<DV, To, Tz, Ty><<<(int)blocks, gdn::rd::kThreads, 0, stream>>>(
        static_cast<const To *>(o), static_cast<const Tz *>(z), gamma, eps, static_cast<Ty *>(y), rows);
    return launch_status();
}

template <int DV, typename To, typename Tz>
gdn_status readout_y(gdn_dtype y_dt, const void *o, const void *z, const float *gamma, float eps, void *y,
                     long long rows, cudaStream_t s) {
    return y_dt == GDN_F32 ? run_readout<DV, To, Tz, float>(o, z, gamma, eps, y, rows, s)
                           : run_readout<DV, To, Tz, __nv_bfloat16>(o, z, gamma, eps, y, rows, s);
}

template <int DV, typename To>
gdn_status readout_z(gdn_dtype z_dt, gdn_dtype y_dt, const void *o, const void *z, const float *gamma, float eps,
                     void *y, long long rows, cudaStream_t s) {
    return z_dt == GDN_F32 ? readout_y<DV, To, float>(y_dt, o, z, gamma, eps, y, rows, s)
                           : readout_y<DV, To, __nv_bfloat16>(y_dt, o, z, gamma, eps, y, rows, s);
}

template <int DV>
gdn_status readout_o(gdn_dtype o_dt, gdn_dtype z_dt, gdn_dtype y_dt, const void *o, const void *z,
                     const float *gamma, float eps, void *y, long long rows, cudaStream_t s) {
    return o_dt == GDN_F32 ? readout_z<DV, float>(z_dt, y_dt, o, z, gamma, eps, y, rows, s)
                           : readout_z<DV, __nv_bfloat16>(z_dt, y_dt, o, z, gamma, eps, y, rows, s);
}

size_t dtype_bytes(gdn_dtype d) { return d == GDN_F32 ? 4 : 2; }

// ---------------------------------------------------------------------------
// Frame-wise delta operator (vda.cuh)
// ---------------------------------------------------------------------------
struct VdaArgs {
    const void *q, *k, *v;
    const float *alpha_f, *beta;
    const float *s_in, *s_in_bwd;
    float *s_out, *s_out_bwd;
    void *o;
    int B, F, U, H, dk, dv, bidir;
    gdn_dtype dt, o_dt;
    void *ws;
    size_t ws_bytes;
    cudaStream_t stream;
};

// workspace: A [F][B*H][dk][dk], B [F][B*H][dk][dv], states [ndir][F][B*H][dk][dv]
size_t vda_workspace(int B, int F, int H, int dk, int dv, int bidir) {
    const size_t fh = (size_t)F * B * H;
    return round_up(fh * dk * dk * 4, 256) + round_up(fh * dk * dv * 4, 256) +
           round_up((bidir ? 2 : 1) * fh * dk * dv * 4, 256);
}

template <int DK, int DV, typename Tin, typename Tout>
gdn_status run_vda(const VdaArgs &a) {
    using namespace gdn::vda;
    const int nbh = a.B * a.H, ndir = a.bidir ? 2 : 1;
    const size_t fh = (size_t)a.F * nbh;
    float *A = static_cast<float *>(a.ws);
    float *Bm = reinterpret_cast<float *>(static_cast<char *>(a.ws) + round_up(fh * DK * DK * 4, 256));
    float *st = reinterpret_cast<float *>(reinterpret_cast<char *>(Bm) + round_up(fh * DK * DV * 4, 256));
    if (std::is_same<Tin, __nv_bfloat16>::value && DK == 128) {
        // bf16 keys and values: the Gram and key-value products on the tensor cores
        CUtensorMap mk, mv;
        if (!encode_map(&mk, a.k, a.B, a.F * a.U, a.H, DK, 64, 128) ||
            !encode_map(&mv, a.v, a.B, a.F * a.U, a.H, DV, 64, 128))
            return GDN_ERR_CUDA;
        unsigned int *err = timeout_counter();
        if (!err) return GDN_ERR_CUDA;
        auto kern = vda_gram_tc_kernel<DV>;
        constexpr int smem = GramTcSmem<DV>::kAlloc;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return GDN_ERR_CUDA;
        gdn::LaunchScope ls("vda_gram_tc", a.stream);
        kern<<<dim3(a.F, nbh), kTcThreads, smem, a.stream>>>(mk, mv, a.beta, A, Bm, a.F, a.U, a.H, err);
        if (launch_status() != GDN_OK) return GDN_ERR_CUDA;
    } else {
        auto kern = vda_gram_kernel<DK, DV, Tin>;
        constexpr int smem = GramSmem<DK, DV>::kBytes;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return GDN_ERR_CUDA;
        gdn::LaunchScope ls("vda_gram", a.stream);
        kern<<<dim3(a.F, nbh), kThreads, smem, a.stream>>>(static_cast<const Tin *>(a.k), static_cast<const Tin *>(a.v),
                                                          a.beta, A, Bm, a.F, a.U, a.H);
        if (launch_status() != GDN_OK) return GDN_ERR_CUDA;
    }
    {
        auto kern = vda_factor_kernel<DK, DV>;
        constexpr int smem = FactorSmem<DK, DV>::kBytes;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return GDN_ERR_CUDA;
        gdn::LaunchScope ls("vda_factor", a.stream);
        kern<<<dim3(a.F, nbh), kChainThreads, smem, a.stream>>>(A);
        if (launch_status() != GDN_OK) return GDN_ERR_CUDA;
    }
    constexpr bool kTc = std::is_same<Tin, __nv_bfloat16>::value && DK == 128;
    {
        auto kern = vda_chain_kernel<DK, DV, kTc>;
        constexpr int smem = ChainSmem<DK, DV>::kBytes;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return GDN_ERR_CUDA;
        gdn::LaunchScope ls("vda_chain", a.stream);
        kern<<<dim3(nbh, ndir, DV / kSlice), kChainThreads, smem, a.stream>>>(A, Bm, a.alpha_f, a.s_in, a.s_in_bwd, a.s_out,
                                                                a.s_out_bwd, st, a.F, a.H);
        if (launch_status() != GDN_OK) return GDN_ERR_CUDA;
    }
    if (kTc) {   // states as operand images: the readout on the tensor cores
        CUtensorMap mq;
        if (!encode_map(&mq, a.q, a.B, a.F * a.U, a.H, DK, 64, 128)) return GDN_ERR_CUDA;
        unsigned int *err = timeout_counter();
        if (!err) return GDN_ERR_CUDA;
        auto kern = vda_readout_tc_kernel<DV, Tout>;
        constexpr int smem = ReadTcSmem<DV>::kAlloc;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return GDN_ERR_CUDA;
        gdn::LaunchScope ls("vda_readout_tc", a.stream);
        kern<<<dim3(a.F * ((a.U + 127) / 128), nbh), 128, smem, a.stream>>>(
            mq, reinterpret_cast<const unsigned char *>(st), static_cast<Tout *>(a.o), a.F, a.U, a.H, ndir, err);
        return launch_status();
    }
    auto kern = vda_readout_kernel<DK, DV, Tin, Tout>;
    constexpr int smem = ReadSmem<DK, DV>::kBytes;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return GDN_ERR_CUDA;
    gdn::LaunchScope ls("vda_readout", a.stream);
    kern<<<dim3(a.F * ((a.U + 63) / 64), nbh), kThreads, smem, a.stream>>>(
        static_cast<const Tin *>(a.q), st, static_cast<Tout *>(a.o), a.F, a.U, a.H, ndir);
    return launch_status();
}

template <typename Tin, typename Tout>
gdn_status vda_dims(const VdaArgs &a) {
    if (a.dk == 128 && a.dv == 128) return run_vda<128, 128, Tin, Tout>(a);
    if (a.dk == 128 && a.dv == 64) return run_vda<128, 64, Tin, Tout>(a);
    if (a.dk == 64 && a.dv == 128) return run_vda<64, 128, Tin, Tout>(a);
    return run_vda<64, 64, Tin, Tout>(a);
}

}  // namespace

// ---------------------------------------------------------------------------
// Scratch of gdn_step_noalloc: a file-scope device array, so that callers
// who cannot allocate device memory still get the workspace a call needs.
// Host code must not pass `g_noalloc_scratch` itself to a kernel (in host
// code the name is a host-side stand-in, not a device address); the device
// address is looked up once per device with cudaGetSymbolAddress.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[GDN_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up on the
// first call per device, with that device current).
gdn_status noalloc_scratch(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GDN_ERR_CUDA;
    std::lock_guard<std::mutex> g(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GDN_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return GDN_OK;
}

}  // namespace

extern "C" {

gdn_status gdn_scan_causal(const void *q, const void *k, const void *v, const float *alpha,
                           const float *beta, const float *state_in, float *state_out, void *o,
                           int B, int T, int H, int dk, int dv, gdn_dtype dt, gdn_dtype o_dt,
                           void *workspace, size_t ws_bytes, void *stream) {
    Args a{q, k, v, alpha, beta, state_in, state_out, o, B, T, H, dk, dv, dt, o_dt,
           workspace, ws_bytes, static_cast<cudaStream_t>(stream)};
    gdn_status s = check_common(a, T > 0);
    if (s != GDN_OK) return s;
    return run(a, 0);
}

gdn_status gdn_scan_bidir(const void *q, const void *k, const void *v, const float *alpha,
                          const float *beta, void *o, int B, int T, int H, int dk, int dv,
                          gdn_dtype dt, gdn_dtype o_dt, void *workspace, size_t ws_bytes,
                          void *stream) {
    Args a{q, k, v, alpha, beta, nullptr, nullptr, o, B, T, H, dk, dv, dt, o_dt,
           workspace, ws_bytes, static_cast<cudaStream_t>(stream)};
    gdn_status s = check_common(a, T > 0);
    if (s != GDN_OK) return s;
    return run(a, 1);
}

gdn_status gdn_scan_bidir_states(const void *q, const void *k, const void *v, const float *alpha,
                                 const float *beta, const float *state_in, const float *state_in_bwd,
                                 float *state_out, float *state_out_bwd, void *o, int B, int T, int H,
                                 int dk, int dv, gdn_dtype dt, gdn_dtype o_dt, void *workspace,
                                 size_t ws_bytes, void *stream) {
    Args a{q, k, v, alpha, beta, state_in, state_out, o, B, T, H, dk, dv, dt, o_dt,
           workspace, ws_bytes, static_cast<cudaStream_t>(stream), state_in_bwd, state_out_bwd};
    gdn_status s = check_common(a, T > 0);
    if (s != GDN_OK) return s;
    return run(a, 1);
}

gdn_status gdn_step(const void *q, const void *k, const void *v, const float *alpha,
                    const float *beta, float *state, void *o, int B, int T, int H, int dk, int dv,
                    gdn_dtype dt, gdn_dtype o_dt, void *workspace, size_t ws_bytes, void *stream) {
    if (!state) return GDN_ERR_NULL;
    Args a{q, k, v, alpha, beta, state, state, o, B, T, H, dk, dv, dt, o_dt,
           workspace, ws_bytes, static_cast<cudaStream_t>(stream)};
    gdn_status s = check_common(a, T > 0);
    if (s != GDN_OK) return s;
    return run(a, 0);
}

gdn_status gdn_step_noalloc(const void *q, const void *k, const void *v, const float *alpha,
                            const float *beta, float *state, void *o, int B, int T, int H, int dk,
                            int dv, gdn_dtype dt, gdn_dtype o_dt, void *stream) {
    if (!state) return GDN_ERR_NULL;
    Args a{q, k, v, alpha, beta, state, state, o, B, T, H, dk, dv, dt, o_dt,
           nullptr, 0, static_cast<cudaStream_t>(stream)};
    gdn_status s = check_common(a, T > 0);
    if (s != GDN_OK) return s;
    const size_t need = plan_workspace(B, T, H, dk, dv, dt, o_dt, 0);
    if (need > GDN_NOALLOC_SCRATCH_BYTES) return GDN_ERR_WORKSPACE;
    if (need > 0) {
        s = noalloc_scratch(&a.ws);
        if (s != GDN_OK) return s;
        a.ws_bytes = GDN_NOALLOC_SCRATCH_BYTES;
    }
    return run(a, 0);
}

size_t gdn_workspace_size(int B, int T, int H, int dk, int dv, gdn_dtype dt, gdn_dtype o_dt,
                          int bidir) {
    Args a{};
    a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv; a.dt = dt; a.o_dt = o_dt;
    if (check_common(a, false) != GDN_OK) return 0;
    return plan_workspace(B, T, H, dk, dv, dt, o_dt, bidir ? 1 : 0);
}

const char *gdn_status_string(gdn_status s) {
    switch (s) {
        case GDN_OK: return "ok";
        case GDN_ERR_NULL: return "a required pointer is NULL";
        case GDN_ERR_SHAPE: return "bad shape (B<1, H<1, T<0, size overflow, or overlapping state buffers)";
        case GDN_ERR_DTYPE: return "unknown dtype";
        case GDN_ERR_ALIGN: return "pointer not 16-byte aligned (workspace: 256-byte)";
        case GDN_ERR_UNSUPPORTED: return "unsupported head dimension (dk, dv must be 64 or 128)";
        case GDN_ERR_WORKSPACE: return "workspace smaller than gdn_workspace_size()";
        case GDN_ERR_CUDA: return "CUDA launch or copy failed";
    }
    return "unknown status";
}

const char *gdn_version(void) { return "gdn-b200 0.1 (sm_100a)"; }

int gdn_device_timeouts(unsigned int *count) {
    if (!count) return GDN_ERR_NULL;
    unsigned int *p = timeout_counter();
    if (!p) return GDN_ERR_CUDA;
    return cudaMemcpy(count, p, sizeof(unsigned int), cudaMemcpyDeviceToHost) == cudaSuccess
               ? GDN_OK : GDN_ERR_CUDA;
}

unsigned long long gdn_launch_count(void) {
    return gdn::LaunchStats::get().launches.load(std::memory_order_relaxed);
}

int gdn_set_short_call_tokens(int max_t) {
    const int v = max_t < 0 ? -1 : (max_t > gdn::tok::kMaxT ? gdn::tok::kMaxT : max_t);
    return g_short_call_tokens.exchange(v);
}

int gdn_set_chain_segments(int g) {
    return g_chain_segments.exchange(g < 1 ? -1 : g);
}

void gdn_set_kernel_timing(int on) { gdn::LaunchStats::get().timing.store(on != 0); }

int gdn_read_kernel_timing(char *names, int name_len, double *total_ms, int *launches, int max) {
    if (max < 0 || name_len < 1) return GDN_ERR_SHAPE;
    if (max > 0 && (!names || !total_ms || !launches)) return GDN_ERR_NULL;
    gdn::LaunchStats &st = gdn::LaunchStats::get();
    std::lock_guard<std::mutex> g(st.mu);
    int n = 0;
    gdn_status status = GDN_OK;
    for (auto &e : st.events) {
        double ms = 0.0;
        for (auto &pr : e.second) {
            float t = 0.f;
            if (cudaEventSynchronize(pr.second) != cudaSuccess ||
                cudaEventElapsedTime(&t, pr.first, pr.second) != cudaSuccess)
                status = GDN_ERR_CUDA;
            ms += t;
            cudaEventDestroy(pr.first);
            cudaEventDestroy(pr.second);
        }
        if (n < max) {
            strncpy(names + (size_t)n * name_len, e.first.c_str(), name_len - 1);
            names[(size_t)n * name_len + name_len - 1] = 0;
            total_ms[n] = ms;
            launches[n] = (int)e.second.size();
            ++n;
        }
    }
    st.events.clear();
    return status == GDN_OK ? n : status;
}

gdn_status gdn_vda_scan(const void *q, const void *k, const void *v, const float *alpha_frame, const float *beta,
                        const float *state_in, const float *state_in_bwd, float *state_out, float *state_out_bwd,
                        void *o, int B, int F, int U, int H, int dk, int dv, int bidir, gdn_dtype dt,
                        gdn_dtype o_dt, void *workspace, size_t ws_bytes, void *stream) {
    // the argument rules of the token scans, with T = F * U
    if (U < 1 || F < 0 || (long long)F * U > (1 << 30)) return GDN_ERR_SHAPE;
    Args c{q, k, v, alpha_frame, beta, state_in, state_out, o, B, F * U, H, dk, dv, dt, o_dt,
           workspace, ws_bytes, static_cast<cudaStream_t>(stream), bidir ? state_in_bwd : nullptr,
           bidir ? state_out_bwd : nullptr};
    gdn_status s = check_common(c, F > 0);
    if (s != GDN_OK) return s;
    if ((long long)F * B * H > 65535LL * 64) return GDN_ERR_SHAPE;
    if (F == 0) return empty_scan(c, bidir ? 1 : 0);
    s = check_ws(c, vda_workspace(B, F, H, dk, dv, bidir ? 1 : 0));
    if (s != GDN_OK) return s;
    const VdaArgs a{q, k, v, alpha_frame, beta, state_in, c.state_in_bwd, state_out, c.state_out_bwd, o,
                    B, F, U, H, dk, dv, bidir ? 1 : 0, dt, o_dt, workspace, ws_bytes, c.stream};
    if (dt == GDN_F32) return o_dt == GDN_F32 ? vda_dims<float, float>(a) : vda_dims<float, __nv_bfloat16>(a);
    return o_dt == GDN_F32 ? vda_dims<__nv_bfloat16, float>(a) : vda_dims<__nv_bfloat16, __nv_bfloat16>(a);
}

size_t gdn_vda_workspace_size(int B, int F, int U, int H, int dk, int dv, int bidir) {
    if (B < 1 || H < 1 || F < 0 || U < 1 || !((dk == 64 || dk == 128) && (dv == 64 || dv == 128))) return 0;
    return F == 0 ? 0 : vda_workspace(B, F, H, dk, dv, bidir ? 1 : 0);
}

gdn_status gdn_readout_gate(const void *o, gdn_dtype o_dt, const void *z, gdn_dtype z_dt, const float *gamma,
                            float eps, void *y, gdn_dtype y_dt, int B, int T, int H, int dv, void *stream) {
    const gdn_dtype dts[3] = {o_dt, z_dt, y_dt};
    for (gdn_dtype d : dts)
        if (d != GDN_F32 && d != GDN_BF16) return GDN_ERR_DTYPE;
    if (B < 1 || H < 1 || T < 0 || (long long)B * H > 65535LL || T > (1 << 30)) return GDN_ERR_SHAPE;
    if (dv != 64 && dv != 128) return GDN_ERR_UNSUPPORTED;
    if (!(eps >= 0.f) || eps > 3.0e38f) return GDN_ERR_SHAPE;   // also rejects NaN
    if (T == 0) return GDN_OK;
    if (!o || !z || !y) return GDN_ERR_NULL;
    if (!aligned(o, 16) || !aligned(z, 16) || !aligned(y, 16) || (gamma && !aligned(gamma, 4)))
        return GDN_ERR_ALIGN;
    // y may be o or z itself (same dtype); no other overlap
    const long long rows = (long long)B * T * H;
    auto span = [&](const void *p, gdn_dtype d) { return (size_t)rows * dv * dtype_bytes(d); };
    auto overlap = [](const void *a, size_t na, const void *b, size_t nb) {
        const char *p = static_cast<const char *>(a), *q = static_cast<const char *>(b);
        return p < q + nb && q < p + na;
    };
    if (overlap(y, span(y, y_dt), o, span(o, o_dt)) && !(y == o && y_dt == o_dt)) return GDN_ERR_SHAPE;
    if (overlap(y, span(y, y_dt), z, span(z, z_dt)) && !(y == z && y_dt == z_dt)) return GDN_ERR_SHAPE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return dv == 128 ? readout_o<128>(o_dt, z_dt, y_dt, o, z, gamma, eps, y, rows, s)
                     : readout_o<64>(o_dt, z_dt, y_dt, o, z, gamma, eps, y, rows, s);
}

}  // extern "C"

