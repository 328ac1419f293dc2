// tc_fused.cuh -- prep and chain in one cooperative launch.
//
// When the chains need fewer CTAs than the GPU has SMs (few heads, long
// sequences), one launch runs both: CTAs [0, n_chain) are chain CTAs (one
// segment of one chain each, as in chain_kernel) and every other CTA runs two
// prep pipelines (each as in prep_kernel, on half of the CTA's shared memory
// and TMEM).  The prep pipelines walk the chunk tasks in the order the chains
// consume them and set a ready flag per record once its stores have landed; a
// chain waits for the flag of each record (and of each chunk bound it reads
// while choosing its starting point) before using it.  The launch is
// cooperative, so every CTA is resident at once: the prep pipelines never wait
// on a chain, and a chain only waits on prep pipelines that are running.
// Every wait is bounded (a flag wait gives up after kFlagWaitNs and flags an
// error).
#pragma once

#include "tc_chain.cuh"
#include "tc_prep.cuh"

namespace gdn {
namespace tc2 {

// Shared memory of a prep CTA of the fused launch: two pipeline areas.
template <int DV>
struct FusedPrepSmem {
    static constexpr int kArea = (PrepSmem<DV>::kBytes + 1023) / 1024 * 1024;
    static constexpr int kCtl = 2 * kArea;          // TMEM base of the CTA
    static constexpr int kBytes = kCtl + 16;
};

// (the dynamic shared memory is 1024-aligned, checked at run time)
template <int DV>
constexpr int fused_smem_alloc() {
    return ChainSmem<DV>::kAlloc > FusedPrepSmem<DV>::kBytes ? ChainSmem<DV>::kAlloc : FusedPrepSmem<DV>::kBytes;
}

// grid n_chain + n_prep CTAs (cooperative), block kChainThreads.
// Chain CTA i: segment i % G, (b,h) (i / G) % nbh, direction i / (G * nbh).
template <int DV, typename Tout>
__global__ void __launch_bounds__(kChainThreads, 1)
fused_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
             const float *__restrict__ alpha, const float *__restrict__ beta, unsigned char *__restrict__ recs,
             float *__restrict__ lb, unsigned int *__restrict__ ready, const ChainStates states,
             const ChainOut<Tout> out, const ChainSeg seg, PrepOrder po, int T, int H, int nC, int nbh, int ndir,
             int n_chain, unsigned int *__restrict__ err)
{
    static_assert(kChainThreads >= 2 * kPrepThreads, "two prep pipelines per CTA");
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    if (smem_u32(smem_raw) & 1023u) {   // no slack was allocated for aligning it here
        if (threadIdx.x == 0 && err) atomicAdd(err, 1u);
        return;
    }
    unsigned char *smem = smem_raw;
    if ((int)blockIdx.x < n_chain) {
        const int i = blockIdx.x;
        chain_body<DV, Tout>(&tm_o, recs, states, out, seg, ready, H, nC, i % seg.G, (i / seg.G) % nbh,
                             i / (seg.G * nbh), nbh, smem, err);
        return;
    }
    // ---- two prep pipelines: warps 0-7 and 8-15 (the rest of the block idles)
    using FS = FusedPrepSmem<DV>;
    const int warp = threadIdx.x >> 5;
    uint32_t *tmem_base_s = reinterpret_cast<uint32_t *>(smem + FS::kCtl);
    if (warp == 0) {
        tmem_alloc(tmem_base_s, 2 * kPrepTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_s;
    if (warp < 16) {
        const int pipe = warp >> 3;
        const int npipes = 2 * ((int)gridDim.x - n_chain);
        prep_pipeline<DV>(&tm_k, &tm_q, &tm_v, alpha, beta, recs, lb, ready, T, H, nC, nbh, ndir, po,
                          2 * ((int)blockIdx.x - n_chain) + pipe, npipes, smem + pipe * FS::kArea,
                          tmem + pipe * kPrepTmemCols, threadIdx.x & (kPrepThreads - 1), 1 + pipe, 3 + pipe,
                          err);
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 2 * kPrepTmemCols);
}

}  // namespace tc2
}  // namespace gdn
