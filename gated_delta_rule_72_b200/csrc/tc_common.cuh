// tc_common.cuh -- pieces shared by the tensor-core prep and chain kernels:
// the per-chunk record they exchange, operand layouts and the bf16 hi/lo split.
//
// Precision scheme.  Every tensor-core contraction is kind::f16 with bf16
// operands and fp32 accumulation.  q, k, v are bf16 already and enter as they
// are (their products are exact).  A computed operand X (the inverse T, the
// readout mask P, the state S, the correction Delta) enters as the pair
// X_hi = bf16(X), X_lo = bf16(X - X_hi), about 16 significant bits, and the
// product X*Y is taken as X_hi*Y + X_lo*Y (three terms when both sides are
// split).  Only W = T diag(beta e^g) K is rounded once to bf16.  Against the
// FP64 sequential recurrence this keeps max|o - exact| / rms(o) near 1.5e-3 on
// 32k-token sequences, where plain bf16 operands reach 4e-2 .. 6e-2.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace gdn {
namespace tc2 {

using namespace gdn::sm100;

constexpr int kDK = 128;                     // key dimension of the tensor-core path
constexpr uint32_t kWaitTries = 1u << 24;    // bounded mbarrier polls (try_wait)
constexpr unsigned long long kFlagWaitNs = 2000000000ull;   // bound of a wait on another CTA (2 s)

// Granule of the U layout in the record (columns of d_v); a chain CTA's
// slice is a whole number of granules.
constexpr int kSliceCols = 32;

// Byte offset of U[row][col] inside one 64 x 32 fp32 granule: 128-byte rows
// whose 16-byte chunks are XOR-swizzled with row % 8, so that eight threads
// reading the same columns of eight consecutive rows hit distinct banks.
__host__ __device__ constexpr int u_off(int row, int col) {
    return row * 128 + ((((col >> 2) ^ row) & 7) << 4) + (col & 3) * 4;
}

// 128B / 64B swizzle of a byte offset inside a 1024-aligned tile, as TMA
// applies it (16-byte chunk bits XORed with the 128-byte row bits).
__device__ __forceinline__ int swz128(int L) { return L ^ (((L >> 7) & 7) << 4); }
__device__ __forceinline__ int swz64(int L) { return L ^ (((L >> 7) & 3) << 4); }

// Per-chunk record written by the prep kernel and read by the chain kernel,
// rows in FORWARD token order for either direction (the reverse direction's
// permutation is folded into the record by the prep kernel):
//   W   bf16, 64 rows x 128 (d_k) as two 128B-swizzled 64-column   16384 B
//       blocks (the image a SWIZZLE_128B tile load would write), so that
//       it stacks under the Q tile into one M=128 operand
//   Ph  bf16, 64 x 64, 128B-swizzled K-major image                  8192 B
//   Pl  bf16, same layout (P - Ph)                                 8192 B
//   U   fp32, [DV/32] granules of 64 x 32, rows swizzled (u_off)  256*DV B
//   dq[64], dkk[64], ds, padding                                   1024 B
// so that a chain CTA fetches its operands with a handful of bulk copies.
template <int DV>
struct Rec {
    static constexpr int kW = 0;
    static constexpr int kPh = 16384;
    static constexpr int kPl = 24576;
    static constexpr int kU = 32768;
    static constexpr int kUSlice = 64 * kSliceCols * 4;     // bytes of one slice of U
    static constexpr int kGate = kU + 64 * DV * 4;
    static constexpr int kGateCopy = 528;                   // dq, dkk, ds rounded to 16 bytes
    static constexpr int kBytes = kGate + 1024;
};

// K-major no-swizzle bf16 tile with 64 MN rows: element (row, k) at
// (k/8)*1024 + row*16 + (k%8)*2  (leading byte offset 1024, stride 128).
__device__ __forceinline__ int kmaj64(int row, int k) { return (k >> 3) * 1024 + row * 16 + (k & 7) * 2; }

// MN-major no-swizzle bf16 tile with K extent KEXT: element (mn, k) at
// (k/8)*128 + (mn/8)*(KEXT*16) + (k%8)*16 + (mn%8)*2  (leading byte offset
// 128 between groups of 8 K-rows, stride byte offset KEXT*16 between groups
// of 8 MN elements).  A thread owning one K-row writes 16-byte cells.
template <int KEXT>
__device__ __forceinline__ int mnmaj(int mn, int k) {
    return (k >> 3) * 128 + (mn >> 3) * (KEXT * 16) + (k & 7) * 16 + (mn & 7) * 2;
}

// Element (row, col) of a 128B-swizzled TMA tile of 64-column blocks
// (block stride `blk`): the 16-byte chunk index is XORed with row % 8.
__device__ __forceinline__ int sw128(int row, int col, int blk) {
    return (col >> 6) * blk + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) + (col & 7) * 2;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&v);
}
// hi = bf16(x), lo = bf16(x - hi)
__device__ __forceinline__ void split2(float a, float b, uint32_t &hi, uint32_t &lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = *reinterpret_cast<const uint32_t *>(&l);
}

// Element (mn, k) of a 128B-swizzled MN-major operand: 128-byte rows of 64
// MN elements, one row per k, atoms of 8 rows (1024 B) along k, groups of 64
// MN elements `mn_group` bytes apart.  (The layout a SWIZZLE_128B tile load
// writes for a [k][mn] tensor; read with sdesc_sw128_mn.)
__device__ __forceinline__ int swz_mn(int mn, int k, int mn_group) {
    return (mn >> 6) * mn_group + (k >> 3) * 1024 + (k & 7) * 128 + ((((mn & 63) >> 3) ^ (k & 7)) << 4) +
           (mn & 7) * 2;
}

// Descriptor of a 128B-swizzled operand used MN-major (MN contiguous inside
// the 128-byte rows): groups of 64 MN elements `mn_group` bytes apart.
__device__ __forceinline__ uint64_t sdesc_sw128_mn(uint32_t saddr, uint32_t mn_group) {
    uint64_t d = sdesc_sw128(saddr);
    return (d & ~(0x3FFFull << 16)) | ((uint64_t)((mn_group >> 4) & 0x3FFF) << 16);
}

// 1-d bulk copy global -> shared, completion counted on `bar`.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void named_barrier(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

}  // namespace tc2
}  // namespace gdn
