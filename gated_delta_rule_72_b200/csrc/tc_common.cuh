// tc_common.cuh -- pieces shared by the tensor-core prep and chain kernels:
// the per-chunk record they exchange, operand layouts and rounding helpers.
//
// Precision scheme.  Every tensor-core contraction of the scan is kind::f16
// with fp16 operands and fp32 accumulation.  The bf16 inputs q, k, v are
// exactly representable in fp16 (8 significant bits; magnitudes of unit-norm
// keys and queries and of N(0,1) values sit far inside fp16's range), so the
// Gram products stay exact; every computed operand (the inverse T scaled by
// the gates, W, U, the decayed keys and queries, the readout mask P, the
// state S and the correction Delta) is rounded once to fp16 (11 significant
// bits).  The state itself is carried in fp32 and only its operand copy is
// rounded.  Emulated against the FP64 sequential recurrence on full-length
// sequences this gives max|o - exact| / rms(o) of 3e-3 .. 8e-3 (tolerance
// 2e-2 for bf16 inputs); bf16 operands would give 4e-2 .. 6e-2.  fp16 caps
// |values| at 65504: the state, U and Delta must stay below that, which holds
// for unit-norm keys and values of moderate size (the scan is linear in v and
// the state, so larger values can be scaled down by the caller).
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"
#include "sm100.cuh"

namespace gdn {
namespace tc2 {

using namespace gdn::sm100;

constexpr int kDK = 128;                     // key dimension of the tensor-core path
constexpr uint32_t kWaitTries = 1u << 24;    // bounded mbarrier polls (try_wait)
constexpr unsigned long long kFlagWaitNs = 2000000000ull;   // bound of a wait on another CTA (2 s)

// Sequence-parallel chains start a segment from a zero state some chunks
// before its first output, far enough back that the product of the skipped
// transitions has 2-norm at most e^kLogWindow = 2^-30 (see tc_chain.cuh).
constexpr float kLogWindow = -20.79441542f;  // ln(2^-30)

// 128B / 64B swizzle of a byte offset inside a 1024-aligned tile, as TMA
// applies it (16-byte chunk bits XORed with the 128-byte row bits).
__device__ __forceinline__ int swz128(int L) { return L ^ (((L >> 7) & 7) << 4); }

// Per-chunk record written by the prep kernel and read by the chain kernel,
// rows in FORWARD token order for either direction (the reverse direction's
// permutation is folded in by the prep kernel), all operands fp16:
//   [Q~; W]  two d_k blocks of 16 KB; block b holds d_k columns 64b..64b+63 of
//            Q~ = diag(e^g) Q (rows 0-63) and W = T diag(beta e^g) K (rows
//            64-127) as one 128-row, 128B-swizzled K-major operand (the image a
//            SWIZZLE_128B tile load would write)                       32768 B
//   K~       diag(e^{g_last - g}) K, the image of a SWIZZLE_128B tile load of
//            the key tile (two 8 KB blocks of 64 d_k columns)           16384 B
//   P        the readout mask, 64 x 64, 128B-swizzled K-major image      8192 B
//   U        T diag(beta) V, 64 rows of DV values; the 16-byte chunks of a
//            row are XOR-swizzled with row % 8 (u16_off)              128*DV B
//   ds       e^{g_last} (fp32), padded to 16 bytes
// so that a chain CTA fetches the whole record with one bulk copy.  The
// readout mask is followed by U so that an M=128 product over P reads finite
// (unused) rows past its end.
template <int DV>
struct Rec {
    static constexpr int kQW = 0;
    static constexpr int kK = 32768;
    static constexpr int kP = 49152;
    static constexpr int kU = 57344;
    static constexpr int kGate = kU + 64 * DV * 2;
    static constexpr int kBytes = kGate + 16;                  // copied per chunk
    static constexpr int kStride = (kBytes + 127) / 128 * 128;   // record pitch in the workspace
    static constexpr int kStage = (kBytes + 1023) / 1024 * 1024; // shared-memory stage
    static_assert(kBytes % 16 == 0, "bulk copies move multiples of 16 bytes");
};

// Byte offset of U[row][col] in the record: rows of 2*DV bytes, 16-byte
// chunks XOR-swizzled with row % 8, so that 32 threads reading the same
// columns of 32 consecutive rows spread over every bank.
template <int DV>
__host__ __device__ constexpr int u16_off(int row, int col) {
    return row * (2 * DV) + ((((col >> 3) ^ row) & 7) | ((col >> 3) & ~7)) * 16 + (col & 7) * 2;
}

// K-major no-swizzle 16-bit tile with 64 MN rows: element (row, k) at
// (k/8)*1024 + row*16 + (k%8)*2  (leading byte offset 1024, stride 128).
__device__ __forceinline__ int kmaj64(int row, int k) { return (k >> 3) * 1024 + row * 16 + (k & 7) * 2; }

// Element (row, col) of a 128B-swizzled TMA tile of 64-column blocks
// (block stride `blk`): the 16-byte chunk index is XORed with row % 8.
__device__ __forceinline__ int sw128(int row, int col, int blk) {
    return (col >> 6) * blk + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) + (col & 7) * 2;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&v);
}
__device__ __forceinline__ uint32_t pack_f16(float a, float b) {
    const __half2 v = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&v);
}
__device__ __forceinline__ float2 unpack_f16(uint32_t u) {
    return __half22float2(*reinterpret_cast<const __half2 *>(&u));
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u));
}
// hi = bf16(x), lo = bf16(x - hi)  (the frame-wise operator's operands)
__device__ __forceinline__ void split2(float a, float b, uint32_t &hi, uint32_t &lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = *reinterpret_cast<const uint32_t *>(&l);
}

// Descriptor of a 128B-swizzled operand used MN-major (MN contiguous inside
// the 128-byte rows): groups of 64 MN elements `mn_group` bytes apart.
__device__ __forceinline__ uint64_t sdesc_sw128_mn(uint32_t saddr, uint32_t mn_group) {
    uint64_t d = sdesc_sw128(saddr);
    return (d & ~(0x3FFFull << 16)) | ((uint64_t)((mn_group >> 4) & 0x3FFF) << 16);
}

// Element (mn, k) of a 128B-swizzled MN-major 16-bit operand: one 128-byte
// row of 64 MN elements per k, atoms of 8 rows (1024 B) along k, groups of 64
// MN elements `mn_group` bytes apart (read with sdesc_sw128_mn).
__device__ __forceinline__ int swz_mn(int mn, int k, int mn_group) {
    return (mn >> 6) * mn_group + (k >> 3) * 1024 + (k & 7) * 128 + ((((mn & 63) >> 3) ^ (k & 7)) << 4) +
           (mn & 7) * 2;
}

// 1-d bulk copy global -> shared, completion counted on `bar`.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Load bypassing L1 (for values another CTA publishes behind a flag).
__device__ __forceinline__ float ld_cg(const float *p) { return __ldcg(p); }

}  // namespace tc2
}  // namespace gdn
