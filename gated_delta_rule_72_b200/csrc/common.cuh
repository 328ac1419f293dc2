// common.cuh -- small device helpers shared by the library's kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

// Tokens per chunk of the chunkwise (WY/UT) evaluation.
constexpr int kChunk = 64;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Position of chunk-local processing row r of chunk c in the token sequence.
// The forward pass walks a chunk front to back; the reverse pass walks the
// same chunk back to front, so its row r is token C-1-r of the chunk.
__device__ __forceinline__ int token_of_row(int c, int r, int dir) {
    return c * kChunk + (dir == 0 ? r : kChunk - 1 - r);
}

}  // namespace gdn
