// common.cuh — small helpers shared by the libgdn kernels (device side).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace gdn {

// Status bits that kernels OR into the per-device status word (a device
// pointer handed to them as an argument) instead of trapping.  Host side:
// gdn_get_status() reads and clears the word.
enum : int { kStatusTimeout = 1 };

__device__ __forceinline__ void raise_status(int* status, int bits) {
    if (status) atomicOr(status, bits);
}

// Element load/store for the two data types of K, V, Q, W, U, O.
__device__ __forceinline__ float ld_elem(const float* p, int64_t i) { return p[i]; }
__device__ __forceinline__ float ld_elem(const __nv_bfloat16* p, int64_t i) {
    return __bfloat162float(p[i]);
}
__device__ __forceinline__ void st_elem(float* p, int64_t i, float v) { p[i] = v; }
__device__ __forceinline__ void st_elem(__nv_bfloat16* p, int64_t i, float v) {
    p[i] = __float2bfloat16_rn(v);
}

}  // namespace gdn
