// gdn_dtype.cuh -- element conversions for the two tensor dtypes (fp32, bf16).
#pragma once
#include <cuda_bf16.h>

namespace gdn {
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void store_as(float* p, float x) { *p = x; }
__device__ __forceinline__ void store_as(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
}  // namespace gdn
