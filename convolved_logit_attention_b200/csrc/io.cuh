// Element access for the two I/O precisions (fp32, bf16); arithmetic is fp32.
#pragma once

#include <cuda_bf16.h>

namespace mta {

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Four consecutive elements widened to fp32; p must be aligned to four
// elements (16 bytes for fp32, 8 for bf16).
__device__ __forceinline__ void load4_f32(const float *p, float y[4]) {
    const float4 t = *reinterpret_cast<const float4 *>(p);
    y[0] = t.x; y[1] = t.y; y[2] = t.z; y[3] = t.w;
}
__device__ __forceinline__ void load4_f32(const __nv_bfloat16 *p, float y[4]) {
    const uint2 t = *reinterpret_cast<const uint2 *>(p);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&t.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&t.y);
    y[0] = __low2float(a); y[1] = __high2float(a); y[2] = __low2float(b); y[3] = __high2float(b);
}

}  // namespace mta
