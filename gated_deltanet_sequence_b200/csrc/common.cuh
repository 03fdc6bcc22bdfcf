// Shared device helpers for libgdn kernels (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdn.h"

namespace gdn {

// Codes a kernel ORs into the device-side error word when it gives up on a
// bounded wait (the word lives in the tensor-core translation unit).
enum : unsigned { kErrWaitTimeout = 1u };

template <typename T> __device__ __forceinline__ float ld_in(const T *p);
template <> __device__ __forceinline__ float ld_in<float>(const float *p) { return *p; }
template <> __device__ __forceinline__ float ld_in<__nv_bfloat16>(const __nv_bfloat16 *p) {
    return __bfloat162float(*p);
}

// Read-only, streaming (do not allocate in L1) 16-byte load / store.
__device__ __forceinline__ float4 ld_stream4(const float *p) {
    float4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w) : "l"(p));
    return r;
}
__device__ __forceinline__ float4 ld_global4(const float *p) {
    float4 r;
    asm volatile("ld.global.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w) : "l"(p));
    return r;
}
__device__ __forceinline__ void st_global4(float *p, float4 v) {
    asm volatile("st.global.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z),
                 "f"(v.w) : "memory");
}

}  // namespace gdn

// Host-side launchers implemented in the kernel translation units.
namespace gdn {
gdn_status_t launch_simt_fwd(const void *q, const void *k, const void *v, const float *beta,
                             const float *g, float *o, const float *s0, float *s_final, int B,
                             int H, int L, int dk, int dv, int chunk, float scale,
                             gdn_dtype_t in_dtype, cudaStream_t stream);
gdn_status_t launch_decode(const void *q, const void *k, const void *v, const float *beta,
                           const float *g, float *state, float *o, int N, int H, int dk, int dv,
                           float scale, gdn_dtype_t in_dtype, cudaStream_t stream);
}  // namespace gdn
