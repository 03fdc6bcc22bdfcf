// Shared device helpers for libgdn kernels (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdn.h"

namespace gdn {

// Codes a kernel ORs into the device-side error word (the word lives in the
// tensor-core translation unit): a bounded wait gave up, or a packed batch's
// sequence offsets were not a non-decreasing list inside [0, T].
enum : unsigned { kErrWaitTimeout = 1u, kErrBadSeqlens = 2u };

// Token range of the (sequence, head) handled by CTA `bid`. Dense batches
// (cu == nullptr): one sequence of length L per row of the (B*H, L) token grid.
// Packed variable-length batches: sequence n of head h is tokens cu[n] .. cu[n+1]-1
// of row h of an (H, L) token grid (CTA bid = n * H + h). A malformed range is
// recorded in the error word and handled as an empty sequence.
struct SeqSpan {
    int head_row;   // row of the token grid (and z coordinate of the TMA maps)
    int t0;         // first token of the sequence in that row
    int len;        // tokens in the sequence
};
__device__ __forceinline__ SeqSpan seq_span(const int *cu, int bid, int H, int L, unsigned *err) {
    if (!cu) return SeqSpan{bid, 0, L};
    const int n = bid / H, h = bid - n * H;
    const int a = cu[n], b = cu[n + 1];
    if (a < 0 || b < a || b > L) {
        if (err && threadIdx.x == 0) atomicOr(err, kErrBadSeqlens);
        return SeqSpan{h, 0, 0};
    }
    return SeqSpan{h, a, b - a};
}

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

// Options of the prefill kernels: o in fp32 or bf16, vector-valued gates, and the Mamba
// D-skip term o_t += D_h (elementwise) v_t, D of shape (H, dv) (page "【CS336】lecture4",
// section "继续改进：Mamba": a term in v added at the output, like a residual branch).
struct FwdOpts {
    bool bf16;            // o is bf16 (round to nearest even), else fp32
    const float *dskip;   // (H, dv) fp32, nullable (no skip term)
    bool gate_per_key;    // g holds one log-decay per key coordinate: (rows, dk) in prefill (fp32
                          // chunk kernel), (N, H, dk) in decode
};
// The same, as a kernel argument: o, and for the D-skip term the input v (bf16 for the
// tensor-core kernels; same (rows, dv) layout as o) with D.
struct OutArgs {
    void *o;
    const __nv_bfloat16 *v;   // nullptr: no D-skip term
    const float *dskip;       // (H, dv)
    int bf16;
};

// One value column of a 64-token output tile: ov[r] = o[row r][column] for r < n, at
// element offset elem0 + r * stride of o. Adds dj * v at the same offsets when v is
// given (the D-skip term, fp32 fused multiply-add), then stores fp32 or bf16.
__device__ __forceinline__ void store_out_rows(float (&ov)[64], void *o, size_t elem0, int n, int stride,
                                               bool bf16, float dj, const __nv_bfloat16 *v) {
#pragma unroll
    for (int r0 = 0; r0 < 64; r0 += 16) {
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = ov[r0 + r];
        if (v) {
#pragma unroll
            for (int r = 0; r < 16; ++r)
                if (r0 + r < n) x[r] = fmaf(dj, __bfloat162float(v[elem0 + static_cast<size_t>(r0 + r) * stride]), x[r]);
        }
        if (bf16) {
            __nv_bfloat16 *ob = static_cast<__nv_bfloat16 *>(o) + elem0;
#pragma unroll
            for (int r = 0; r < 16; ++r)
                if (r0 + r < n) ob[static_cast<size_t>(r0 + r) * stride] = __float2bfloat16_rn(x[r]);
        } else {
            float *of = static_cast<float *>(o) + elem0;
#pragma unroll
            for (int r = 0; r < 16; ++r)
                if (r0 + r < n) of[static_cast<size_t>(r0 + r) * stride] = x[r];
        }
    }
}

}  // namespace gdn

// Host-side launchers implemented in the kernel translation units.
namespace gdn {
// cu (device, nullable): sequence offsets of a packed batch; B is then the number of
// sequences and L the packed length T of each head row.
gdn_status_t launch_simt_fwd(const void *q, const void *k, const void *v, const float *beta,
                             const float *g, void *o, const float *s0, float *s_final,
                             const int *cu, int B, int H, int L, int dk, int dv, int chunk,
                             float scale, gdn_dtype_t in_dtype, FwdOpts oo, cudaStream_t stream);
gdn_status_t launch_decode(const void *q, const void *k, const void *v, const float *beta,
                           const float *g, float *state, void *o, int N, int H, int dk, int dv,
                           float scale, gdn_dtype_t in_dtype, FwdOpts oo, cudaStream_t stream);
}  // namespace gdn
