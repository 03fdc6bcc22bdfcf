// Shared device helpers for libgdn kernels (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdn.h"

namespace gdn {

// Codes a kernel ORs into the device-side error word (the word lives in the
// tensor-core translation unit): a bounded wait gave up, a packed batch's sequence offsets
// were not a non-decreasing list inside [0, T], a stored result was not finite, or (debug
// builds) an access index fell outside the extent its launch implies.
enum : unsigned { kErrWaitTimeout = 1u, kErrBadSeqlens = 2u, kErrNonFinite = 4u, kErrBounds = 8u };

// Bounds checks of the debug build (-DGDN_DEBUG_BOUNDS): in_bounds(i, n, err) is true for
// 0 <= i < n; otherwise it sets kErrBounds in the error word and the caller skips the access
// (nothing traps). Release builds compile every check to true.
#ifdef GDN_DEBUG_BOUNDS
__device__ __forceinline__ bool in_bounds(long long i, long long n, unsigned *err) {
    if (i >= 0 && i < n) return true;
    if (err) atomicOr(err, kErrBounds);
    return false;
}
#else
__device__ __forceinline__ bool in_bounds(long long, long long, unsigned *) { return true; }
#endif

// Non-finite detector for stored results: nf <- nf + 0 * x keeps nf at 0 for finite x and
// turns it into NaN for an infinite or NaN x (0 * inf = NaN), one FMA per value (IEEE
// arithmetic: the build does not relax it).
__device__ __forceinline__ void probe_finite(float &nf, float x) { nf = fmaf(x, 0.f, nf); }
// The probe over the first n values of a 64-value tile: a pairwise sum (an inf or NaN value
// makes the sum inf or NaN; so would finite values summing beyond fp32 range, itself an
// overflow), then one probe step. 63 adds of depth 6, so no long dependency chain.
__device__ __forceinline__ void probe_tile(float &nf, const float (&x)[64], int n) {
    float t[32];
    if (n >= 64) {
#pragma unroll
        for (int i = 0; i < 32; ++i) t[i] = x[2 * i] + x[2 * i + 1];
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) t[i] = (2 * i < n ? x[2 * i] : 0.f) + (2 * i + 1 < n ? x[2 * i + 1] : 0.f);
    }
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) t[i] += t[i + w];
    probe_finite(nf, t[0]);
}
// The kernels probe the last output tile of each sequence and the whole final state. A
// non-finite value that reaches the state (any fp16 overflow of the state chain) stays in it
// and so reaches the last tile and the final state; a non-finite value confined to rows of an
// earlier tile is not seen. Probing every tile cost 1.5-2.5 % of the prefill time.
__device__ __forceinline__ bool probe_chunk(int c, int nchunks) { return c == nchunks - 1; }
// Records kErrNonFinite once per warp when some lane's probe saw a non-finite value. Every
// lane of the warp calls it; a CTA that gave up on a wait passes 0 (its stores stopped early
// and the timeout is what gdn_sync_status reports).
__device__ __forceinline__ void report_nonfinite(float nf, unsigned *err) {
    const bool bad = __any_sync(0xffffffffu, nf != nf);
    if (bad && (threadIdx.x & 31) == 0 && err) atomicOr(err, kErrNonFinite);
}

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

// Packed batches of at most this many sequences start their longest sequences first.
constexpr int kLongestFirstMax = 256;

// Block bid of a packed batch of nseq sequences -> state index n * H + h of the (sequence,
// head) pair it takes: blocks r * H .. r * H + H - 1 take the sequence of rank r by length
// (longest first, ties by index). Blocks start in index order as SMs free up, so the longest
// sequences start first and the call ends about when its longest sequence does. A malformed
// offset array still gives a permutation (the chosen sequence's offsets are checked after).
__device__ __forceinline__ int longest_first(const int *__restrict__ cu, int bid, int H, int nseq) {
    __shared__ int len[kLongestFirstMax];
    __shared__ int pick;
    if (nseq > kLongestFirstMax) return bid;
    const int r = bid / H, h = bid - r * H;
    for (int i = threadIdx.x; i < nseq; i += blockDim.x) len[i] = cu[i + 1] - cu[i];
    __syncthreads();
    for (int i = threadIdx.x; i < nseq; i += blockDim.x) {
        const int li = len[i];
        int rank = 0;
        for (int k = 0; k < nseq; ++k) rank += (len[k] > li || (len[k] == li && k < i)) ? 1 : 0;
        if (rank == r) pick = i;
    }
    __syncthreads();
    return pick * H + h;
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
// Output normalisation (page "LinearAttention 概述", section "The Devil in Linear
// Transformer": the normaliser's denominator is dropped and the output is normalised
// instead, O = XNorm(Q (K^T V))): each output row of each head over its dv values, after
// the skip term and before the output rounding, times a weight (H, dv) (nullable: ones).
enum : int { kXNormNone = 0, kXNormRms = 1, kXNormLayer = 2 };
struct FwdOpts {
    bool bf16;            // o is bf16 (round to nearest even), else fp32
    const float *dskip;   // (H, dv) fp32, nullable (no skip term)
    bool gate_per_key;    // g holds one log-decay per key coordinate: (rows, dk) in prefill (fp32
                          // chunk kernel), (N, H, dk) in decode
    int xnorm;            // kXNorm*
    const float *xw;      // (H, dv) fp32 weight of the output normalisation, nullable
    float xeps;           // added under the root to the row's mean square (variance)
};
// The same, as a kernel argument: o, and for the D-skip term the input v (bf16 for the
// tensor-core kernels; same (rows, dv) layout as o) with D.
struct OutArgs {
    void *o;
    const __nv_bfloat16 *v;   // nullptr: no D-skip term
    const float *dskip;       // (H, dv)
    int bf16;
    int xnorm;                // kXNorm*
    const float *xw;          // (H, dv), nullable
    float xeps;
};

// The kernel argument of the tensor-core kernels (bf16 v for the skip term).
inline OutArgs make_out_args(void *o, const void *v, const FwdOpts &oo) {
    return OutArgs{o, oo.dskip ? static_cast<const __nv_bfloat16 *>(v) : nullptr, oo.dskip, oo.bf16 ? 1 : 0,
                   oo.xnorm, oo.xw, oo.xeps};
}

// ---------------------------------------------------------------- row statistics
// A 64-row tile held by a warp with one column per lane (a[r] = this lane's value of row
// r): on exit a[0] and a[1] hold the warp's sums over its 32 columns of rows 2 lane and
// 2 lane + 1 (a transposing butterfly: each level keeps half of the rows and adds the
// partner lane's values of them, 62 shuffles in all).
template <int N>
__device__ __forceinline__ void fold_rows(float *a, bool up, int k) {
#pragma unroll
    for (int i = 0; i < N; ++i) {
        const float send = up ? a[i] : a[i + N];
        const float keep = up ? a[i + N] : a[i];
        a[i] = keep + __shfl_xor_sync(0xffffffffu, send, k);
    }
}
__device__ __forceinline__ void warp_row_sums(float (&a)[64]) {
    const int lane = threadIdx.x & 31;
    fold_rows<32>(a, lane & 16, 16);
    fold_rows<16>(a, lane & 8, 8);
    fold_rows<8>(a, lane & 4, 4);
    fold_rows<4>(a, lane & 2, 2);
    fold_rows<2>(a, lane & 1, 1);
}
__device__ __forceinline__ void group_bar(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Row sums over the 128 columns (4 warps) of a 64-row tile held by a 128-thread group
// (thread gt = column): red (4 x 64 floats of shared memory) takes the warp sums, and
// out[r] = post_mul * sum of row r for r < 64. The group meets twice on bar_id.
__device__ __forceinline__ void group_row_sums(float (&a)[64], int gt, int bar_id, float *red, float *out,
                                               float post_mul) {
    warp_row_sums(a);
    const int w = gt >> 5, l = gt & 31;
    red[w * 64 + 2 * l] = a[0];
    red[w * 64 + 2 * l + 1] = a[1];
    group_bar(bar_id, 128);
    if (gt < 64) out[gt] = (red[gt] + red[64 + gt] + red[128 + gt] + red[192 + gt]) * post_mul;
    group_bar(bar_id, 128);
}
// Output normalisation of a 64-row tile held by a 128-thread group, dv = 128 columns
// (thread gt = column, x[r] its value of row r): x[r] <- (x[r] - mean_r) w / sqrt(var_r +
// eps), with mean_r = 0 and var_r the mean square for the RMS form (two passes for the
// layer form: the mean first, then the mean square of the centred row). red: 4 x 64
// floats, stat: 2 x 64 floats of shared memory.
__device__ __forceinline__ void group_xnorm_128(float (&x)[64], int kind, float eps, float w, int gt, int bar_id,
                                                float *red, float *stat) {
    float t[64];
    if (kind == kXNormLayer) {
#pragma unroll
        for (int r = 0; r < 64; ++r) t[r] = x[r];
        group_row_sums(t, gt, bar_id, red, stat, 1.f / 128.f);
#pragma unroll
        for (int r = 0; r < 64; r += 4) {
            const float4 m = *reinterpret_cast<const float4 *>(stat + r);
            x[r] -= m.x; x[r + 1] -= m.y; x[r + 2] -= m.z; x[r + 3] -= m.w;
        }
    }
#pragma unroll
    for (int r = 0; r < 64; ++r) t[r] = x[r] * x[r];
    group_row_sums(t, gt, bar_id, red, stat + 64, 1.f / 128.f);
#pragma unroll
    for (int r = 0; r < 64; r += 4) {
        const float4 m = *reinterpret_cast<const float4 *>(stat + 64 + r);
        x[r] *= w * rsqrtf(m.x + eps);
        x[r + 1] *= w * rsqrtf(m.y + eps);
        x[r + 2] *= w * rsqrtf(m.z + eps);
        x[r + 3] *= w * rsqrtf(m.w + eps);
    }
}

// One value column of a 64-token output tile: stores ov[r] (r < n) at element offset
// elem0 + r * stride of o, in fp32 or rounded to bf16 (nearest, ties to even); with `probe`
// the stored values go through the non-finite probe nf (probe_tile).
__device__ __forceinline__ void store_out_rows_final(const float (&ov)[64], void *o, size_t elem0, int n, int stride,
                                                     bool bf16, bool probe, float &nf) {
    if (probe) probe_tile(nf, ov, n);
    if (bf16) {
        __nv_bfloat16 *ob = static_cast<__nv_bfloat16 *>(o) + elem0;
#pragma unroll
        for (int r = 0; r < 64; ++r)
            if (r < n) ob[static_cast<size_t>(r) * stride] = __float2bfloat16_rn(ov[r]);
    } else {
        float *of = static_cast<float *>(o) + elem0;
#pragma unroll
        for (int r = 0; r < 64; ++r)
            if (r < n) of[static_cast<size_t>(r) * stride] = ov[r];
    }
}
// The same for a 128-thread group holding the tile's 128 value columns (thread gt =
// column), with the output normalisation when out.xnorm is set. The whole group calls it
// (it meets on bar_id); red and stat are shared scratch of 256 and 128 floats. head
// indexes the (H, dv) weights of the skip term and of the normalisation.
__device__ __forceinline__ void store_out_rows_group(float (&ov)[64], const OutArgs &out, size_t elem0, int n,
                                                     int head, int gt, int bar_id, float *red, float *stat, bool probe,
                                                     float &nf) {
    if (out.v) {
        const float dj = out.dskip[head * 128 + gt];
#pragma unroll
        for (int r = 0; r < 64; ++r)
            if (r < n) ov[r] = fmaf(dj, __bfloat162float(out.v[elem0 + static_cast<size_t>(r) * 128]), ov[r]);
    }
    if (out.xnorm != kXNormNone)
        group_xnorm_128(ov, out.xnorm, out.xeps, out.xw ? out.xw[head * 128 + gt] : 1.f, gt, bar_id, red, stat);
    store_out_rows_final(ov, out.o, elem0, n, 128, out.bf16 != 0, probe, nf);
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
// Backward pass: floats of workspace it needs, and the launch (ws: that many floats).
size_t bwd_workspace_floats(long BH, int L, int dk, int dv, int chunk);
gdn_status_t launch_bwd(const void *q, const void *k, const void *v, const float *beta, const float *g,
                        const float *s0, const float *dout, const float *dsf, float *dq, float *dk, float *dv,
                        float *dbeta, float *dg, float *ds0, float *ws, int B, int H, int L, int dk_, int dv_,
                        int chunk, float scale, gdn_dtype_t in_dtype, cudaStream_t stream);
// Sequence-split prefill: s_out = ((lambda M + N) - N) / lambda s_in + N for `count` d x d
// states, and scaled identity states (value on the diagonal).
gdn_status_t launch_state_compose(const float *mn, const float *n, const float *s_in, float *s_out, float lambda,
                                  int count, int d, cudaStream_t stream);
gdn_status_t launch_state_identity(float *s, float value, int count, int d, cudaStream_t stream);
}  // namespace gdn
