// One-token recurrent decode step, state updated in place (HBM-streaming).
//
// Page "【CS336】lecture4 线性注意力|Mamba|GDN|DSA", sections "朴素线性注意力" and
// "继续改进：GDN": a decoded token costs O(d^2) because k^T S is formed first and
// the erase term (I - beta k k^T) is never materialised. With q' = scale q:
//   sk = S^T k,  sq = S^T q'                       (one pass over S)
//   u  = beta (v - alpha sk)    (u = v without the delta term)
//   o  = alpha sq + (q'.k) u    (= S_new^T q')
//   S <- alpha S + k u^T        (written back from registers)
// The state is read once and written once; everything else is O(d).
// With a vector-valued gate (alpha_t[j] per key row j) the decayed state diag(alpha) S
// replaces alpha S: sk = (diag(alpha) S)^T k, sq = (diag(alpha) S)^T q', o = sq + (q'.k) u,
// S <- diag(alpha) S + k u^T. The options variant also takes the skip term o += D_h v
// a bf16 output and the output normalisation of the prefill calls.
//
// Layout: one CTA per (sequence, head); thread t owns 4 consecutive value
// columns (float4) of RPT rows strided by the number of row groups, so every
// warp-wide access is a contiguous 256-512 B run of one or two state rows.
#include "common.cuh"
#include "tc_kernels.cuh"

namespace gdn {
namespace {

constexpr int kDecThreads = 256;

// OPT: the options variant (vector gate when vec, skip term when dskip, bf16 o when out_bf16)
template <int DK, int DV, typename IT, bool DELTA, bool OPT>
__global__ void __launch_bounds__(kDecThreads)
decode_step_kernel(const IT *__restrict__ q, const IT *__restrict__ k, const IT *__restrict__ v,
                   const float *__restrict__ beta, const float *__restrict__ g,
                   float *__restrict__ state, void *__restrict__ o, float scale, int H, int vec,
                   int out_bf16, const float *__restrict__ dskip, int xnorm, const float *__restrict__ xw,
                   float xeps, unsigned *__restrict__ err) {
    constexpr int CG = DV / 4;               // float4 column groups
    constexpr int RG = kDecThreads / CG;     // row groups
    constexpr int RPT = DK / RG;             // rows per thread
    static_assert(RPT >= 1 && RG * RPT == DK, "bad decode tiling");
    __shared__ float s_k[DK], s_q[DK], s_v[DV];
    __shared__ float red_k[DELTA ? RG : 1][DV];
    __shared__ float red_q[RG][DV];
    __shared__ float s_qk;
    __shared__ float s_a[OPT ? DK : 1];   // per-row decay (vector gate)
    const bool vg = OPT && vec;

    const long head = blockIdx.x;
    const int tid = threadIdx.x;
    const int cg = tid % CG, rg = tid / CG;
    float *S = state + head * (long)DK * DV;
    // extents the launch implies (bounds checks of the debug build)
    const long long nh = gridDim.x;

    // stream the state rows into registers first (independent 16 B loads)
    float4 sreg[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
        sreg[i] = in_bounds((head * DK + rg + RG * i) * (long long)DV + 4 * cg + 3, nh * DK * DV, err)
                      ? ld_global4(S + (long)(rg + RG * i) * DV + 4 * cg) : make_float4(0.f, 0.f, 0.f, 0.f);

    for (int i = tid; i < DK; i += kDecThreads) {
        const bool in = in_bounds(head * DK + i, nh * DK, err);
        s_k[i] = in ? ld_in(k + head * DK + i) : 0.f;
        s_q[i] = in ? scale * ld_in(q + head * DK + i) : 0.f;
    }
    for (int i = tid; i < DV; i += kDecThreads) s_v[i] = in_bounds(head * DV + i, nh * DV, err) ? ld_in(v + head * DV + i) : 0.f;
    if (vg)
        for (int i = tid; i < DK; i += kDecThreads)
            s_a[i] = g && in_bounds(head * DK + i, nh * DK, err) ? expf(g[head * DK + i]) : 1.f;
    const bool head_in = in_bounds(head, nh, err);
    const float alpha = (g && !vg && head_in) ? expf(g[head]) : 1.f;
    const float bt = DELTA && head_in ? beta[head] : 0.f;
    __syncthreads();

    // partial S^T k and S^T q' over this thread's rows
    float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int j = rg + RG * i;
        float kj = s_k[j], qj = s_q[j];
        if (vg) {           // read the decayed row alpha_j S[j, :]
            kj *= s_a[j];
            qj *= s_a[j];
        }
        if (DELTA) {
            pk.x = fmaf(sreg[i].x, kj, pk.x); pk.y = fmaf(sreg[i].y, kj, pk.y);
            pk.z = fmaf(sreg[i].z, kj, pk.z); pk.w = fmaf(sreg[i].w, kj, pk.w);
        }
        pq.x = fmaf(sreg[i].x, qj, pq.x); pq.y = fmaf(sreg[i].y, qj, pq.y);
        pq.z = fmaf(sreg[i].z, qj, pq.z); pq.w = fmaf(sreg[i].w, qj, pq.w);
    }
    if (DELTA) *reinterpret_cast<float4 *>(&red_k[rg][4 * cg]) = pk;
    *reinterpret_cast<float4 *>(&red_q[rg][4 * cg]) = pq;
    if (tid < 32) {
        float x = 0.f;
        for (int j = tid; j < DK; j += 32) x = fmaf(s_q[j], s_k[j], x);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
        if (tid == 0) s_qk = x;
    }
    __syncthreads();

    float sk[4] = {0.f, 0.f, 0.f, 0.f}, sq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < RG; ++r) {
        const float4 b = *reinterpret_cast<const float4 *>(&red_q[r][4 * cg]);
        sq[0] += b.x; sq[1] += b.y; sq[2] += b.z; sq[3] += b.w;
        if (DELTA) {
            const float4 a = *reinterpret_cast<const float4 *>(&red_k[r][4 * cg]);
            sk[0] += a.x; sk[1] += a.y; sk[2] += a.z; sk[3] += a.w;
        }
    }
    float u[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const float vc = s_v[4 * cg + c];
        u[c] = DELTA ? bt * (vc - alpha * sk[c]) : vc;   // alpha = 1 with a vector gate
    }
    if (rg == 0) {
        const float qk = s_qk;
        float4 ov;
        ov.x = fmaf(alpha, sq[0], qk * u[0]);
        ov.y = fmaf(alpha, sq[1], qk * u[1]);
        ov.z = fmaf(alpha, sq[2], qk * u[2]);
        ov.w = fmaf(alpha, sq[3], qk * u[3]);
        const bool o_in = in_bounds(head * DV + 4 * cg + 3, nh * DV, err);
        if (!OPT) {
            if (o_in) st_global4(static_cast<float *>(o) + head * DV + 4 * cg, ov);
        } else {
            if (dskip) {        // skip term D_h v (head = sequence * H + h)
                const float *dh = dskip + (head % H) * DV + 4 * cg;
                ov.x = fmaf(dh[0], s_v[4 * cg], ov.x);
                ov.y = fmaf(dh[1], s_v[4 * cg + 1], ov.y);
                ov.z = fmaf(dh[2], s_v[4 * cg + 2], ov.z);
                ov.w = fmaf(dh[3], s_v[4 * cg + 3], ov.w);
            }
            if (xnorm != kXNormNone) {
                // output normalisation over the DV outputs, held 4 per lane by lanes 0..CG-1
                constexpr unsigned mask = CG >= 32 ? 0xffffffffu : ((1u << CG) - 1u);
                float mean = 0.f;
                if (xnorm == kXNormLayer) {
                    float s1 = (ov.x + ov.y) + (ov.z + ov.w);
#pragma unroll
                    for (int off = CG / 2; off > 0; off >>= 1) s1 += __shfl_xor_sync(mask, s1, off);
                    mean = s1 * (1.f / DV);
                }
                ov.x -= mean; ov.y -= mean; ov.z -= mean; ov.w -= mean;
                float s2 = (ov.x * ov.x + ov.y * ov.y) + (ov.z * ov.z + ov.w * ov.w);
#pragma unroll
                for (int off = CG / 2; off > 0; off >>= 1) s2 += __shfl_xor_sync(mask, s2, off);
                const float rs = rsqrtf(s2 * (1.f / DV) + xeps);
                const float *wh = xw ? xw + (head % H) * DV + 4 * cg : nullptr;
                ov.x *= rs * (wh ? wh[0] : 1.f);
                ov.y *= rs * (wh ? wh[1] : 1.f);
                ov.z *= rs * (wh ? wh[2] : 1.f);
                ov.w *= rs * (wh ? wh[3] : 1.f);
            }
            if (o_in && out_bf16) {
                __nv_bfloat16 *ob = static_cast<__nv_bfloat16 *>(o) + head * DV + 4 * cg;
                ob[0] = __float2bfloat16_rn(ov.x);
                ob[1] = __float2bfloat16_rn(ov.y);
                ob[2] = __float2bfloat16_rn(ov.z);
                ob[3] = __float2bfloat16_rn(ov.w);
            } else if (o_in) {
                st_global4(static_cast<float *>(o) + head * DV + 4 * cg, ov);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int j = rg + RG * i;
        const float kj = s_k[j];
        const float aj = vg ? s_a[j] : alpha;
        float4 s = sreg[i];
        s.x = fmaf(aj, s.x, kj * u[0]);
        s.y = fmaf(aj, s.y, kj * u[1]);
        s.z = fmaf(aj, s.z, kj * u[2]);
        s.w = fmaf(aj, s.w, kj * u[3]);
        if (in_bounds((head * DK + j) * (long long)DV + 4 * cg + 3, nh * DK * DV, err)) st_global4(S + (long)j * DV + 4 * cg, s);
    }
}

template <int DK, int DV, typename IT, bool OPT>
gdn_status_t launch_dec_t(const void *q, const void *k, const void *v, const float *beta,
                          const float *g, float *state, void *o, long NH, int H, float scale, const FwdOpts &oo,
                          cudaStream_t stream) {
    const int vec = oo.gate_per_key ? 1 : 0, ob = oo.bf16 ? 1 : 0;
    unsigned *err = device_error_word();
    if (!err) return GDN_ERR_CUDA;
    if (beta)
        decode_step_kernel<DK, DV, IT, true, OPT><<<(unsigned)NH, kDecThreads, 0, stream>>>(
            (const IT *)q, (const IT *)k, (const IT *)v, beta, g, state, o, scale, H, vec, ob, oo.dskip, oo.xnorm,
            oo.xw, oo.xeps, err);
    else
        decode_step_kernel<DK, DV, IT, false, OPT><<<(unsigned)NH, kDecThreads, 0, stream>>>(
            (const IT *)q, (const IT *)k, (const IT *)v, beta, g, state, o, scale, H, vec, ob, oo.dskip, oo.xnorm,
            oo.xw, oo.xeps, err);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

template <typename IT, bool OPT>
gdn_status_t launch_dec_dt(const void *q, const void *k, const void *v, const float *beta,
                           const float *g, float *state, void *o, long NH, int H, int dk, int dv,
                           float scale, const FwdOpts &oo, cudaStream_t stream) {
    if (dk == 128 && dv == 128)
        return launch_dec_t<128, 128, IT, OPT>(q, k, v, beta, g, state, o, NH, H, scale, oo, stream);
    if (dk == 128 && dv == 64)
        return launch_dec_t<128, 64, IT, OPT>(q, k, v, beta, g, state, o, NH, H, scale, oo, stream);
    if (dk == 64 && dv == 128)
        return launch_dec_t<64, 128, IT, OPT>(q, k, v, beta, g, state, o, NH, H, scale, oo, stream);
    return launch_dec_t<64, 64, IT, OPT>(q, k, v, beta, g, state, o, NH, H, scale, oo, stream);
}

}  // namespace

gdn_status_t launch_decode(const void *q, const void *k, const void *v, const float *beta,
                           const float *g, float *state, void *o, int N, int H, int dk, int dv,
                           float scale, gdn_dtype_t in_dtype, FwdOpts oo, cudaStream_t stream) {
    const long NH = (long)N * H;
    const bool opt = oo.bf16 || oo.dskip || oo.gate_per_key || oo.xnorm != kXNormNone;
    if (in_dtype == GDN_F32)
        return opt ? launch_dec_dt<float, true>(q, k, v, beta, g, state, o, NH, H, dk, dv, scale, oo, stream)
                   : launch_dec_dt<float, false>(q, k, v, beta, g, state, o, NH, H, dk, dv, scale, oo, stream);
    return opt ? launch_dec_dt<__nv_bfloat16, true>(q, k, v, beta, g, state, o, NH, H, dk, dv, scale, oo, stream)
               : launch_dec_dt<__nv_bfloat16, false>(q, k, v, beta, g, state, o, NH, H, dk, dv, scale, oo, stream);
}

}  // namespace gdn
