// Backward pass of the operator (gradients for training on full sequences): plain /
// gated linear attention, DeltaNet and Gated DeltaNet, fp32 CUDA-core arithmetic.
//
// Page "混合注意力学习(1)", section "Transformers 就是 RNNs": on the full training sequence
// every gradient follows from the chain rule through the recurrence. Per head, with the
// state S (dk x dv, key rows), alpha_t = exp(g_t), q'_t = scale q_t:
//   forward   u_t = beta_t (v_t - alpha_t S_{t-1}^T k_t),  S_t = alpha_t S_{t-1} + k_t u_t^T,
//             o_t = S_t^T q'_t   (u_t = v_t without the delta term)
// the adjoint Lambda_t = dLoss/dS_t runs backwards from Lambda_L = dS_final:
//   Lambda_t += q'_t do_t^T;   dq_t = scale S_t do_t
//   du = Lambda_t^T k_t;       dv_t = beta_t du            (dv_t = du without beta)
//   dk_t = Lambda_t u_t - alpha_t beta_t S_{t-1} du
//   dbeta_t = du . (v_t - alpha_t S_{t-1}^T k_t)
//   dalpha_t = <Lambda_t, S_{t-1}> - beta_t du . (S_{t-1}^T k_t);   dg_t = alpha_t dalpha_t
//   Lambda_{t-1} = alpha_t (Lambda_t - beta_t k_t du^T)
// and dS_0 = Lambda_0. S_{t-1} is needed for every t in reverse order: a forward pass
// stores the state at the start of every chunk of C tokens (checkpoints); the reverse
// pass, chunk by chunk from the last, recomputes the states inside the chunk from its
// checkpoint into a slab of C states and walks its tokens backwards. Both live in the
// caller's workspace (gdn_chunk_bwd_workspace_bytes).
//
// Layout: one CTA per (sequence, head), 256 threads; thread t owns 4 consecutive value
// columns (float4) of RPT key rows strided by the number of row groups (the decode
// step's tiling), for S and for Lambda alike; row reductions are warp shuffles over the
// column groups of a row group, column reductions go through shared memory.
#include <mutex>

#include "common.cuh"

namespace gdn {
namespace {

constexpr int kBwdThreads = 256;

template <int DK, int DV, typename IT, bool DELTA, bool GATED>
__global__ void __launch_bounds__(kBwdThreads)
gdn_bwd_kernel(const IT *__restrict__ q, const IT *__restrict__ k, const IT *__restrict__ v,
               const float *__restrict__ beta, const float *__restrict__ g, const float *__restrict__ s0,
               const float *__restrict__ dout, const float *__restrict__ dsf, float *__restrict__ dq,
               float *__restrict__ dk, float *__restrict__ dv, float *__restrict__ dbeta,
               float *__restrict__ dg, float *__restrict__ ds0, float *__restrict__ ws, int L, int C,
               float scale) {
    constexpr int CG = DV / 4;               // float4 column groups (a row group's threads)
    constexpr int RG = kBwdThreads / CG;     // row groups
    constexpr int RPT = DK / RG;             // rows per thread
    static_assert(RPT >= 1 && RG * RPT == DK && CG <= 32 && 32 % CG == 0, "bad tiling");
    __shared__ float s_q[DK], s_k[DK], s_v[DV], s_do[DV], s_u[DV], s_du[DV], s_sk[DV];
    __shared__ float red[RG][DV];
    __shared__ float red_s[2][kBwdThreads / 32];

    const long bh = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int cg = tid % CG, rg = tid / CG;
    const int nck = (L + C - 1) / C;
    float *ckpt = ws + bh * static_cast<long>(nck + C) * DK * DV;   // nck checkpoints, then C slab states
    float *slab = ckpt + static_cast<long>(nck) * DK * DV;
    const long tok0 = bh * static_cast<long>(L);                  // first token of this head
    auto elem = [&](int i) { return static_cast<long>(rg + RG * i) * DV + 4 * cg; };   // this thread's float4

    float4 S[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
        S[i] = s0 ? *reinterpret_cast<const float4 *>(s0 + bh * DK * DV + elem(i)) : make_float4(0.f, 0.f, 0.f, 0.f);

    // loads token t's q', k, v (and do) into shared memory; alpha, beta into registers
    auto load_token = [&](long t, bool with_do, float &alpha, float &bt) {
        for (int i = tid; i < DK; i += kBwdThreads) {
            s_k[i] = ld_in(k + t * DK + i);
            s_q[i] = scale * ld_in(q + t * DK + i);
        }
        for (int i = tid; i < DV; i += kBwdThreads) {
            s_v[i] = ld_in(v + t * DV + i);
            if (with_do) s_do[i] = dout[t * DV + i];
        }
        alpha = GATED ? expf(g[t]) : 1.f;
        bt = DELTA ? beta[t] : 1.f;
    };
    // column sums over the key rows: x[c] (4 per thread) summed over all rows -> out[c]
    auto col_sum = [&](const float (&x)[4], float *out) {
        *reinterpret_cast<float4 *>(&red[rg][4 * cg]) = make_float4(x[0], x[1], x[2], x[3]);
        __syncthreads();
        for (int c = tid; c < DV; c += kBwdThreads) {
            float s = 0.f;
#pragma unroll
            for (int r = 0; r < RG; ++r) s += red[r][c];
            out[c] = s;
        }
        __syncthreads();
    };
    // sum over the CG column-group threads of a row group (a warp or half a warp)
    auto row_sum = [&](float x) {
#pragma unroll
        for (int off = CG / 2; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
        return x;
    };
    // sum over the whole block of two scalars -> both returned to every thread
    auto block_sum2 = [&](float a, float b, float &ra, float &rb) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            a += __shfl_xor_sync(0xffffffffu, a, off);
            b += __shfl_xor_sync(0xffffffffu, b, off);
        }
        if (lane == 0) { red_s[0][wid] = a; red_s[1][wid] = b; }
        __syncthreads();
        ra = 0.f;
        rb = 0.f;
#pragma unroll
        for (int w = 0; w < kBwdThreads / 32; ++w) { ra += red_s[0][w]; rb += red_s[1][w]; }
        __syncthreads();
    };
    // one forward token step on the registers S (the state before the token -> after it);
    // leaves S^T k in s_sk and u in s_u
    auto fwd_step = [&](float alpha, float bt) {
        float pk[4] = {0.f, 0.f, 0.f, 0.f};
        if (DELTA) {
#pragma unroll
            for (int i = 0; i < RPT; ++i) {
                const float kj = s_k[rg + RG * i];
                pk[0] = fmaf(S[i].x, kj, pk[0]); pk[1] = fmaf(S[i].y, kj, pk[1]);
                pk[2] = fmaf(S[i].z, kj, pk[2]); pk[3] = fmaf(S[i].w, kj, pk[3]);
            }
            col_sum(pk, s_sk);
        }
        for (int c = tid; c < DV; c += kBwdThreads) s_u[c] = DELTA ? bt * (s_v[c] - alpha * s_sk[c]) : s_v[c];
        __syncthreads();
        const float4 u = *reinterpret_cast<const float4 *>(&s_u[4 * cg]);
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const float kj = s_k[rg + RG * i];
            S[i].x = fmaf(alpha, S[i].x, kj * u.x); S[i].y = fmaf(alpha, S[i].y, kj * u.y);
            S[i].z = fmaf(alpha, S[i].z, kj * u.z); S[i].w = fmaf(alpha, S[i].w, kj * u.w);
        }
    };

    // ---- forward pass: the state at the start of every chunk -> checkpoints
    for (int t = 0; t < L; ++t) {
        if (t % C == 0) {
            float *dst = ckpt + static_cast<long>(t / C) * DK * DV;
#pragma unroll
            for (int i = 0; i < RPT; ++i) *reinterpret_cast<float4 *>(dst + elem(i)) = S[i];
        }
        float alpha, bt;
        __syncthreads();
        load_token(tok0 + t, false, alpha, bt);
        __syncthreads();
        fwd_step(alpha, bt);
    }

    // ---- reverse pass
    float4 Lm[RPT];   // the adjoint Lambda, same tiling as S
#pragma unroll
    for (int i = 0; i < RPT; ++i)
        Lm[i] = dsf ? *reinterpret_cast<const float4 *>(dsf + bh * DK * DV + elem(i)) : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = nck - 1; c >= 0; --c) {
        const int t0 = c * C, n = min(C, L - t0);
        // recompute the states before each token of the chunk into the slab
        {
            const float *src = ckpt + static_cast<long>(c) * DK * DV;
#pragma unroll
            for (int i = 0; i < RPT; ++i) S[i] = *reinterpret_cast<const float4 *>(src + elem(i));
        }
        for (int i = 0; i < n; ++i) {
            float *dst = slab + static_cast<long>(i) * DK * DV;
#pragma unroll
            for (int r = 0; r < RPT; ++r) *reinterpret_cast<float4 *>(dst + elem(r)) = S[r];
            if (i + 1 == n) break;   // the state after the last token is not needed
            float alpha, bt;
            __syncthreads();
            load_token(tok0 + t0 + i, false, alpha, bt);
            __syncthreads();
            fwd_step(alpha, bt);
        }
        // walk the chunk's tokens backwards
        for (int i = n - 1; i >= 0; --i) {
            const long t = tok0 + t0 + i;
            float alpha, bt;
            __syncthreads();
            load_token(t, true, alpha, bt);
            {
                const float *src = slab + static_cast<long>(i) * DK * DV;
#pragma unroll
                for (int r = 0; r < RPT; ++r) S[r] = *reinterpret_cast<const float4 *>(src + elem(r));
            }
            __syncthreads();
            // Lambda_t += q' do^T; du = Lambda_t^T k (neither needs S_t)
            const float4 dov = *reinterpret_cast<const float4 *>(&s_do[4 * cg]);
            {
                float pd[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const int j = rg + RG * r;
                    const float qj = s_q[j], kj = s_k[j];
                    Lm[r].x = fmaf(qj, dov.x, Lm[r].x); Lm[r].y = fmaf(qj, dov.y, Lm[r].y);
                    Lm[r].z = fmaf(qj, dov.z, Lm[r].z); Lm[r].w = fmaf(qj, dov.w, Lm[r].w);
                    pd[0] = fmaf(Lm[r].x, kj, pd[0]); pd[1] = fmaf(Lm[r].y, kj, pd[1]);
                    pd[2] = fmaf(Lm[r].z, kj, pd[2]); pd[3] = fmaf(Lm[r].w, kj, pd[3]);
                }
                col_sum(pd, s_du);
            }
            const float4 du = *reinterpret_cast<const float4 *>(&s_du[4 * cg]);
            // with S = S_{t-1}: the rows of S_{t-1} du and <Lambda_t, S_{t-1}>
            float sdu[RPT];
            float lsp = 0.f;
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                sdu[r] = DELTA ? row_sum(S[r].x * du.x + S[r].y * du.y + S[r].z * du.z + S[r].w * du.w) : 0.f;
                if (GATED) lsp += Lm[r].x * S[r].x + Lm[r].y * S[r].y + Lm[r].z * S[r].z + Lm[r].w * S[r].w;
            }
            fwd_step(alpha, bt);   // S <- S_t; s_sk = S_{t-1}^T k; s_u = u_t
            // dq_t = scale S_t do_t;  dk_t = Lambda_t u - alpha beta S_{t-1} du
            const float4 u = *reinterpret_cast<const float4 *>(&s_u[4 * cg]);
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const int j = rg + RG * r;
                const float xq = row_sum(S[r].x * dov.x + S[r].y * dov.y + S[r].z * dov.z + S[r].w * dov.w);
                const float xk = row_sum(Lm[r].x * u.x + Lm[r].y * u.y + Lm[r].z * u.z + Lm[r].w * u.w);
                if (cg == 0) {
                    dq[t * DK + j] = scale * xq;
                    dk[t * DK + j] = DELTA ? xk - alpha * bt * sdu[r] : xk;
                }
            }
            // dv_t, dbeta_t, dalpha_t
            float pb = 0.f, pa = 0.f;
            if (cg + rg * CG < CG) {   // row group 0 holds each column once
                const float4 vv = *reinterpret_cast<const float4 *>(&s_v[4 * cg]);
                const float4 sk = *reinterpret_cast<const float4 *>(&s_sk[4 * cg]);
                float4 dvo = du;
                if (DELTA) {
                    dvo = make_float4(bt * du.x, bt * du.y, bt * du.z, bt * du.w);
                    pb = du.x * (vv.x - alpha * sk.x) + du.y * (vv.y - alpha * sk.y) + du.z * (vv.z - alpha * sk.z) +
                         du.w * (vv.w - alpha * sk.w);
                    pa = -bt * (du.x * sk.x + du.y * sk.y + du.z * sk.z + du.w * sk.w);
                }
                *reinterpret_cast<float4 *>(dv + t * DV + 4 * cg) = dvo;
            }
            if (DELTA || GATED) {
                float sb, sa;
                block_sum2(pb, pa + lsp, sb, sa);
                if (tid == 0) {
                    if (DELTA) dbeta[t] = sb;
                    if (GATED) dg[t] = alpha * sa;
                }
            }
            // Lambda_{t-1} = alpha (Lambda_t - beta k du^T)
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const float kb = DELTA ? bt * s_k[rg + RG * r] : 0.f;
                Lm[r].x = alpha * (Lm[r].x - kb * du.x); Lm[r].y = alpha * (Lm[r].y - kb * du.y);
                Lm[r].z = alpha * (Lm[r].z - kb * du.z); Lm[r].w = alpha * (Lm[r].w - kb * du.w);
            }
        }
    }
    if (ds0) {
#pragma unroll
        for (int i = 0; i < RPT; ++i) *reinterpret_cast<float4 *>(ds0 + bh * DK * DV + elem(i)) = Lm[i];
    }
}

template <int DK, int DV, typename IT>
gdn_status_t launch_bwd_t(const void *q, const void *k, const void *v, const float *beta, const float *g,
                          const float *s0, const float *dout, const float *dsf, float *dq, float *dk, float *dv,
                          float *dbeta, float *dg, float *ds0, float *ws, int BH, int L, int C, float scale,
                          cudaStream_t stream) {
    const IT *q_ = static_cast<const IT *>(q), *k_ = static_cast<const IT *>(k), *v_ = static_cast<const IT *>(v);
#define GDN_BWD_LAUNCH(D, G)                                                                                   \
    gdn_bwd_kernel<DK, DV, IT, D, G><<<BH, kBwdThreads, 0, stream>>>(q_, k_, v_, beta, g, s0, dout, dsf, dq, dk, dv, \
                                                                    dbeta, dg, ds0, ws, L, C, scale)
    if (beta && g) GDN_BWD_LAUNCH(true, true);
    else if (beta) GDN_BWD_LAUNCH(true, false);
    else if (g) GDN_BWD_LAUNCH(false, true);
    else GDN_BWD_LAUNCH(false, false);
#undef GDN_BWD_LAUNCH
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

template <typename IT>
gdn_status_t launch_bwd_dt(const void *q, const void *k, const void *v, const float *beta, const float *g,
                           const float *s0, const float *dout, const float *dsf, float *dq, float *dk, float *dv,
                           float *dbeta, float *dg, float *ds0, float *ws, int BH, int L, int dk_, int dv_, int C,
                           float scale, cudaStream_t stream) {
    if (dk_ == 128 && dv_ == 128)
        return launch_bwd_t<128, 128, IT>(q, k, v, beta, g, s0, dout, dsf, dq, dk, dv, dbeta, dg, ds0, ws, BH, L, C,
                                          scale, stream);
    if (dk_ == 128 && dv_ == 64)
        return launch_bwd_t<128, 64, IT>(q, k, v, beta, g, s0, dout, dsf, dq, dk, dv, dbeta, dg, ds0, ws, BH, L, C,
                                         scale, stream);
    if (dk_ == 64 && dv_ == 128)
        return launch_bwd_t<64, 128, IT>(q, k, v, beta, g, s0, dout, dsf, dq, dk, dv, dbeta, dg, ds0, ws, BH, L, C,
                                         scale, stream);
    return launch_bwd_t<64, 64, IT>(q, k, v, beta, g, s0, dout, dsf, dq, dk, dv, dbeta, dg, ds0, ws, BH, L, C, scale,
                                    stream);
}

}  // namespace

size_t bwd_workspace_floats(long BH, int L, int dk, int dv, int chunk) {
    const long nck = (L + chunk - 1) / chunk;
    return static_cast<size_t>(BH) * static_cast<size_t>(nck + chunk) * static_cast<size_t>(dk) * dv;
}

gdn_status_t launch_bwd(const void *q, const void *k, const void *v, const float *beta, const float *g,
                        const float *s0, const float *dout, const float *dsf, float *dq, float *dk, float *dv,
                        float *dbeta, float *dg, float *ds0, float *ws, int B, int H, int L, int dk_, int dv_,
                        int chunk, float scale, gdn_dtype_t in_dtype, cudaStream_t stream) {
    const int BH = B * H;
    if (in_dtype == GDN_F32)
        return launch_bwd_dt<float>(q, k, v, beta, g, s0, dout, dsf, dq, dk, dv, dbeta, dg, ds0, ws, BH, L, dk_, dv_,
                                    chunk, scale, stream);
    return launch_bwd_dt<__nv_bfloat16>(q, k, v, beta, g, s0, dout, dsf, dq, dk, dv, dbeta, dg, ds0, ws, BH, L, dk_,
                                        dv_, chunk, scale, stream);
}

// ---------------------------------------------------------------- no-allocation variant
// Workspace of gdn_chunk_bwd_noalloc: one fixed array in the library's static device memory.
// Every device that loads the library holds it until the process exits; every call of the
// entry point on a device shares it.
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB
static __device__ __align__(256) float g_bwd_scratch[kNoAllocScratchBytes / sizeof(float)];

// Device address of g_bwd_scratch on the current device, looked up once per device (with
// that device current); nullptr if the lookup fails. In host code the array's name is only a
// host-side stand-in, so kernels must be given this address, never the name.
float *bwd_scratch_address() {
    static std::mutex mu;
    static float *addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || p == nullptr) return nullptr;
        addr[dev] = static_cast<float *>(p);
    }
    return addr[dev];
}
}  // namespace

}  // namespace gdn

extern "C" gdn_status_t gdn_chunk_bwd_noalloc(const void *q, const void *k, const void *v, const float *beta,
                                              const float *g, const float *s0, const float *d_o,
                                              const float *ds_final, float *dq, float *dk, float *dv,
                                              float *dbeta, float *dg, float *ds0, int B, int H, int L,
                                              int dk_size, int dv_size, int chunk, float scale,
                                              gdn_dtype_t in_dtype, void *cuda_stream) {
    const size_t need = gdn_chunk_bwd_workspace_bytes(B, H, L, dk_size, dv_size, chunk);
    if (need == 0) return gdn_chunk_bwd(q, k, v, beta, g, s0, d_o, ds_final, dq, dk, dv, dbeta, dg, ds0, nullptr, 0,
                                        B, H, L, dk_size, dv_size, chunk, scale, in_dtype, cuda_stream);
    if (need > gdn::kNoAllocScratchBytes) return GDN_ERR_UNSUPPORTED;
    float *ws = gdn::bwd_scratch_address();
    if (!ws) return GDN_ERR_CUDA;
    return gdn_chunk_bwd(q, k, v, beta, g, s0, d_o, ds_final, dq, dk, dv, dbeta, dg, ds0, ws, gdn::kNoAllocScratchBytes,
                         B, H, L, dk_size, dv_size, chunk, scale, in_dtype, cuda_stream);
}
