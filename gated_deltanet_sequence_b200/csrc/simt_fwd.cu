// SIMT (fp32 CUDA-core) chunkwise prefill for plain / gated linear attention,
// DeltaNet and Gated DeltaNet. It serves fp32 inputs (where fp32 arithmetic is
// needed to meet a 1e-5 tolerance), head sizes 64, and chunk sizes other than
// 64; bf16 inputs with dk = dv = 128 and chunk 64 take the tcgen05 kernel.
//
// One CTA owns one (batch, head) and a 32-wide slice of the value columns:
// the state's value columns evolve independently (column c of S only ever
// mixes with column c of V), so slices need no communication. Per chunk of n
// rows (page "混合注意力学习(1)", sections "FWP分块并行机制" and "DeltaNet 分块并行机制";
// page "LinearAttention 概述", section "FLASH": the chunk form is exact):
//   G = within-chunk cumsum(g); gamma = exp(G); Gamma_rs = exp(G_r - G_s), s <= r
//   A_rs = beta_r Gamma_rs k_r.k_s (s < r);  T = (I + A)^-1 (forward substitution)
//   W = T diag(beta gamma) K;  Ut = T diag(beta) V - W S    (Ut = V without delta)
//   O = diag(gamma) Q S + (Q K^T o Gamma) Ut
//   S <- gamma_n S + sum_s exp(G_n - G_s) k_s Ut_s^T
// Vector-valued gates (one log-decay per key coordinate; row j of S decays by
// exp(g_t[j])) give the same steps with a decay per key coordinate: G_r[j] is the
// cumulative sum per coordinate, the masks become A_rs = beta_r sum_j k_r[j] k_s[j]
// exp(G_r[j] - G_s[j]) and P_rs = sum_j q_r[j] k_s[j] exp(G_r[j] - G_s[j]), W =
// T diag(beta) (K o exp(G)), the inter-chunk output uses Q o exp(G), and the state
// update uses k_s o exp(G_n - G_s) with row j of S scaled by exp(G_n[j]). Every decay
// factor is one exp of a difference of cumulative sums, so no decay strength overflows.
// Chunks whose cumulative log-decays all lie in [-60, 60] take the factored form
// exp(G_r - G_s) = exp(G_r) exp(-G_s) (both factors far inside fp32 range): Q, K and
// beta-free W are pre-scaled per element and the masks become plain dot products.
#include "common.cuh"
#include "tc_kernels.cuh"

namespace gdn {
namespace {

constexpr int kSimtThreads = 1024;   // one CTA per SM (the tiles take 215 KB of shared memory): all warps in one block
constexpr int kDvs = 32;      // value columns per CTA
constexpr int kCmax = 64;     // largest supported chunk

template <int DK, bool VEC, bool XN>
struct SimtSmem {
    static constexpr int KP = DK + 1;            // padded row pitch for K, Q, W
    static constexpr int CP = kCmax + 1;         // padded row pitch for A, T, P
    float K[kCmax * KP];
    float Q[kCmax * KP];
    float W[kCmax * KP];
    float V[kCmax * kDvs];
    float U[kCmax * kDvs];
    float S[DK * kDvs];
    float A[kCmax * CP];
    float T[kCmax * CP];
    float P[kCmax * CP];
    float G[kCmax];
    float bt[kCmax];
    float GV[VEC ? kCmax * KP : 1];              // per-key cumulative log-decay (vector gates)
    float Ob[XN ? kCmax * kDvs : 1];             // output tile before the normalisation
    float part[XN ? 2 * kCmax : 1];              // this CTA's row sums, by reduction-round parity
};

// Sum over the cluster's CTAs (the dv / 32 value slices of one head) of x, one value per
// output row r < n: each CTA leaves its row sums in its part[] buffer of this round's parity,
// the cluster meets once, and every CTA adds all buffers through distributed shared
// memory. Double buffering by round parity keeps a buffer untouched until every CTA has
// passed the next round's barrier, i.e. has finished reading it.
__device__ __forceinline__ float cluster_row_sum(float *part, int round, int r, float x, bool writer, int nslices) {
    float *buf = part + (round & 1) * kCmax;
    if (writer) buf[r] = x;
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    float total = 0.f;
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(buf + r));
    for (int rank = 0; rank < nslices; ++rank) {
        uint32_t ra;
        float y;
        asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
        asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(y) : "r"(ra) : "memory");
        total += y;
    }
    return total;
}

template <int DK, typename IT, bool DELTA, bool VEC, bool XN>
__global__ void __launch_bounds__(kSimtThreads)
simt_chunk_fwd_kernel(const IT *__restrict__ q, const IT *__restrict__ k, const IT *__restrict__ v,
                      const float *__restrict__ beta, const float *__restrict__ g,
                      void *__restrict__ o, int out_bf16, const float *__restrict__ dskip,
                      int xnorm, const float *__restrict__ xw, float xeps,
                      const float *__restrict__ s0,
                      float *__restrict__ s_final, const int *__restrict__ cu, int H, int Lrow,
                      int dv, int C, float scale, unsigned *__restrict__ err) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    using Sm = SimtSmem<DK, VEC, XN>;
    Sm &sm = *reinterpret_cast<Sm *>(smem_raw);
    constexpr int KP = Sm::KP, CP = Sm::CP;
    const int tid = threadIdx.x;
    // (sequence, head): state index; packed batches take their sequences longest first
    const long bh = cu ? longest_first(cu, static_cast<int>(blockIdx.x), H, static_cast<int>(gridDim.x) / H)
                       : static_cast<long>(blockIdx.x);
    const int c0 = blockIdx.y * kDvs;            // first value column of this CTA
    const SeqSpan sp = seq_span(cu, static_cast<int>(bh), H, Lrow, err);
    const int L = sp.len;                        // tokens of this sequence
    const long r0 = (long)sp.head_row * Lrow + sp.t0;   // its first row in the token grid

    const IT *qh = q + r0 * DK;
    const IT *kh = k + r0 * DK;
    const IT *vh = v + r0 * dv;
    const float *bh_beta = DELTA ? beta + r0 : nullptr;
    const float *bh_g = (g && !VEC) ? g + r0 : nullptr;
    const float *bh_gv = (g && VEC) ? g + r0 * DK : nullptr;   // (L, DK) log-decays per key
    const long o0 = r0 * dv;                     // first output element of the sequence
    // extents the launch implies (bounds checks of the debug build): token rows of the grid, and
    // state elements
    const long long n_rows = static_cast<long long>(cu ? H : gridDim.x) * Lrow;
    const long long n_state = static_cast<long long>(gridDim.x) * DK * dv;
    const float *dsk = dskip ? dskip + static_cast<long>(sp.head_row % H) * dv + c0 : nullptr;

    for (int i = tid; i < DK * kDvs; i += kSimtThreads) {
        const int j = i / kDvs, c = i % kDvs;
        sm.S[i] = s0 && in_bounds((bh * DK + j) * dv + c0 + c, n_state, err) ? s0[(bh * DK + j) * dv + c0 + c] : 0.f;
    }

    int round = 0;   // reduction rounds across the cluster (output normalisation)
    for (int t0 = 0; t0 < L; t0 += C) {
        const int n = min(C, L - t0);
        __syncthreads();
        // ---- load the chunk ------------------------------------------------
        for (int i = tid; i < n * DK; i += kSimtThreads) {
            const int r = i / DK, j = i % DK;
            const bool in = in_bounds((r0 + t0 + r) * DK + j, n_rows * DK, err);
            sm.K[r * KP + j] = in ? ld_in(kh + (long)(t0 + r) * DK + j) : 0.f;
            sm.Q[r * KP + j] = in ? scale * ld_in(qh + (long)(t0 + r) * DK + j) : 0.f;
        }
        for (int i = tid; i < n * kDvs; i += kSimtThreads) {
            const int r = i / kDvs, c = i % kDvs;
            sm.V[i] = in_bounds((r0 + t0 + r) * dv + c0 + c, n_rows * dv, err) ? ld_in(vh + (long)(t0 + r) * dv + c0 + c) : 0.f;
        }
        int wide = 0;   // a cumulative log-decay of this chunk is outside [-60, 60]
        if (VEC) {
            // the chunk's log-decays (n x DK, coalesced), then per key coordinate j the
            // inclusive within-chunk cumulative sum of g[:, j], in place
            for (int i = tid; i < n * DK; i += kSimtThreads) {
                const int r = i / DK, j = i % DK;
                sm.GV[r * KP + j] = bh_gv && in_bounds((r0 + t0 + r) * DK + j, n_rows * DK, err)
                                        ? bh_gv[(long)(t0 + r) * DK + j] : 0.f;
            }
            __syncthreads();
            if (tid < DK) {
                float carry = 0.f;
                for (int r = 0; r < n; ++r) {
                    carry += sm.GV[r * KP + tid];
                    sm.GV[r * KP + tid] = carry;
                    wide |= !(fabsf(carry) <= 60.f);
                }
            }
        }
        if (!VEC && tid < 32) {
            // inclusive within-chunk cumulative sum of g (warp scan, two passes of 32)
            float carry = 0.f;
            for (int base = 0; base < n; base += 32) {
                const int r = base + tid;
                float x = (bh_g && r < n && in_bounds(r0 + t0 + r, n_rows, err)) ? bh_g[t0 + r] : 0.f;
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, x, off);
                    if (tid >= off) x += y;
                }
                if (r < n) sm.G[r] = carry + x;
                carry += __shfl_sync(0xffffffffu, x, 31);
            }
        } else if (DELTA && tid >= 64 && tid < 64 + kCmax) {
            const int r = tid - 64;
            if (r < n) sm.bt[r] = in_bounds(r0 + t0 + r, n_rows, err) ? bh_beta[t0 + r] : 0.f;
        }
        const bool direct = VEC && __syncthreads_or(wide);   // VEC: direct exp per decay factor
        if (!VEC) __syncthreads();
        if (VEC && !direct) {
            // factored decays: Q <- Q o exp(G), K <- K o exp(-G), W <- K o exp(G) (delta term)
            for (int i = tid; i < n * DK; i += kSimtThreads) {
                const int r = i / DK, j = i % DK;
                const float gr = sm.GV[r * KP + j], kv = sm.K[r * KP + j];
                const float e = expf(gr);
                sm.Q[r * KP + j] *= e;
                sm.K[r * KP + j] = kv * expf(-gr);
                if (DELTA) sm.W[r * KP + j] = kv * e;
            }
            __syncthreads();
        }
        // ---- Gram products with the decay mask ---------------------------------
        for (int i = tid; i < n * n; i += kSimtThreads) {
            const int r = i / n, s = i % n;
            float p = 0.f, a = 0.f;
            if (s <= r && VEC && !direct) {
#pragma unroll 8
                for (int j = 0; j < DK; ++j) {
                    p = fmaf(sm.Q[r * KP + j], sm.K[s * KP + j], p);
                    if (DELTA) a = fmaf(sm.W[r * KP + j], sm.K[s * KP + j], a);
                }
                if (DELTA) a = (s < r) ? sm.bt[r] * a : 0.f;
            } else if (s <= r && VEC) {
#pragma unroll 4
                for (int j = 0; j < DK; ++j) {
                    const float dec = expf(sm.GV[r * KP + j] - sm.GV[s * KP + j]);
                    const float ks = dec * sm.K[s * KP + j];
                    p = fmaf(sm.Q[r * KP + j], ks, p);
                    if (DELTA) a = fmaf(sm.K[r * KP + j], ks, a);
                }
                if (DELTA) a = (s < r) ? sm.bt[r] * a : 0.f;
            } else if (s <= r) {
                const float dec = expf(sm.G[r] - sm.G[s]);
#pragma unroll 8
                for (int j = 0; j < DK; ++j) {
                    p = fmaf(sm.Q[r * KP + j], sm.K[s * KP + j], p);
                    if (DELTA) a = fmaf(sm.K[r * KP + j], sm.K[s * KP + j], a);
                }
                p *= dec;
                if (DELTA) a = (s < r) ? sm.bt[r] * dec * a : 0.f;
            }
            sm.P[r * CP + s] = p;
            if (DELTA) sm.A[r * CP + s] = a;
        }
        __syncthreads();
        if (DELTA) {
            // ---- T = (I + A)^-1: thread j solves column j by forward substitution
            if (tid < n) {
                const int jc = tid;
                for (int r = 0; r < n; ++r) {
                    float x = (r == jc) ? 1.f : 0.f;
                    for (int s = jc; s < r; ++s) x = fmaf(-sm.A[r * CP + s], sm.T[s * CP + jc], x);
                    sm.T[r * CP + jc] = (r < jc) ? 0.f : x;
                }
            }
            __syncthreads();
            // ---- W = T diag(beta gamma) K ;  U = T diag(beta) V ----------------------
            if (VEC) {
                // thread per key column j: W[:, j] = T (beta o exp(G[:, j]) o K[:, j]), formed
                // in place from the last row up (row r reads rows s <= r only)
                for (int j = tid; j < DK; j += kSimtThreads) {
                    for (int s = 0; s < n; ++s)   // factored chunks: W already holds K o exp(G)
                        sm.W[s * KP + j] = sm.bt[s] * (direct ? expf(sm.GV[s * KP + j]) * sm.K[s * KP + j]
                                                              : sm.W[s * KP + j]);
                    for (int r = n - 1; r >= 0; --r) {
                        float w = 0.f;
                        for (int s = 0; s <= r; ++s) w = fmaf(sm.T[r * CP + s], sm.W[s * KP + j], w);
                        sm.W[r * KP + j] = w;
                    }
                }
            } else {
                for (int i = tid; i < n * DK; i += kSimtThreads) {
                    const int r = i / DK, j = i % DK;
                    float w = 0.f;
                    for (int s = 0; s <= r; ++s)
                        w = fmaf(sm.T[r * CP + s] * sm.bt[s] * expf(sm.G[s]), sm.K[s * KP + j], w);
                    sm.W[r * KP + j] = w;
                }
            }
            for (int i = tid; i < n * kDvs; i += kSimtThreads) {
                const int r = i / kDvs, c = i % kDvs;
                float u = 0.f;
                for (int s = 0; s <= r; ++s) u = fmaf(sm.T[r * CP + s] * sm.bt[s], sm.V[s * kDvs + c], u);
                sm.U[i] = u;
            }
            __syncthreads();
            // ---- Ut = U - W S ----------------------------------------------------------
            for (int i = tid; i < n * kDvs; i += kSimtThreads) {
                const int r = i / kDvs, c = i % kDvs;
                float ws = 0.f;
#pragma unroll 8
                for (int j = 0; j < DK; ++j) ws = fmaf(sm.W[r * KP + j], sm.S[j * kDvs + c], ws);
                sm.U[i] -= ws;
            }
            __syncthreads();
        }
        const float *Ut = DELTA ? sm.U : sm.V;
        if (VEC) {
            // the raw tiles are no longer read: Q <- Q o exp(G), K <- K o exp(G_n - G)
            // (factored chunks: Q is already scaled and K holds K o exp(-G))
            for (int i = tid; i < n * DK; i += kSimtThreads) {
                const int r = i / DK, j = i % DK;
                const float gr = sm.GV[r * KP + j], gn = sm.GV[(n - 1) * KP + j];
                if (direct) {
                    sm.Q[r * KP + j] *= expf(gr);
                    sm.K[r * KP + j] *= expf(gn - gr);
                } else {
                    sm.K[r * KP + j] *= expf(gn);
                }
            }
            __syncthreads();
        }
        // ---- O = diag(gamma) Q S + P Ut ---------------------------------------------
        for (int i = tid; i < n * kDvs; i += kSimtThreads) {
            const int r = i / kDvs, c = i % kDvs;
            float qs = 0.f;
#pragma unroll 8
            for (int j = 0; j < DK; ++j) qs = fmaf(sm.Q[r * KP + j], sm.S[j * kDvs + c], qs);
            float pu = 0.f;
            for (int s = 0; s <= r; ++s) pu = fmaf(sm.P[r * CP + s], Ut[s * kDvs + c], pu);
            float ov = (VEC ? qs : expf(sm.G[r]) * qs) + pu;
            if (dsk) ov = fmaf(dsk[c], sm.V[i], ov);     // D-skip term D_h v_t
            if (XN) {
                sm.Ob[i] = ov;
                continue;
            }
            const long oi = o0 + (long)(t0 + r) * dv + c0 + c;
            if (!in_bounds(oi, n_rows * dv, err)) {
            } else if (out_bf16) static_cast<__nv_bfloat16 *>(o)[oi] = __float2bfloat16_rn(ov);
            else static_cast<float *>(o)[oi] = ov;
        }
        __syncthreads();
        if (XN) {
            // ---- output normalisation of each row over all dv columns (the cluster's
            //      slices): warp w takes rows w, w + 32 (lane = column of this slice)
            const int lane = tid & 31, warp = tid >> 5, nsl = dv / kDvs;
            const float wc = xw ? xw[static_cast<long>(sp.head_row % H) * dv + c0 + lane] : 1.f;
#pragma unroll
            for (int rr = 0; rr < kCmax; rr += 32) {
                const int r = rr + warp;
                // every thread takes part in both rounds (the cluster barrier is CTA-wide);
                // rows past n contribute zeros and store nothing
                float x = r < n ? sm.Ob[r * kDvs + lane] : 0.f;
                float mean = 0.f;
                if (xnorm == kXNormLayer) {
                    float s1 = x;
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) s1 += __shfl_xor_sync(0xffffffffu, s1, off);
                    mean = cluster_row_sum(sm.part, round++, r, s1, lane == 0, nsl) / dv;
                }
                x -= mean;
                float s2 = x * x;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, off);
                const float ms = cluster_row_sum(sm.part, round++, r, s2, lane == 0, nsl) / dv;
                const float y = x * rsqrtf(ms + xeps) * wc;
                if (r < n) {
                    const long oi = o0 + (long)(t0 + r) * dv + c0 + lane;
                    if (!in_bounds(oi, n_rows * dv, err)) {
                    } else if (out_bf16) static_cast<__nv_bfloat16 *>(o)[oi] = __float2bfloat16_rn(y);
                    else static_cast<float *>(o)[oi] = y;
                }
            }
            __syncthreads();
        }
        // ---- S <- gamma_n S + sum_s exp(G_n - G_s) k_s Ut_s^T ----------------------
        {
            const float Gn = sm.G[n - 1];
            for (int i = tid; i < DK * kDvs; i += kSimtThreads) {
                const int j = i / kDvs, c = i % kDvs;
                if (VEC) {
                    // K already holds k_s o exp(G_n - G_s)
                    float x = expf(sm.GV[(n - 1) * KP + j]) * sm.S[i];
                    for (int s = 0; s < n; ++s) x = fmaf(sm.K[s * KP + j], Ut[s * kDvs + c], x);
                    sm.S[i] = x;
                } else {
                    float x = expf(Gn) * sm.S[i];
                    for (int s = 0; s < n; ++s)
                        x = fmaf(expf(Gn - sm.G[s]) * sm.K[s * KP + j], Ut[s * kDvs + c], x);
                    sm.S[i] = x;
                }
            }
        }
    }
    __syncthreads();
    if (s_final) {
        for (int i = tid; i < DK * kDvs; i += kSimtThreads) {
            const int j = i / kDvs, c = i % kDvs;
            if (in_bounds((bh * DK + j) * dv + c0 + c, n_state, err)) s_final[(bh * DK + j) * dv + c0 + c] = sm.S[i];
        }
    }
}

template <int DK, typename IT, bool DELTA, bool VEC, bool XN>
gdn_status_t launch_simt_x(const void *q, const void *k, const void *v, const float *beta,
                           const float *g, void *o, const float *s0, float *s_final, const int *cu,
                           int BH, int H, int L, int dv, int chunk, float scale, const FwdOpts &oo, unsigned *err,
                           cudaStream_t stream) {
    auto kern = simt_chunk_fwd_kernel<DK, IT, DELTA, VEC, XN>;
    const unsigned smem = static_cast<unsigned>(sizeof(SimtSmem<DK, VEC, XN>));
    if (!ensure_smem_limit(reinterpret_cast<const void *>(kern), smem)) return GDN_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(BH, dv / kDvs);
    cfg.blockDim = dim3(kSimtThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    if (XN) {
        // the value slices of one head form a cluster: the output normalisation adds their
        // row sums through distributed shared memory
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 1;
        attr[0].val.clusterDim.y = static_cast<unsigned>(dv / kDvs);
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, kern, (const IT *)q, (const IT *)k, (const IT *)v, beta, g, o, oo.bf16 ? 1 : 0,
                              oo.dskip, oo.xnorm, oo.xw, oo.xeps, s0, s_final, cu, H, L, dv, chunk, scale, err) ==
                   cudaSuccess
               ? GDN_OK
               : GDN_ERR_CUDA;
}

template <int DK, typename IT, bool DELTA, bool VEC>
gdn_status_t launch_simt_t(const void *q, const void *k, const void *v, const float *beta,
                           const float *g, void *o, const float *s0, float *s_final, const int *cu,
                           int BH, int H, int L, int dv, int chunk, float scale, FwdOpts oo, unsigned *err,
                           cudaStream_t stream) {
    if (oo.xnorm != kXNormNone)
        return launch_simt_x<DK, IT, DELTA, VEC, true>(q, k, v, beta, g, o, s0, s_final, cu, BH, H, L, dv, chunk,
                                                       scale, oo, err, stream);
    return launch_simt_x<DK, IT, DELTA, VEC, false>(q, k, v, beta, g, o, s0, s_final, cu, BH, H, L, dv, chunk, scale,
                                                    oo, err, stream);
}

}  // namespace

gdn_status_t launch_simt_fwd(const void *q, const void *k, const void *v, const float *beta,
                             const float *g, void *o, const float *s0, float *s_final,
                             const int *cu, int B, int H, int L, int dk, int dv, int chunk,
                             float scale, gdn_dtype_t in_dtype, FwdOpts oo, cudaStream_t stream) {
    const int BH = B * H;
    const bool delta = beta != nullptr;
    unsigned *err = nullptr;
    if (cu && !(err = device_error_word())) return GDN_ERR_CUDA;
#define GDN_SIMT_CASE(DKV, IT)                                                                          \
    return delta ? (vec ? launch_simt_t<DKV, IT, true, true>(q, k, v, beta, g, o, s0, s_final, cu, BH, H, L, dv, \
                                                           chunk, scale, oo, err, stream)                   \
                        : launch_simt_t<DKV, IT, true, false>(q, k, v, beta, g, o, s0, s_final, cu, BH, H, L,  \
                                                            dv, chunk, scale, oo, err, stream))             \
                 : (vec ? launch_simt_t<DKV, IT, false, true>(q, k, v, beta, g, o, s0, s_final, cu, BH, H, L,  \
                                                            dv, chunk, scale, oo, err, stream)              \
                        : launch_simt_t<DKV, IT, false, false>(q, k, v, beta, g, o, s0, s_final, cu, BH, H, L, \
                                                             dv, chunk, scale, oo, err, stream))
    const bool vec = oo.gate_per_key && g != nullptr;   // one log-decay per key coordinate
    if (in_dtype == GDN_F32) {
        if (dk == 64) { GDN_SIMT_CASE(64, float); }
        GDN_SIMT_CASE(128, float);
    }
    if (dk == 64) { GDN_SIMT_CASE(64, __nv_bfloat16); }
    GDN_SIMT_CASE(128, __nv_bfloat16);
#undef GDN_SIMT_CASE
}

}  // namespace gdn
