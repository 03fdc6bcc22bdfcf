// Tensor-core chunkwise causal linear attention for sm_100a, plain (alpha = 1) or
// with a scalar per-token decay; bf16 inputs, dk = dv = 128, chunk C = 64, fp32
// accumulation, output and state, no normaliser.
//
// Page "混合注意力学习(1)", section "FWP分块并行机制": inside a chunk the output mixes
// the carried state (inter-chunk part) with a causally masked product over the
// chunk's own rows (intra-chunk part); page "LinearAttention 概述", sections
// "快速预览" / "Lightning Attention": O = (Q K^T o M) V with the diagonal included.
// Per chunk, with G the within-chunk cumulative sum of g (0 when ungated),
// gamma = exp(G), Gamma_rs = exp(G_r - G_s) (s <= r), d_s = exp(G_last - G_s):
//   Gram   [K;Q] K^T (the Q K^T half is used)      M=128 UMMA
//   QS     (Q S)^T = S^T Q^T                        M=128 (value rows)
//   out    O^T = V^T (scale Q K^T o Gamma)^T;  o = scale gamma (QS) + O
//   state  S <- gamma_last S + K^T diag(d) V        M=128 (key rows)
// One CTA per (batch, head); the fp32 state stays in tensor memory; Q, K, V stream
// through a 3-stage TMA ring because this kernel is bound by HBM bandwidth. UMMA
// operands are fp16: the bf16 tiles are converted in place (exact in fp16 range)
// and the computed operands (S, P, diag(d) V) are rounded to fp16.
#include <mutex>

#include "tc_kernels.cuh"
#include "tc_ptx.cuh"

namespace gdn {

namespace {
using namespace ptx;

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kThreads = 128;
constexpr int kStages = 3;

constexpr uint32_t kStageBytes = 49152;
constexpr uint32_t ST_K0 = 0, ST_Q0 = 8192, ST_K1 = 16384, ST_Q1 = 24576, ST_V0 = 32768, ST_V1 = 40960;
constexpr uint32_t OFF_PG = kStages * kStageBytes;   // scale (Q K^T o Gamma), K-major 64 x 64
constexpr uint32_t OFF_S = OFF_PG + 8192;            // S as MN-major A: 2 x (128 key rows x 64 v)
constexpr uint32_t OFF_VD = OFF_S + 32768;           // diag(d) V, same layout as the V tiles
constexpr uint32_t OFF_VEC = OFF_VD + 16384;         // G, gamma, d
constexpr uint32_t OFF_BAR = OFF_VEC + 1024;
constexpr uint32_t kSmemBytes = OFF_BAR + 64;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;
static_assert(kSmemAlloc <= 232448, "shared memory budget");

constexpr uint32_t TM_S = 0, TM_G = 128, TM_QS = 192, TM_O = 256;

constexpr uint32_t ID_GRAM = idesc_f16(128, 64, false, false);
constexpr uint32_t ID_SQ = idesc_f16(128, 64, true, false);
constexpr uint32_t ID_O = idesc_f16(128, 64, true, false);
constexpr uint32_t ID_ST = idesc_f16(128, 128, true, true);

template <bool GATED>
__global__ void __launch_bounds__(kThreads, 1)
tc_la_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ g, float *__restrict__ o,
             const float *__restrict__ s0, float *__restrict__ s_final, int L, float scale,
             long long wait_limit, unsigned *__restrict__ err_word) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base derived by pointer arithmetic on the shared array, so the
    // compiler keeps every access below in the shared address space (LDS/STS)
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(smem);
    float *Gs = reinterpret_cast<float *>(smem + OFF_VEC);
    float *gms = Gs + 64, *dss = Gs + 128;
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *bar_mma = bar_tma + kStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_mma + 1);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x;
    const int nchunks = (L + kC - 1) / kC;
    const size_t row0 = static_cast<size_t>(bh) * L;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&bar_tma[s], 1);
        mbar_init(bar_mma, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);

    auto issue_tma = [&](int c) {
        const int s = c % kStages;
        uint8_t *st = smem + s * kStageBytes;
        mbar_arrive_expect_tx(&bar_tma[s], kStageBytes);
        tma_load_3d(st + ST_K0, &tm_k, &bar_tma[s], 0, c * kC, bh);
        tma_load_3d(st + ST_K1, &tm_k, &bar_tma[s], 64, c * kC, bh);
        tma_load_3d(st + ST_Q0, &tm_q, &bar_tma[s], 0, c * kC, bh);
        tma_load_3d(st + ST_Q1, &tm_q, &bar_tma[s], 64, c * kC, bh);
        tma_load_3d(st + ST_V0, &tm_v, &bar_tma[s], 0, c * kC, bh);
        tma_load_3d(st + ST_V1, &tm_v, &bar_tma[s], 64, c * kC, bh);
    };
    if (tid == 0)
        for (int c = 0; c < kStages && c < nchunks; ++c) issue_tma(c);

    {
        const float *src = s0 ? s0 + (static_cast<size_t>(bh) * kD + tid) * kD : nullptr;
#pragma unroll 1
        for (int cc = 0; cc < 8; ++cc) {
            float r[16];
#pragma unroll
            for (int e = 0; e < 16; e += 4) {
                float4 x = src ? *reinterpret_cast<const float4 *>(src + cc * 16 + e) : make_float4(0.f, 0.f, 0.f, 0.f);
                r[e] = x.x; r[e + 1] = x.y; r[e + 2] = x.z; r[e + 3] = x.w;
            }
            tmem_st16(trow + TM_S + cc * 16, r);
        }
        tmem_wait_st();
    }

    uint32_t mma_phase = 0;
#pragma unroll 1
    for (int c = 0; c < nchunks; ++c) {
        const int t0 = c * kC;
        const int n = min(kC, L - t0);
        const int stage = c % kStages;
        const uint32_t stg = sb + stage * kStageBytes;

        if (GATED) {
            if (tid < 64) {
                float x = (tid < n) ? g[row0 + t0 + tid] : 0.f;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, x, off);
                    if (lane >= off) x += y;
                }
                Gs[tid] = x;
            }
            __syncthreads();
            if (tid >= 32 && tid < 64) Gs[tid] += Gs[31];
            __syncthreads();
            if (tid < 64) {
                gms[tid] = __expf(Gs[tid]);
                dss[tid] = __expf(Gs[63] - Gs[tid]);
            }
        }
        if (!mbar_wait(&bar_tma[stage], (c / kStages) & 1, wait_limit)) {
            atomicOr(err_word, kErrWaitTimeout);
            *abort_flag = 1;
        }
        tc_fence_before();
        __syncthreads();
        if (*abort_flag) break;
        // fp16 tensor-core operands: convert this chunk's bf16 tiles in place
        convert_tile_bf16_to_f16(smem + stage * kStageBytes, kStageBytes, tid, kThreads);
        fence_proxy_async();
        __syncthreads();

        // ---- (1) [K;Q] K^T -> TM_G
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
                mma_f16(tmem + TM_G, sdesc_sw128(stg + ST_K0 + off, 16, 1024),
                         sdesc_sw128(stg + ST_K0 + off, 16, 1024), ID_GRAM, kk > 0);
            }
            mma_commit(bar_mma);
        }

        // ---- (E1a, overlapping the Gram MMA) S row j -> S tile; S <- gamma_last S;
        //      diag(d) V tile for the gated state update
        {
            const int j = tid;
            const float gl = GATED ? gms[63] : 1.f;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                float sv[16];
                tmem_ld16(trow + TM_S + cc * 16, sv);
                tmem_wait_ld();
                const uint32_t base = sb + OFF_S + (cc >> 2) * 16384u;
                const int ch = (cc & 3) * 2;
                st_shared_v4(base + sw128(j, ch), pack_h2(sv[0], sv[1]), pack_h2(sv[2], sv[3]),
                             pack_h2(sv[4], sv[5]), pack_h2(sv[6], sv[7]));
                st_shared_v4(base + sw128(j, ch + 1), pack_h2(sv[8], sv[9]), pack_h2(sv[10], sv[11]),
                             pack_h2(sv[12], sv[13]), pack_h2(sv[14], sv[15]));
                if (GATED) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) sv[e] *= gl;
                    tmem_st16(trow + TM_S + cc * 16, sv);
                }
            }
            if (GATED) {
                tmem_wait_st();
                // 16 KB of V (1024 chunks of 16 B): chunk at byte offset b sits in row (b / 128) % 64
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint32_t b = (i * kThreads + tid) * 16u;
                    const int row = (b >> 7) & 63;
                    const uint4 x = *reinterpret_cast<const uint4 *>(smem + stage * kStageBytes + ST_V0 + b);
                    const float dsc = dss[row];
                    const __half2 *h = reinterpret_cast<const __half2 *>(&x);
                    uint32_t y[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __half22float2(h[e]);
                        y[e] = pack_h2(f.x * dsc, f.y * dsc);
                    }
                    st_shared_v4(sb + OFF_VD + b, y[0], y[1], y[2], y[3]);
                }
            }
        }
        if (!mbar_wait(bar_mma, mma_phase, wait_limit)) {
            atomicOr(err_word, kErrWaitTimeout);
            *abort_flag = 1;
        }
        mma_phase ^= 1;
        tc_fence_after();
        // ---- (E1b) rows 64-127 of the Gram: scale Gamma_rs q_r.k_s (s <= r) -> PG (bf16)
        if (warp >= 2) {
            const int r = tid - 64;
            float v[64];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                float t16[16];
                tmem_ld16(trow + TM_G + cc * 16, t16);
#pragma unroll
                for (int e = 0; e < 16; ++e) v[cc * 16 + e] = t16[e];
            }
            tmem_wait_ld();
            const float Gr = GATED ? Gs[r] : 0.f;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                uint32_t pk[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int s = ch * 8 + 2 * e;
                    const float w0 = GATED ? __expf(Gr - Gs[s]) : 1.f;
                    const float w1 = GATED ? __expf(Gr - Gs[s + 1]) : 1.f;
                    const float p0 = (s <= r) ? scale * w0 * v[s] : 0.f;
                    const float p1 = (s + 1 <= r) ? scale * w1 * v[s + 1] : 0.f;
                    pk[e] = pack_h2(p0, p1);
                }
                st_shared_v4(sb + OFF_PG + sw128(r, ch), pk[0], pk[1], pk[2], pk[3]);
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();

        // ---- (2) (Q S)^T -> TM_QS ; O^T = V^T PG^T -> TM_O ; S += K^T diag(d) V
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
                mma_f16(tmem + TM_QS, sdesc_sw128(sb + OFF_S + kk * 2048, 16384, 1024),
                         sdesc_sw128(stg + ST_Q0 + off, 16, 1024), ID_SQ, kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(tmem + TM_O, sdesc_sw128(stg + ST_V0 + kk * 2048, 8192, 1024),
                         sdesc_sw128(sb + OFF_PG + kk * 32, 16, 1024), ID_O, kk > 0);
            const uint32_t vb = GATED ? sb + OFF_VD : stg + ST_V0;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(tmem + TM_S, sdesc_sw128(stg + ST_K0 + kk * 2048, 16384, 1024),
                         sdesc_sw128(vb + kk * 2048, 8192, 1024), ID_ST, 1u);
            mma_commit(bar_mma);
        }
        if (!mbar_wait(bar_mma, mma_phase, wait_limit)) {
            atomicOr(err_word, kErrWaitTimeout);
            *abort_flag = 1;
        }
        mma_phase ^= 1;
        tc_fence_after();
        if (tid == 0 && c + kStages < nchunks) issue_tma(c + kStages);

        // ---- (E2) o[r][v] = scale gamma_r (Q S)[r][v] + O[r][v]
        {
            const int vcol = tid;
            float *orow = o + (row0 + t0) * kD + vcol;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                float qs[16], ov[16];
                tmem_ld16(trow + TM_QS + cc * 16, qs);
                tmem_ld16(trow + TM_O + cc * 16, ov);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int r = cc * 16 + e;
                    const float gr = GATED ? gms[r] : 1.f;
                    if (r < n) orow[static_cast<size_t>(r) * kD] = fmaf(scale * gr, qs[e], ov[e]);
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        if (*abort_flag) break;
    }

    if (!*abort_flag && s_final) {
        tc_fence_after();
        float *dst = s_final + (static_cast<size_t>(bh) * kD + tid) * kD;
#pragma unroll 1
        for (int cc = 0; cc < 8; ++cc) {
            float sv[16];
            tmem_ld16(trow + TM_S + cc * 16, sv);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; e += 4)
                *reinterpret_cast<float4 *>(dst + cc * 16 + e) = make_float4(sv[e], sv[e + 1], sv[e + 2], sv[e + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <bool GATED>
gdn_status_t launch_la_t(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv, const float *g,
                         float *o, const float *s0, float *s_final, int BH, int L, float scale,
                         cudaStream_t stream) {
    auto kern = tc_la_kernel<GATED>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [&] {
        attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
    });
    if (attr_err != cudaSuccess) return GDN_ERR_CUDA;
    unsigned *err = device_error_word();
    if (!err) return GDN_ERR_CUDA;
    kern<<<BH, kThreads, kSmemAlloc, stream>>>(mq, mk, mv, g, o, s0, s_final, L, scale, kWaitLimitCycles, err);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace

gdn_status_t launch_tc_la(const void *q, const void *k, const void *v, const float *g, float *o,
                          const float *s0, float *s_final, int B, int H, int L, float scale,
                          cudaStream_t stream) {
    const int BH = B * H;
    CUtensorMap mq, mk, mv;
    if (!make_qkv_map(&mq, q, L, BH) || !make_qkv_map(&mk, k, L, BH) || !make_qkv_map(&mv, v, L, BH))
        return GDN_ERR_CUDA;
    return g ? launch_la_t<true>(mq, mk, mv, g, o, s0, s_final, BH, L, scale, stream)
             : launch_la_t<false>(mq, mk, mv, g, o, s0, s_final, BH, L, scale, stream);
}

}  // namespace gdn
