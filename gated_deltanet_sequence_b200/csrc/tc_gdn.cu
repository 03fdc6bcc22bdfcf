// Tensor-core chunkwise DeltaNet / Gated DeltaNet prefill for sm_100a
// (bf16 inputs, dk = dv = 128, chunk C = 64; fp32 accumulation, output and state).
//
// One CTA per (batch, head) walks the chunks in order; the fp32 state S (dk x dv)
// lives in tensor memory for the whole sequence and never goes to HBM until the
// end. Per chunk of C rows (page "混合注意力学习(1)", sections "DeltaNet 分块并行机制",
// "重新定义降低内存占用", "HouseHolder变换和WY表示"; page "LinearAttention 概述", section
// "FLASH"), with G the within-chunk cumulative sum of g, gamma = exp(G),
// Gamma_rs = exp(G_r - G_s) (s <= r) and d_s = exp(G_last - G_s):
//   Gram   [K;Q] K^T                     one M=128 UMMA (rows: K K^T, then Q K^T)
//   UT     A = tril(diag(beta) KK^T o Gamma, -1), T = (I + A)^-1   (forward subst.)
//   W, U   W^T = K^T (T diag(beta gamma))^T, U^T = V^T (T diag(beta))^T
//   Ut     Ut^T = U^T - S^T W^T   (accumulated onto U^T with a negated operand)
//   QS     (Q S)^T = S^T Q^T
//   state  S <- gamma_last S + K^T (diag(d) Ut)
//   out    O^T = Ut^T (scale Q K^T o Gamma)^T;  o = scale gamma (QS) + O
// Every product is written with dk or dv (= 128) as the UMMA M dimension so each
// tcgen05.mma is a full 128-lane M=128 instruction; TMEM lane = row of the result.
//
// Shared-memory operands use the 128-byte swizzled canonical layouts (TMA writes
// Q, K, V that way; the epilogue threads write T, P, W, S and Ut the same way).
// All UMMA operands are fp16 (10-bit mantissa): the bf16 input tiles are converted
// in place (exact within the fp16 range) and every computed operand (T, P, W, S,
// Ut) is rounded to fp16, which keeps the rounding of the chunk intermediates ~8x
// below what bf16 operands give; accumulation is fp32 throughout.
#include <mutex>

#include "tc_kernels.cuh"
#include "tc_ptx.cuh"

namespace gdn {

// Device-side error word (static storage in the library image, one per device).
__device__ unsigned g_device_error = 0u;

unsigned *device_error_word() {
    static std::mutex mu;
    static unsigned *addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        addr[dev] = static_cast<unsigned *>(p);
    }
    return addr[dev];
}

bool read_and_clear_device_error(unsigned *err) {
    const unsigned zero = 0u;
    if (cudaMemcpyFromSymbol(err, g_device_error, sizeof(unsigned)) != cudaSuccess) return false;
    if (*err != 0u && cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess)
        return false;
    return true;
}

namespace {
using namespace ptx;

constexpr int kC = 64;          // chunk rows
constexpr int kD = 128;         // dk = dv
constexpr int kThreads = 128;   // 4 warps: warp w owns TMEM lanes 32w..32w+31

// ---- shared memory map (byte offsets from a 1024-aligned base) ------------------
constexpr uint32_t kStageBytes = 49152;  // one chunk of K, Q, V (bf16, swizzled)
constexpr uint32_t ST_K0 = 0;            // K, key columns 0-63   (64 rows x 128 B)
constexpr uint32_t ST_Q0 = 8192;         // Q, key columns 0-63   (directly after K: [K;Q])
constexpr uint32_t ST_K1 = 16384;        // K, key columns 64-127
constexpr uint32_t ST_Q1 = 24576;        // Q, key columns 64-127
constexpr uint32_t ST_V0 = 32768;        // V, value columns 0-63
constexpr uint32_t ST_V1 = 40960;        // V, value columns 64-127
constexpr uint32_t OFF_T1 = 2 * kStageBytes;       // T diag(beta gamma), K-major 64 x 64
constexpr uint32_t OFF_T2 = OFF_T1 + 8192;         // T diag(beta)
constexpr uint32_t OFF_PG = OFF_T2 + 8192;         // scale (Q K^T o Gamma), K-major 64 x 64
constexpr uint32_t OFF_W = OFF_PG + 8192;          // W as MN-major B: 128 key rows x 64 r
constexpr uint32_t OFF_S = OFF_W + 16384;          // S as MN-major A: 2 x (128 key rows x 64 v)
constexpr uint32_t OFF_UB = OFF_S + 32768;         // Ut, K-major: 128 value rows x 64 s
constexpr uint32_t OFF_UD = OFF_UB + 16384;        // diag(d) Ut, K-major
constexpr uint32_t OFF_A = OFF_UD + 16384;         // A fp32 64 x 64 (float4 groups swizzled)
constexpr uint32_t OFF_VEC = OFF_A + kC * kC * 4;  // G, beta, gamma, d: 4 x 64 fp32
constexpr uint32_t OFF_BAR = OFF_VEC + 1024;       // 3 mbarriers, TMEM base, abort flag
constexpr uint32_t kSmemBytes = OFF_BAR + 64;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;  // slack to align the base to 1024 B
static_assert(kSmemAlloc <= 232448, "shared memory budget");

// ---- tensor memory columns (512 allocated) ----------------------------------------
constexpr uint32_t TM_S = 0;     // state S: lane = key row j, 128 value columns
constexpr uint32_t TM_G = 128;   // [K;Q] K^T: lanes 0-63 K K^T, 64-127 Q K^T; 64 columns s
constexpr uint32_t TM_W = 192;   // W^T: lane = key j, 64 columns r
constexpr uint32_t TM_U = 256;   // U^T then Ut^T: lane = value v, 64 columns r
constexpr uint32_t TM_QS = 320;  // (Q S)^T: lane = value v, 64 columns r
constexpr uint32_t TM_O = 384;   // Ut^T P^T: lane = value v, 64 columns r

constexpr uint32_t ID_GRAM = idesc_f16(128, 64, false, false);
constexpr uint32_t ID_WU = idesc_f16(128, 64, true, false);
constexpr uint32_t ID_SW = idesc_f16(128, 64, true, true, /*neg_a=*/true);
constexpr uint32_t ID_SQ = idesc_f16(128, 64, true, false);
constexpr uint32_t ID_ST = idesc_f16(128, 128, true, false);
constexpr uint32_t ID_O = idesc_f16(128, 64, false, false);

__device__ __forceinline__ void record_timeout(unsigned *err, int *abort_flag) {
    atomicOr(err, kErrWaitTimeout);
    *abort_flag = 1;
}

template <bool GATED>
__global__ void __launch_bounds__(kThreads, 1)
tc_gdn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ beta,
              const float *__restrict__ g, float *__restrict__ o, const float *__restrict__ s0,
              float *__restrict__ s_final, int L, float scale, long long wait_limit,
              unsigned *__restrict__ err_word) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    float *Gs = reinterpret_cast<float *>(smem + OFF_VEC);
    float *bts = Gs + 64, *gms = Gs + 128, *dss = Gs + 192;
    float *Am = reinterpret_cast<float *>(smem + OFF_A);
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *bar_mma = bar_tma + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_mma + 1);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x;
    const int nchunks = (L + kC - 1) / kC;
    const size_t row0 = static_cast<size_t>(bh) * L;   // first token row of this head

    if (tid == 0) {
        mbar_init(&bar_tma[0], 1);
        mbar_init(&bar_tma[1], 1);
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
    const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);  // this warp's lanes

    auto issue_tma = [&](int c) {
        const int s = c & 1;
        uint8_t *st = smem + s * kStageBytes;
        mbar_arrive_expect_tx(&bar_tma[s], kStageBytes);
        tma_load_3d(st + ST_K0, &tm_k, &bar_tma[s], 0, c * kC, bh);
        tma_load_3d(st + ST_K1, &tm_k, &bar_tma[s], 64, c * kC, bh);
        tma_load_3d(st + ST_Q0, &tm_q, &bar_tma[s], 0, c * kC, bh);
        tma_load_3d(st + ST_Q1, &tm_q, &bar_tma[s], 64, c * kC, bh);
        tma_load_3d(st + ST_V0, &tm_v, &bar_tma[s], 0, c * kC, bh);
        tma_load_3d(st + ST_V1, &tm_v, &bar_tma[s], 64, c * kC, bh);
    };
    if (tid == 0) {
        issue_tma(0);
        if (nchunks > 1) issue_tma(1);
    }

    // initial state -> TMEM (thread t holds key row j = t)
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
        const uint32_t stg = sb + (c & 1) * kStageBytes;

        // ---- gate cumulative sum and beta for the 64 rows (rows >= n padded: g = beta = 0)
        if (tid < 64) {
            float x = (GATED && tid < n) ? g[row0 + t0 + tid] : 0.f;
            bts[tid] = (tid < n) ? beta[row0 + t0 + tid] : 0.f;
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
            gms[tid] = GATED ? __expf(Gs[tid]) : 1.f;
            dss[tid] = GATED ? __expf(Gs[63] - Gs[tid]) : 1.f;
        }
        // ---- wait for this chunk's Q, K, V tiles
        if (!mbar_wait(&bar_tma[c & 1], (c >> 1) & 1, wait_limit)) record_timeout(err_word, abort_flag);
        tc_fence_before();
        __syncthreads();
        if (*abort_flag) break;
        // the tensor-core operands are fp16: convert this chunk's bf16 tiles in place
        convert_tile_bf16_to_f16(smem + (c & 1) * kStageBytes, kStageBytes, tid, kThreads);
        fence_proxy_async();
        __syncthreads();

        // ---- (1) Gram [K;Q] K^T -> TM_G
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
        if (!mbar_wait(bar_mma, mma_phase, wait_limit)) record_timeout(err_word, abort_flag);
        mma_phase ^= 1;
        tc_fence_after();

        // ---- (E1) rows 0-63: A = beta_r Gamma_rs k_r.k_s (s < r), fp32, float4 groups
        //      swizzled by row; rows 64-127: scale Gamma_rs q_r.k_s (s <= r), bf16 -> PG
        {
            float v[64];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                float t16[16];
                tmem_ld16(trow + TM_G + cc * 16, t16);
#pragma unroll
                for (int e = 0; e < 16; ++e) v[cc * 16 + e] = t16[e];
            }
            tmem_wait_ld();
            if (warp < 2) {
                const int r = tid;
                const float br = bts[r], Gr = Gs[r];
                float *Arow = Am + r * kC;
#pragma unroll
                for (int qg = 0; qg < 16; ++qg) {
                    float a[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int s = qg * 4 + e;
                        a[e] = (s < r) ? br * __expf(Gr - Gs[s]) * v[s] : 0.f;
                    }
                    *reinterpret_cast<float4 *>(Arow + ((qg ^ (r & 15)) << 2)) = make_float4(a[0], a[1], a[2], a[3]);
                }
            } else {
                const int r = tid - 64;
                const float Gr = Gs[r];
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint32_t pk[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int s0i = ch * 8 + 2 * e;
                        const float p0 = (s0i <= r) ? scale * __expf(Gr - Gs[s0i]) * v[s0i] : 0.f;
                        const float p1 = (s0i + 1 <= r) ? scale * __expf(Gr - Gs[s0i + 1]) * v[s0i + 1] : 0.f;
                        pk[e] = pack_h2(p0, p1);
                    }
                    st_shared_v4(sb + OFF_PG + sw128(r, ch), pk[0], pk[1], pk[2], pk[3]);
                }
                fence_proxy_async();
            }
        }
        __syncthreads();

        // ---- (UT) T = (I + A)^-1: thread j (< 64) solves column j by forward substitution,
        //      then writes T diag(beta gamma) and T diag(beta) (bf16, K-major rows r)
        if (warp < 2) {
            const int j = tid;
            float x[64];
#pragma unroll
            for (int r = 0; r < 64; ++r) x[r] = 0.f;
#pragma unroll
            for (int r = 0; r < 64; ++r) {
                float a0 = (r == j) ? 1.f : 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
                const float *Ar = Am + r * kC;
#pragma unroll
                for (int qg = 0; qg < (r + 3) / 4; ++qg) {
                    const float4 av = *reinterpret_cast<const float4 *>(Ar + ((qg ^ (r & 15)) << 2));
                    a0 = fmaf(-av.x, x[4 * qg], a0);
                    a1 = fmaf(-av.y, x[4 * qg + 1], a1);
                    a2 = fmaf(-av.z, x[4 * qg + 2], a2);
                    a3 = fmaf(-av.w, x[4 * qg + 3], a3);
                }
                x[r] = (a0 + a1) + (a2 + a3);
            }
            const float bj = bts[j], bgj = bj * gms[j];
            uint8_t *t1 = smem + OFF_T1, *t2 = smem + OFF_T2;
#pragma unroll
            for (int r = 0; r < 64; ++r) {
                const uint32_t off = sw128(r, j >> 3) + (j & 7) * 2;
                *reinterpret_cast<__half *>(t1 + off) = __float2half_rn(x[r] * bgj);
                *reinterpret_cast<__half *>(t2 + off) = __float2half_rn(x[r] * bj);
            }
            fence_proxy_async();
        }
        __syncthreads();

        // ---- (2) W^T = K^T T1^T -> TM_W ; U^T = V^T T2^T -> TM_U
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(tmem + TM_W, sdesc_sw128(stg + ST_K0 + kk * 2048, 16384, 1024),
                         sdesc_sw128(sb + OFF_T1 + kk * 32, 16, 1024), ID_WU, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(tmem + TM_U, sdesc_sw128(stg + ST_V0 + kk * 2048, 8192, 1024),
                         sdesc_sw128(sb + OFF_T2 + kk * 32, 16, 1024), ID_WU, kk > 0);
            mma_commit(bar_mma);
        }
        if (!mbar_wait(bar_mma, mma_phase, wait_limit)) record_timeout(err_word, abort_flag);
        mma_phase ^= 1;
        tc_fence_after();

        // ---- (E3) W^T row j -> W tile (MN-major B); S row j -> S tile (MN-major A), and
        //      S <- gamma_last S in TMEM ahead of the state update
        {
            const int j = tid;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                float w[16];
                tmem_ld16(trow + TM_W + cc * 16, w);
                tmem_wait_ld();
                st_shared_v4(sb + OFF_W + sw128(j, 2 * cc), pack_h2(w[0], w[1]), pack_h2(w[2], w[3]),
                             pack_h2(w[4], w[5]), pack_h2(w[6], w[7]));
                st_shared_v4(sb + OFF_W + sw128(j, 2 * cc + 1), pack_h2(w[8], w[9]),
                             pack_h2(w[10], w[11]), pack_h2(w[12], w[13]), pack_h2(w[14], w[15]));
            }
            const float gl = gms[63];
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
            if (GATED) tmem_wait_st();
            fence_proxy_async();
        }
        tc_fence_before();
        __syncthreads();

        // ---- (3) Ut^T = U^T - S^T W^T (into TM_U) ; (Q S)^T = S^T Q^T -> TM_QS
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_f16(tmem + TM_U, sdesc_sw128(sb + OFF_S + kk * 2048, 16384, 1024),
                         sdesc_sw128(sb + OFF_W + kk * 2048, 8192, 1024), ID_SW, 1u);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
                mma_f16(tmem + TM_QS, sdesc_sw128(sb + OFF_S + kk * 2048, 16384, 1024),
                         sdesc_sw128(stg + ST_Q0 + off, 16, 1024), ID_SQ, kk > 0);
            }
            mma_commit(bar_mma);
        }
        if (!mbar_wait(bar_mma, mma_phase, wait_limit)) record_timeout(err_word, abort_flag);
        mma_phase ^= 1;
        tc_fence_after();

        // ---- (E4) Ut^T row v -> Ut tile and diag(d) Ut tile (K-major, rows v)
        {
            const int vrow = tid;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                float u[16];
                tmem_ld16(trow + TM_U + cc * 16, u);
                tmem_wait_ld();
                st_shared_v4(sb + OFF_UB + sw128(vrow, 2 * cc), pack_h2(u[0], u[1]), pack_h2(u[2], u[3]),
                             pack_h2(u[4], u[5]), pack_h2(u[6], u[7]));
                st_shared_v4(sb + OFF_UB + sw128(vrow, 2 * cc + 1), pack_h2(u[8], u[9]),
                             pack_h2(u[10], u[11]), pack_h2(u[12], u[13]), pack_h2(u[14], u[15]));
                float ud[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) ud[e] = GATED ? u[e] * dss[cc * 16 + e] : u[e];
                st_shared_v4(sb + OFF_UD + sw128(vrow, 2 * cc), pack_h2(ud[0], ud[1]), pack_h2(ud[2], ud[3]),
                             pack_h2(ud[4], ud[5]), pack_h2(ud[6], ud[7]));
                st_shared_v4(sb + OFF_UD + sw128(vrow, 2 * cc + 1), pack_h2(ud[8], ud[9]),
                             pack_h2(ud[10], ud[11]), pack_h2(ud[12], ud[13]), pack_h2(ud[14], ud[15]));
            }
            fence_proxy_async();
        }
        tc_fence_before();
        __syncthreads();

        // ---- (4) S += K^T (diag(d) Ut) -> TM_S ; O^T = Ut^T PG^T -> TM_O
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(tmem + TM_S, sdesc_sw128(stg + ST_K0 + kk * 2048, 16384, 1024),
                         sdesc_sw128(sb + OFF_UD + kk * 32, 16, 1024), ID_ST, 1u);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(tmem + TM_O, sdesc_sw128(sb + OFF_UB + kk * 32, 16, 1024),
                         sdesc_sw128(sb + OFF_PG + kk * 32, 16, 1024), ID_O, kk > 0);
            mma_commit(bar_mma);
        }
        if (!mbar_wait(bar_mma, mma_phase, wait_limit)) record_timeout(err_word, abort_flag);
        mma_phase ^= 1;
        tc_fence_after();
        // this stage's tiles are consumed: prefetch chunk c + 2 into it
        if (tid == 0 && c + 2 < nchunks) issue_tma(c + 2);

        // ---- (E5) o[r][v] = scale gamma_r (Q S)[r][v] + O[r][v]   (thread = value column v)
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
                    if (r < n) orow[static_cast<size_t>(r) * kD] = fmaf(scale * gms[r], qs[e], ov[e]);
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        if (*abort_flag) break;
    }

    // ---- final state TMEM -> HBM
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

}  // namespace

// ---------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// (BH, L, 128) bf16 -> 3-D map, 64 x 64 boxes, 128-byte swizzle, zero fill out of range.
bool make_qkv_map(CUtensorMap *m, const void *ptr, int L, int BH) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(BH)};
    const cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(L) * 256};
    const cuuint32_t box[3] = {64, 64, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

template <bool GATED>
gdn_status_t launch_gdn_t(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv, const float *beta,
                          const float *g, float *o, const float *s0, float *s_final, int BH, int L, float scale,
                          cudaStream_t stream) {
    auto kern = tc_gdn_kernel<GATED>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [&] {
        attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
    });
    if (attr_err != cudaSuccess) return GDN_ERR_CUDA;
    unsigned *err = device_error_word();
    if (!err) return GDN_ERR_CUDA;
    kern<<<BH, kThreads, kSmemAlloc, stream>>>(mq, mk, mv, beta, g, o, s0, s_final, L, scale, kWaitLimitCycles,
                                               err);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace

bool tc_supported(gdn_dtype_t in_dtype, int dk, int dv, int chunk) {
    return in_dtype == GDN_BF16 && dk == 128 && dv == 128 && chunk == 64 && encode_fn() != nullptr;
}

gdn_status_t launch_tc_gdn(const void *q, const void *k, const void *v, const float *beta, const float *g,
                           float *o, const float *s0, float *s_final, int B, int H, int L, float scale,
                           cudaStream_t stream) {
    const int BH = B * H;
    CUtensorMap mq, mk, mv;
    if (!make_qkv_map(&mq, q, L, BH) || !make_qkv_map(&mk, k, L, BH) || !make_qkv_map(&mv, v, L, BH))
        return GDN_ERR_CUDA;
    return g ? launch_gdn_t<true>(mq, mk, mv, beta, g, o, s0, s_final, BH, L, scale, stream)
             : launch_gdn_t<false>(mq, mk, mv, beta, g, o, s0, s_final, BH, L, scale, stream);
}

}  // namespace gdn
