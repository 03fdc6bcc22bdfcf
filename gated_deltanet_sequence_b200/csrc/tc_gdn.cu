// Tensor-core chunkwise DeltaNet / Gated DeltaNet prefill for sm_100a
// (bf16 inputs, dk = dv = 128, chunk C = 64; fp32 accumulation, output and state).
//
// One CTA per (batch, head) walks the chunks in order; the fp32 state lives in tensor
// memory for the whole sequence and goes to HBM only at the end. Per chunk of C rows
// (page "混合注意力学习(1)", sections "DeltaNet 分块并行机制", "重新定义降低内存占用",
// "HouseHolder变换和WY表示"; page "LinearAttention 概述", section "FLASH"), with G the
// within-chunk cumulative sum of g, gamma = exp(G), Gamma_rs = exp(G_r - G_s) (s <= r)
// and d_s = exp(G_last - G_s):
//   Gram   [K;Q] K^T                        one M=128 UMMA (rows: K K^T, then Q K^T)
//   UT     A = tril(diag(beta) KK^T o Gamma, -1), T = (I + A)^-1   (forward substitution)
//   W, U   W^T = K^T (T diag(beta gamma))^T, U^T = V^T (T diag(beta))^T
//   Ut     Ut^T = U^T + (-S^T) W^T
//   out    O^T = (-S^T)(-Q')^T + Ut^T P^T,  Q' = diag(scale gamma) Q,  P = scale (Q K^T o Gamma)
//   state  S^T <- gamma_last S^T + (Ut^T diag(d)) K
// The state is held transposed (S^T: TMEM lane = value column v), so its fp16 copy
// (-S^T, the A operand of the two state products) and the fp16 copies of Ut^T (plain
// for the output, scaled by d for the state update) are formed lane by lane inside
// tensor memory and read by the UMMAs from there: the serial chain per chunk is
// S^T -> fp16, S Q' and U - W S (16 UMMAs), Ut^T -> fp16, the state update (4 UMMAs).
// Every UMMA has M = 128 (dk or dv rows).
//
// Warp roles (512 threads):
//   warp 0      TMA producer (3-stage ring of Q, K, V tiles)
//   warp 1      Gram and W/U issuer: issues whichever of Gram(c+1) / W/U(c) is ready
//   warp 2      chain issuer: S Q', U - W S, state update, P Ut
//   warp 3      gate warp: G, gamma, d, exp(-G), beta per chunk (3-buffer ring)
//   warps 4-7   state group: S^T -> fp16 (and the decay), O^T -> o, the W operand
//               (W^T -> fp16), Ut^T -> fp16 copies
//   warps 8-11  solve group: UT solve of A (16 x 16 diagonal blocks by substitution,
//               off-diagonal blocks by warp-level tf32 MMA) and the fp16 T factors
//   warps 12-15 prep group: A / P masks from the Gram, K, V -> fp16, Q -> -Q'
// The prep and solve of later chunks run while the chain works on chunk c; every
// hand-off is an mbarrier with one arrival. Buffers shared by consecutive chunks are
// multi-buffered (stages and gate values x3, A^T and P x2) with per-buffer barriers, so
// no parity wait can see its barrier two phases ahead.
//
// Decay factors: Gamma_rs = exp(G_r - G_s) is formed as gamma_r * exp(-G_s) when the
// chunk's total log-decay G_last >= -60 (both factors then stay far inside fp32
// range); chunks with stronger decay take one exp per element instead.
//
// Precision: the Gram product runs on the bf16 input tiles (exact products, fp32
// sums). Every other UMMA takes fp16 operands (10-bit mantissa): K, V are converted in
// place after the Gram has read them, Q is replaced by -Q' in fp16, and every computed
// operand (T, P, W, S, Ut) is rounded to fp16, which keeps the rounding of the chunk
// intermediates ~8x below what bf16 operands give; A enters the UT solve in fp16 (its
// block products run in tf32, whose mantissa is the same). Shared-memory operands use
// the 128-byte swizzled canonical layouts.
#include <cuda_fp16.h>

#include "tc_gdn_parts.cuh"

namespace gdn {

namespace {
using namespace ptx;
using namespace tcgdn;
constexpr int kThreads = 512;
constexpr int kStages = 3;
constexpr int kGroupS = 4;       // first warp of the state group (4 warps)
constexpr int kGroupT = 8;       // first warp of the solve group (4 warps)
constexpr int kGroupM = 12;      // first warp of the prep group (4 warps)
constexpr int kBarS = 1, kBarT = 2, kBarM = 3;   // named barriers of the three groups (128 threads each)
constexpr float kFastDecayLimit = -60.f;   // G_last >= this: Gamma = gamma_r * exp(-G_s)

// ---- shared memory map (byte offsets from a 1024-aligned base) ------------------
constexpr uint32_t kStageBytes = 49152;   // one chunk of K, Q, V
constexpr uint32_t ST_K0 = 0;             // K, key columns 0-63   (64 rows x 128 B)
constexpr uint32_t ST_Q0 = 8192;          // Q, key columns 0-63   (directly after K: [K;Q])
constexpr uint32_t ST_K1 = 16384;         // K, key columns 64-127
constexpr uint32_t ST_Q1 = 24576;         // Q, key columns 64-127
constexpr uint32_t ST_V0 = 32768;         // V, value columns 0-63; holds W (MN-major, 128 key
constexpr uint32_t ST_V1 = 40960;         //   rows x 64 r) once U has been formed
constexpr uint32_t ST_W = ST_V0;
constexpr uint32_t OFF_AT = kStages * kStageBytes;  // 2 x A^T fp16 64 x 64 (UT-solve input)
constexpr uint32_t kAtBytes = 8192;
constexpr uint32_t OFF_TF = OFF_AT + 2 * kAtBytes;  // T fp32 64 x 68 (pitch 68)
constexpr int kTP = 68;
constexpr uint32_t OFF_R = OFF_TF + 64 * kTP * 4;   // 4 x 16 x 16 fp32 per-warp block scratch
constexpr uint32_t OFF_PG = OFF_R + 4096;           // 2 x scale (Q K^T o Gamma), K-major 64 x 64 fp16
constexpr uint32_t OFF_T1 = OFF_PG + 16384;         // T diag(beta gamma), K-major 64 x 64 fp16
constexpr uint32_t OFF_T2 = OFF_T1 + 8192;          // T diag(beta)
constexpr uint32_t OFF_VEC = OFF_T2 + 8192;         // 3 x {G, beta, gamma, d, exp(-G), flag}
constexpr uint32_t kVecBytes = 1536;                //   (64 fp32 each; flag = fast decay path)
constexpr int V_G = 0, V_B = 64, V_GAM = 128, V_D = 192, V_IG = 256, V_FAST = 320;
constexpr uint32_t OFF_XN = OFF_VEC + kStages * kVecBytes;   // output-normalisation scratch (384 fp32)
constexpr uint32_t OFF_BAR = OFF_XN + 1536;         // mbarriers, TMEM base, abort flag
constexpr uint32_t kSmemBytes = OFF_BAR + 512;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;  // slack to align the base to 1024 B
static_assert(kSmemAlloc <= 232448, "shared memory budget");
static_assert(OFF_T1 % 1024 == 0 && OFF_T2 % 1024 == 0 && OFF_PG % 1024 == 0, "UMMA tiles need 1024-B alignment");

// ---- tensor memory columns (512 allocated) ----------------------------------------
constexpr uint32_t TM_S = 0;      // S^T fp32: lane = value column v, 128 key columns j
constexpr uint32_t TM_SH = 128;   // -S^T fp16 (A operand): 64 columns of key pairs
constexpr uint32_t TM_G = 192;    // [K;Q] K^T: lanes 0-63 K K^T, 64-127 Q K^T; 64 columns s
constexpr uint32_t TM_W = 256;    // W^T: lane = key j, 64 columns r
constexpr uint32_t TM_U = 320;    // U^T then Ut^T: lane = value v, 64 columns r
constexpr uint32_t TM_UH = 384;   // Ut^T fp16 (A operand of the output): 32 columns of row pairs
constexpr uint32_t TM_UD = 416;   // (Ut^T diag(d)) fp16 (A operand of the state update)
constexpr uint32_t TM_O = 448;    // O^T: lane = value v, 64 columns r

constexpr uint32_t ID_GRAM = idesc_f16(128, 64, false, false, false, /*bf16=*/true);
constexpr uint32_t ID_WU = idesc_f16(128, 64, true, false);
constexpr uint32_t ID_SW = idesc_f16(128, 64, false, true);    // A (-S^T) from TMEM, B = W MN-major
constexpr uint32_t ID_SQ = idesc_f16(128, 64, false, false);   // A (-S^T) from TMEM, B = -Q' K-major
constexpr uint32_t ID_ST = idesc_f16(128, 128, false, true);   // A (Ut^T d) from TMEM, B = K MN-major
constexpr uint32_t ID_O = idesc_f16(128, 64, false, false);    // A (Ut^T) from TMEM, B = P K-major

// mbarriers (index into the barrier array). Per-buffer barriers ([n]) are indexed by the
// buffer a chunk uses (c % 3 for stages and gate values, c & 1 for A^T and P) and
// waited with the parity of that buffer's use count; single barriers with c & 1.
enum : int {
    B_FULL = 0,      // [3] TMA -> Gram issuer
    B_SFREE = 3,     // [3] state update of the stage's chunk done -> TMA
    B_VEC = 6,       // [3] gate values ready -> prep, solve, state groups
    B_VFREE = 9,     // [3] state group done with the gate values -> gate warp
    B_ATRDY = 12,    // [2] A^T and P written -> solve group, chain issuer
    B_ATFREE = 14,   // [2] solve group done with A^T -> prep group
    B_PFREE = 16,    // [2] P Ut done (P buffer free) -> prep group
    B_CONV = 18,     // [3] K, V fp16 and -Q' written -> Gram/WU issuer, chain issuer
    B_GRAM = 21,     // Gram done -> prep group
    B_GFREE = 22,    // prep group has read the Gram -> Gram/WU issuer
    B_TRDY = 23,     // T factors written -> Gram/WU issuer
    B_WU = 24,       // W/U done -> state group (W epilogue), solve group (T buffer free)
    B_WRDY = 25,     // W operand written, W^T read -> chain issuer, Gram/WU issuer
    B_SRDY = 26,     // -S^T fp16 written, S^T decayed -> chain issuer
    B_OFREE = 27,    // state group has read O^T -> chain issuer
    B_ADONE = 28,    // U - W S and S Q' done -> state group
    B_URDY = 29,     // Ut^T fp16 copies written, U^T read -> chain issuer, Gram/WU issuer
    B_SDONE = 30,    // state update done -> state group
    B_ODONE = 31,    // P Ut done (O^T complete) -> state group
    kNumBars = 32
};

// Non-blocking test of a barrier phase (the Gram/WU issuer polls two queues, so neither
// may suspend it).
__device__ __forceinline__ bool ready(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

template <bool GATED, bool OPTS>
__global__ void __launch_bounds__(kThreads, 1)
tc_gdn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ beta,
              const float *__restrict__ g, const OutArgs out, const float *__restrict__ s0,
              float *__restrict__ s_final, const int *__restrict__ cu, int H, int Lrow, float scale,
              long long wait_limit, unsigned *__restrict__ err_word) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base derived by pointer arithmetic on the shared array, so the
    // compiler keeps every access below in the shared address space (LDS/STS)
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kNumBars);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
    const Ctl ctl{bars, abort_flag, err_word, wait_limit};

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x;                          // (sequence, head): state index
    const SeqSpan sp = seq_span(cu, bh, H, Lrow, err_word);
    const int L = sp.len;                               // tokens of this sequence
    const int zc = sp.head_row, ty0 = sp.t0;            // TMA head and first-token coordinates
    const int nchunks = (L + kC - 1) / kC;
    const size_t row0 = static_cast<size_t>(zc) * Lrow + ty0;   // first token row in the grid

    if (tid == 0) {
        for (int b = 0; b < kNumBars; ++b) mbar_init(&bars[b], 1);
        abort_flag[0] = 0;
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
    auto vec_of = [&](int c) { return reinterpret_cast<float *>(smem + OFF_VEC + (c % kStages) * kVecBytes); };

    if (warp == 0) {
        // ================================================================ TMA producer
        if (lane == 0) {
            int last[kStages] = {-1, -1, -1};   // last chunk loaded into each stage
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % kStages;
                if (c >= kStages && !ctl.wait_lazy(B_SFREE + s, ((c - kStages) / kStages) & 1)) break;
                uint8_t *st = smem + s * kStageBytes;
                uint64_t *fb = &bars[B_FULL + s];
                mbar_arrive_expect_tx(fb, kStageBytes);
                tma_load_3d(st + ST_K0, &tm_k, fb, 0, ty0 + c * kC, zc);
                tma_load_3d(st + ST_Q0, &tm_q, fb, 0, ty0 + c * kC, zc);
                tma_load_3d(st + ST_K1, &tm_k, fb, 64, ty0 + c * kC, zc);
                tma_load_3d(st + ST_Q1, &tm_q, fb, 64, ty0 + c * kC, zc);
                tma_load_3d(st + ST_V0, &tm_v, fb, 0, ty0 + c * kC, zc);
                tma_load_3d(st + ST_V1, &tm_v, fb, 64, ty0 + c * kC, zc);
                last[s] = c;
            }
            // never leave a copy in flight past the end of the CTA
            for (int s = 0; s < kStages; ++s)
                if (last[s] >= 0) ctl.drain(B_FULL + s, (last[s] / kStages) & 1);
        }
    } else if (warp == 1) {
        // ================================================================ Gram / W-U issuer
        // Gram(c) on the bf16 tiles once they have landed and the prep group has read
        // Gram(c-1); W/U(c) once the T factors and the fp16 K, V of chunk c are written and
        // chunk c-1 has released W^T (W epilogue) and U^T (Ut copies). Whichever is ready
        // is issued first, so neither queue blocks the other.
        if (lane == 0) {
            int ng = 0, nw = 0, last_bar = -1, last_par = 0;
            long long t0 = clock64();
            while (nw < nchunks) {
                bool issued = false;
                if (ng < nchunks && ng < nw + kStages && ready(&bars[B_FULL + ng % kStages], (ng / kStages) & 1) &&
                    (ng == 0 || ready(&bars[B_GFREE], (ng - 1) & 1))) {
                    const uint32_t stg = sb + (ng % kStages) * kStageBytes;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
                        mma_f16(tmem + TM_G, sdesc_sw128(stg + ST_K0 + off, 16, 1024),
                                sdesc_sw128(stg + ST_K0 + off, 16, 1024), ID_GRAM, kk > 0);
                    }
                    mma_commit(&bars[B_GRAM]);
                    last_bar = B_GRAM;
                    last_par = ng & 1;
                    ++ng;
                    issued = true;
                }
                if (nw < ng && ready(&bars[B_TRDY], nw & 1) && ready(&bars[B_CONV + nw % kStages], (nw / kStages) & 1) &&
                    (nw == 0 || (ready(&bars[B_WRDY], (nw - 1) & 1) && ready(&bars[B_URDY], (nw - 1) & 1)))) {
                    const uint32_t stg = sb + (nw % kStages) * kStageBytes;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16(tmem + TM_W, sdesc_sw128(stg + ST_K0 + kk * 2048, 16384, 1024),
                                sdesc_sw128(sb + OFF_T1 + kk * 32, 16, 1024), ID_WU, kk > 0);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16(tmem + TM_U, sdesc_sw128(stg + ST_V0 + kk * 2048, 8192, 1024),
                                sdesc_sw128(sb + OFF_T2 + kk * 32, 16, 1024), ID_WU, kk > 0);
                    mma_commit(&bars[B_WU]);
                    last_bar = B_WU;
                    last_par = nw & 1;
                    ++nw;
                    issued = true;
                }
                if (issued) {
                    t0 = clock64();
                } else if (__nanosleep(32), ctl.aborted()) {
                    break;
                } else if (clock64() - t0 > ctl.limit) {
                    ctl.give_up();
                    break;
                }
            }
            // UMMAs complete in issue order: the last commit covers everything issued
            if (last_bar >= 0) ctl.drain(last_bar, last_par);
        }
    } else if (warp == 2) {
        // ================================================================ chain issuer
        // per chunk: S Q' and U - W S; the state update; then P Ut
        if (lane == 0) {
            int last_bar = -1, last_par = 0;   // last commit, for the final drain
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % kStages, p = c & 1;
                const uint32_t stg = sb + s * kStageBytes;
                if (!ctl.wait(B_SRDY, c & 1)) break;
                if (c >= 1 && !ctl.wait(B_OFREE, (c - 1) & 1)) break;
                if (!ctl.wait(B_CONV + s, (c / kStages) & 1)) break;
                tc_fence_after();
                // O^T = (-S^T)(-Q')^T
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
                    mma_f16_ts(tmem + TM_O, tmem + TM_SH + kk * 8, sdesc_sw128(stg + ST_Q0 + off, 16, 1024), ID_SQ,
                               kk > 0);
                }
                if (!ctl.wait(B_WRDY, c & 1)) {
                    // cover the UMMAs just issued by a commit, so the final drain waits for them
                    mma_commit(&bars[B_ADONE]);
                    last_bar = B_ADONE;
                    last_par = c & 1;
                    break;
                }
                tc_fence_after();
                // Ut^T = U^T + (-S^T) W^T
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_f16_ts(tmem + TM_U, tmem + TM_SH + kk * 8, sdesc_sw128(stg + ST_W + kk * 2048, 8192, 1024),
                               ID_SW, 1u);
                mma_commit(&bars[B_ADONE]);
                last_bar = B_ADONE;
                last_par = c & 1;
                if (!ctl.wait(B_URDY, c & 1)) break;
                tc_fence_after();
                // S^T += (Ut^T diag(d)) K
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f16_ts(tmem + TM_S, tmem + TM_UD + kk * 8, sdesc_sw128(stg + ST_K0 + kk * 2048, 16384, 1024),
                               ID_ST, 1u);
                mma_commit(&bars[B_SDONE]);
                mma_commit(&bars[B_SFREE + s]);
                last_bar = B_SFREE + s;
                last_par = (c / kStages) & 1;
                // O^T += Ut^T P^T
                if (!ctl.wait(B_ATRDY + p, (c >> 1) & 1)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f16_ts(tmem + TM_O, tmem + TM_UH + kk * 8,
                               sdesc_sw128(sb + OFF_PG + p * 8192 + kk * 32, 16, 1024), ID_O, 1u);
                mma_commit(&bars[B_ODONE]);
                mma_commit(&bars[B_PFREE + p]);
                last_bar = B_PFREE + p;
                last_par = (c >> 1) & 1;
            }
            // UMMAs complete in issue order: the last commit covers everything issued
            if (last_bar >= 0) ctl.drain(last_bar, last_par);
        }
    } else if (warp == 3) {
        // ================================================================ gate warp
        // lane l owns rows 2l, 2l+1 of each chunk; values of chunk c+1 are fetched one
        // chunk ahead to hide the HBM latency
        float g_nx[2] = {0.f, 0.f}, b_nx[2] = {0.f, 0.f};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int t = 2 * lane + e;
            if (t < L) {
                if (GATED) g_nx[e] = g[row0 + t];
                b_nx[e] = beta[row0 + t];
            }
        }
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kStages;
            float *vec = vec_of(c);
            // the buffer of chunk c - 3 is free once the state group is done with it
            if (c >= kStages) {
                int w = 1;
                if (lane == 0) w = ctl.wait_lazy(B_VFREE + s, ((c - kStages) / kStages) & 1) ? 1 : 0;
                if (__shfl_sync(0xffffffffu, w, 0) == 0) break;
            }
            const float g0 = g_nx[0], g1 = g_nx[1], b0 = b_nx[0], b1 = b_nx[1];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int t = (c + 1) * kC + 2 * lane + e;
                g_nx[e] = (GATED && c + 1 < nchunks && t < L) ? g[row0 + t] : 0.f;
                b_nx[e] = (c + 1 < nchunks && t < L) ? beta[row0 + t] : 0.f;
            }
            // inclusive scan of the 64 log-decays (pairs, then a warp scan of pair sums)
            float x = g0 + g1;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, off);
                if (lane >= off) x += y;
            }
            const float G1 = x, G0 = x - g1;
            const float Glast = __shfl_sync(0xffffffffu, x, 31);
            const bool fast = Glast >= kFastDecayLimit;
            vec[V_G + 2 * lane] = G0;
            vec[V_G + 2 * lane + 1] = G1;
            vec[V_B + 2 * lane] = b0;
            vec[V_B + 2 * lane + 1] = b1;
            vec[V_GAM + 2 * lane] = GATED ? __expf(G0) : 1.f;
            vec[V_GAM + 2 * lane + 1] = GATED ? __expf(G1) : 1.f;
            vec[V_D + 2 * lane] = GATED ? __expf(Glast - G0) : 1.f;
            vec[V_D + 2 * lane + 1] = GATED ? __expf(Glast - G1) : 1.f;
            vec[V_IG + 2 * lane] = (GATED && fast) ? __expf(-G0) : 1.f;
            vec[V_IG + 2 * lane + 1] = (GATED && fast) ? __expf(-G1) : 1.f;
            if (lane == 0) reinterpret_cast<int *>(vec)[V_FAST] = fast ? 1 : 0;
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_VEC + s]);
        }
    } else if (warp >= kGroupS && warp < kGroupS + 4) {
        // ================================================================ state group
        const int v = tid - kGroupS * 32;                // = TMEM lane (value column v)
        const bool lead = (v == 0);
        const int head = zc % H;                         // head of this row (dense and packed grids)
        float *xn = reinterpret_cast<float *>(smem + OFF_XN);
        const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        {
            // S^T row v = column v of the initial state (a warp reads 32 consecutive floats)
            const float *src = s0 ? s0 + static_cast<size_t>(bh) * kD * kD + v : nullptr;
#pragma unroll 1
            for (int cc = 0; cc < 8; ++cc) {
                float r[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) r[e] = src ? src[static_cast<size_t>(cc * 16 + e) * kD] : 0.f;
                tmem_st16(trow + TM_S + cc * 16, r);
            }
            tmem_wait_st();
        }
        int stored = 0;   // chunks whose output tile has been stored
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const float *vec = vec_of(c);
            // ---- S(c) complete: S^T row v -> -S^T fp16 pairs; S^T <- gamma_last S^T
            if (!ctl.group_wait_all({c >= 1 ? static_cast<int>(B_SDONE) : -1, B_VEC + c % kStages},
                                    {static_cast<uint32_t>(c - 1) & 1u, static_cast<uint32_t>(c / kStages) & 1u},
                                    kBarS, lead))
                break;
            tc_fence_after();
            {
                const float gl = GATED ? vec[V_GAM + 63] : 1.f;
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    float sv[32];
                    ld_cols<32>(trow + TM_S + h * 32, sv);
                    float hv[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) hv[e] = __uint_as_float(pack_h2(-sv[2 * e], -sv[2 * e + 1]));
                    tmem_st16(trow + TM_SH + h * 16, hv);
                    if (GATED) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) sv[e] *= gl;
                        tmem_st16(trow + TM_S + h * 32, *reinterpret_cast<float (*)[16]>(sv));
                        tmem_st16(trow + TM_S + h * 32 + 16, *reinterpret_cast<float (*)[16]>(sv + 16));
                    }
                }
                tmem_wait_st();
            }
            tc_fence_before();
            named_bar(kBarS, 128);
            if (lead) mbar_arrive(&bars[B_SRDY]);
            // ---- output of chunk c-1 (complete since its P Ut): read it, release O^T; then the
            //      W epilogue of chunk c (W^T row j = TMEM lane v -> fp16 MN-major W in the V slot
            //      of its stage, which U has consumed), then store the output tile
            float ov[64];
            if (c >= 1) {
                if (!ctl.group_wait(B_ODONE, (c - 1) & 1, kBarS, lead)) break;
                tc_fence_after();
                ld_cols<64>(trow + TM_O, ov);
                tc_fence_before();
                named_bar(kBarS, 128);
                if (lead) mbar_arrive(&bars[B_OFREE]);
            }
            if (!ctl.group_wait(B_WU, c & 1, kBarS, lead)) break;
            tc_fence_after();
            store_w_row(trow + TM_W, sb + (c % kStages) * kStageBytes + ST_W, v);
            fence_proxy_async();
            tc_fence_before();
            named_bar(kBarS, 128);
            if (lead) mbar_arrive(&bars[B_WRDY]);
            if (c >= 1) {
                const int cp = c - 1;
                const size_t elem0 = (row0 + static_cast<size_t>(cp) * kC) * kD + v;
                if constexpr (OPTS) {
                    store_out_rows_group(ov, out, elem0, kC, head, v, kBarS, xn, xn + 256);
                } else {
                    float *ocol = static_cast<float *>(out.o) + elem0;
#pragma unroll
                    for (int r = 0; r < 64; ++r) ocol[static_cast<size_t>(r) * kD] = ov[r];
                }
                stored = c;
            }
            // ---- Ut^T row v -> fp16 pairs, plain (output) and scaled by d_s (state update)
            if (!ctl.group_wait(B_ADONE, c & 1, kBarS, lead)) break;
            tc_fence_after();
            {
                float u[64];
                ld_cols<64>(trow + TM_U, u);
                float uh[32], ud[32];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const float4 d4 = GATED ? *reinterpret_cast<const float4 *>(vec + V_D + 2 * e)
                                            : make_float4(1.f, 1.f, 1.f, 1.f);
                    uh[e] = __uint_as_float(pack_h2(u[2 * e], u[2 * e + 1]));
                    uh[e + 1] = __uint_as_float(pack_h2(u[2 * e + 2], u[2 * e + 3]));
                    ud[e] = __uint_as_float(pack_h2(d4.x * u[2 * e], d4.y * u[2 * e + 1]));
                    ud[e + 1] = __uint_as_float(pack_h2(d4.z * u[2 * e + 2], d4.w * u[2 * e + 3]));
                }
                tmem_st16(trow + TM_UH, *reinterpret_cast<float (*)[16]>(uh));
                tmem_st16(trow + TM_UH + 16, *reinterpret_cast<float (*)[16]>(uh + 16));
                tmem_st16(trow + TM_UD, *reinterpret_cast<float (*)[16]>(ud));
                tmem_st16(trow + TM_UD + 16, *reinterpret_cast<float (*)[16]>(ud + 16));
                tmem_wait_st();
            }
            tc_fence_before();
            named_bar(kBarS, 128);
            if (lead) {
                mbar_arrive(&bars[B_URDY]);
                mbar_arrive(&bars[B_VFREE + c % kStages]);
            }
        }
        // ---- last output tile and the final state
        if (nchunks > 0 && stored == nchunks - 1) {
            const int cp = nchunks - 1;
            if (ctl.group_wait(B_ODONE, cp & 1, kBarS, lead)) {
                tc_fence_after();
                float ov[64];
                ld_cols<64>(trow + TM_O, ov);
                const int n = L - cp * kC;
                const size_t elem0 = (row0 + static_cast<size_t>(cp) * kC) * kD + v;
                if constexpr (OPTS) {
                    store_out_rows_group(ov, out, elem0, n, head, v, kBarS, xn, xn + 256);
                } else {
                    float *ocol = static_cast<float *>(out.o) + elem0;
#pragma unroll
                    for (int r = 0; r < 64; ++r)
                        if (r < n) ocol[static_cast<size_t>(r) * kD] = ov[r];
                }
                stored = nchunks;
            }
        }
        if (s_final && stored == nchunks) {
            // column v of the final state (a warp writes 32 consecutive floats); with no chunk
            // the state is the initial one
            float *dst = s_final + static_cast<size_t>(bh) * kD * kD + v;
#pragma unroll 1
            for (int cc = 0; cc < 8; ++cc) {
                float sv[16];
                tmem_ld16(trow + TM_S + cc * 16, sv);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) dst[static_cast<size_t>(cc * 16 + e) * kD] = sv[e];
            }
        }
    } else if (warp >= kGroupT && warp < kGroupT + 4) {
        // ================================================================ solve group
        // T = (I + A)^-1 of each chunk: the 16 x 16 diagonal blocks D_i = (I + A_ii)^-1 by
        // right-looking substitution (warp i); then the two 32 x 32 diagonal blocks
        // (T_10 = -D_1 A_10 D_0, T_32 = -D_3 A_32 D_2); then the lower-left 32 x 32 block
        // by doubling, T_BL = -T_BR (A_BL T_TL), as X_ij = A_{i,0..1} T_{0..1,j} followed by
        // T_2j = -D_2 X_2j, T_3j = -(T_32 X_2j + D_3 X_3j). Blocks of T are kept in fp32 (Tf)
        // for the products that follow and copied, once final, into the fp16 factors
        // T1 = T diag(beta gamma), T2 = T diag(beta) (K-major rows r); the upper blocks of
        // T1/T2 are zero from the start.
        const int t = tid - kGroupT * 32;                // 0..127
        const int bi = warp - kGroupT, cl = lane & 15;
        for (int i = t; i < 16384 / 16; i += 128)
            *reinterpret_cast<uint4 *>(smem + OFF_T1 + i * 16) = make_uint4(0u, 0u, 0u, 0u);
        float *Tf = reinterpret_cast<float *>(smem + OFF_TF);   // Tf[r * kTP + c] = T[r][c]
        float *Rw = reinterpret_cast<float *>(smem + OFF_R);
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const int p = c & 1;
            const float *vec = vec_of(c);
            const __half *At = reinterpret_cast<const __half *>(smem + OFF_AT + p * kAtBytes);   // At[s*64+r] = A[r][s]
            auto a_at = [&](int r, int s) { return __half2float(At[s * 64 + r]); };
            if (!ctl.group_wait_all({B_ATRDY + p, B_VEC + c % kStages},
                                    {static_cast<uint32_t>(c >> 1) & 1u, static_cast<uint32_t>(c / kStages) & 1u},
                                    kBarT, t == 0))
                break;
            // one 16 x 16 block (bi2, bj2) of Tf -> T1/T2; lane: row lane / 2, 8 columns
            auto emit = [&](int bi2, int bj2) {
                __syncwarp();
                const int r = 16 * bi2 + (lane >> 1), c0 = 16 * bj2 + 8 * (lane & 1);
                const float4 b0 = *reinterpret_cast<const float4 *>(vec + V_B + c0);
                const float4 b1 = *reinterpret_cast<const float4 *>(vec + V_B + c0 + 4);
                float4 g0 = make_float4(1.f, 1.f, 1.f, 1.f), g1 = g0;
                if (GATED) {
                    g0 = *reinterpret_cast<const float4 *>(vec + V_GAM + c0);
                    g1 = *reinterpret_cast<const float4 *>(vec + V_GAM + c0 + 4);
                }
                const float4 t0 = *reinterpret_cast<const float4 *>(Tf + r * kTP + c0);
                const float4 t1v = *reinterpret_cast<const float4 *>(Tf + r * kTP + c0 + 4);
                const float u[8] = {t0.x * b0.x, t0.y * b0.y, t0.z * b0.z, t0.w * b0.w,
                                    t1v.x * b1.x, t1v.y * b1.y, t1v.z * b1.z, t1v.w * b1.w};
                const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
                const uint32_t off = sw128(r, c0 >> 3);
                st_shared_v4(sb + OFF_T2 + off, pack_h2(u[0], u[1]), pack_h2(u[2], u[3]), pack_h2(u[4], u[5]),
                             pack_h2(u[6], u[7]));
                st_shared_v4(sb + OFF_T1 + off, pack_h2(u[0] * gg[0], u[1] * gg[1]), pack_h2(u[2] * gg[2], u[3] * gg[3]),
                             pack_h2(u[4] * gg[4], u[5] * gg[5]), pack_h2(u[6] * gg[6], u[7] * gg[7]));
            };
            // diagonal block bi: lane = column (lanes 16-31 mirror 0-15)
            {
                float acc[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) acc[i] = (i == cl) ? 1.f : 0.f;
                // column s2 of A_ii: A[16 bi + i][16 bi + s2] (zero for i <= s2), 16 halves; the
                // next step's column is loaded while this step's multiply-adds run
                const uint4 *acol = reinterpret_cast<const uint4 *>(At + 16 * bi * 64 + 16 * bi);
                uint4 cur0 = acol[0], cur1 = acol[1];
#pragma unroll
                for (int s2 = 0; s2 < 15; ++s2) {
                    uint4 nx0 = cur0, nx1 = cur1;
                    if (s2 < 14) {
                        if (s2 + 1 < 7) nx0 = acol[(s2 + 1) * 8];
                        nx1 = acol[(s2 + 1) * 8 + 1];
                    }
                    const float xs = acc[s2];
#pragma unroll
                    for (int k8 = 0; k8 < 2; ++k8) {
                        if (8 * k8 + 7 <= s2) continue;          // rows of this group are not below s2
                        const uint4 a8 = k8 == 0 ? cur0 : cur1;
                        const __half2 *h2 = reinterpret_cast<const __half2 *>(&a8);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 a2 = __half22float2(h2[e]);
                            acc[8 * k8 + 2 * e] = fmaf(-a2.x, xs, acc[8 * k8 + 2 * e]);
                            acc[8 * k8 + 2 * e + 1] = fmaf(-a2.y, xs, acc[8 * k8 + 2 * e + 1]);
                        }
                    }
                    cur0 = nx0;
                    cur1 = nx1;
                }
                if (lane < 16) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) Tf[(16 * bi + i) * kTP + 16 * bi + cl] = acc[i];
                }
            }
            // the T factors of chunk c-1 must have been read by its W/U before they are overwritten
            const bool ok = ctl.group_wait(B_WU, (c - 1) & 1, kBarT, t == 0 && c >= 1);
            if (ok) {
                emit(bi, bi);
                // level 1 (warps 0, 1): T_10 = -D_1 (A_10 D_0), T_32 = -D_3 (A_32 D_2)
                if (bi < 2) {
                    const int i = 2 * bi + 1, j = 2 * bi;
                    float *R = Rw + bi * 256;
                    float acc2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                    block_mm<2>(acc2, [&](int r, int k) { return a_at(16 * i + r, 16 * j + k); },
                                [&](int k, int n) { return Tf[(16 * j + k) * kTP + 16 * j + n]; }, lane);
                    block_store(acc2, [&](int r, int n, float x) { R[r * 16 + n] = x; }, lane, 1.f);
                    __syncwarp();
                    float acc3[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                    block_mm<2>(acc3, [&](int r, int k) { return Tf[(16 * i + r) * kTP + 16 * i + k]; },
                                [&](int k, int n) { return R[k * 16 + n]; }, lane);
                    block_store(acc3, [&](int r, int n, float x) { Tf[(16 * i + r) * kTP + 16 * j + n] = x; }, lane,
                                -1.f);
                    emit(i, j);
                }
                named_bar(kBarT, 128);
                // level 2 (warp w -> block (i, j) = (2 + w / 2, w % 2)): X_ij = A_{i,0..1} T_{0..1,j}
                const int ii = 2 + (bi >> 1), jj = bi & 1;
                {
                    float acc2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                    if (jj == 0)
                        block_mm<4>(acc2, [&](int r, int k) { return a_at(16 * ii + r, k); },
                                    [&](int k, int n) { return Tf[k * kTP + n]; }, lane);
                    else
                        block_mm<2>(acc2, [&](int r, int k) { return a_at(16 * ii + r, 16 + k); },
                                    [&](int k, int n) { return Tf[(16 + k) * kTP + 16 + n]; }, lane);
                    float *R = Rw + bi * 256;
                    block_store(acc2, [&](int r, int n, float x) { R[r * 16 + n] = x; }, lane, 1.f);
                }
                named_bar(kBarT, 128);
                if (t == 0) mbar_arrive(&bars[B_ATFREE + p]);      // the last read of A^T is done
                // level 3: T_2j = -D_2 X_2j,  T_3j = -(T_32 X_2j + D_3 X_3j)
                {
                    const float *X2 = Rw + jj * 256, *X3 = Rw + (2 + jj) * 256;
                    float acc3[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                    if (ii == 2)
                        block_mm<2>(acc3, [&](int r, int k) { return Tf[(32 + r) * kTP + 32 + k]; },
                                    [&](int k, int n) { return X2[k * 16 + n]; }, lane);
                    else
                        block_mm<4>(acc3, [&](int r, int k) { return Tf[(48 + r) * kTP + 32 + k]; },
                                    [&](int k, int n) { return k < 16 ? X2[k * 16 + n] : X3[(k - 16) * 16 + n]; },
                                    lane);
                    // block (ii, jj) of Tf is read by no other warp at this level
                    block_store(acc3, [&](int r, int n, float x) { Tf[(16 * ii + r) * kTP + 16 * jj + n] = x; },
                                lane, -1.f);
                    emit(ii, jj);
                }
            }
            fence_proxy_async();
            named_bar(kBarT, 128);
            if (!ok) break;                                // uniform: the verdict came from the barrier
            if (t == 0) mbar_arrive(&bars[B_TRDY]);
        }
    } else if (warp >= kGroupM) {
        // ================================================================ prep group
        // per chunk c: the A / P masks from the Gram, K, V -> fp16 and Q -> -Q' in place
        const int m = tid - kGroupM * 32;                // 0..127 = TMEM lane of the Gram row
        const bool lead = (m == 0);
        const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            {
                const int s = c % kStages, p = c & 1;
                const float *vec = vec_of(c);
                uint8_t *st = smem + s * kStageBytes;
                // the Gram and gate values of chunk c; P and A^T of parity p free (chunk c-2 done)
                if (!ctl.group_wait_all({B_GRAM, B_VEC + s, c >= 2 ? B_PFREE + p : -1, c >= 2 ? B_ATFREE + p : -1},
                                        {static_cast<uint32_t>(c) & 1u, static_cast<uint32_t>(c / kStages) & 1u,
                                         static_cast<uint32_t>((c - 2) >> 1) & 1u, static_cast<uint32_t>((c - 2) >> 1) & 1u},
                                        kBarM, lead))
                    break;
                tc_fence_after();
                const bool fast = !GATED || reinterpret_cast<const int *>(vec)[V_FAST] != 0;
                // ---- Gram row m: rows 0-63 -> A^T (fp16), rows 64-127 -> scale Gamma o Q K^T (P)
                {
                    float x[64];
                    ld_cols<64>(trow + TM_G, x);
                    tc_fence_before();
                    named_bar(kBarM, 128);                       // every Gram row has been read
                    if (lead) mbar_arrive(&bars[B_GFREE]);
                    const int r = m & 63;
                    // x[e] <- the masked, decayed Gram value of column e, with every factor read
                    // from shared memory before the first store (so no store orders a reload)
                    {
                        const float br = vec[V_B + r], gr = vec[V_GAM + r], Gr = vec[V_G + r];
                        const float lead_r = m < 64 ? br * gr : scale * gr;
                        const int lim = m < 64 ? r : r + 1;     // A: s < r; P: s <= r
                        if (fast) {
#pragma unroll
                            for (int e4 = 0; e4 < 64; e4 += 4) {
                                const float4 ig = *reinterpret_cast<const float4 *>(vec + V_IG + e4);
                                x[e4] = e4 < lim ? lead_r * ig.x * x[e4] : 0.f;
                                x[e4 + 1] = e4 + 1 < lim ? lead_r * ig.y * x[e4 + 1] : 0.f;
                                x[e4 + 2] = e4 + 2 < lim ? lead_r * ig.z * x[e4 + 2] : 0.f;
                                x[e4 + 3] = e4 + 3 < lim ? lead_r * ig.w * x[e4 + 3] : 0.f;
                            }
                        } else {
                            const float f = m < 64 ? br : scale;
#pragma unroll
                            for (int e4 = 0; e4 < 64; e4 += 4) {
                                const float4 gs = *reinterpret_cast<const float4 *>(vec + V_G + e4);
                                x[e4] = e4 < lim ? f * __expf(Gr - gs.x) * x[e4] : 0.f;
                                x[e4 + 1] = e4 + 1 < lim ? f * __expf(Gr - gs.y) * x[e4 + 1] : 0.f;
                                x[e4 + 2] = e4 + 2 < lim ? f * __expf(Gr - gs.z) * x[e4 + 2] : 0.f;
                                x[e4 + 3] = e4 + 3 < lim ? f * __expf(Gr - gs.w) * x[e4 + 3] : 0.f;
                            }
                        }
                    }
                    if (m < 64) {
                        __half *At = reinterpret_cast<__half *>(smem + OFF_AT + p * kAtBytes);   // At[s*64+r]
#pragma unroll
                        for (int e = 0; e < 64; ++e) At[e * 64 + r] = __float2half_rn(x[e]);
                    } else {
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch)
                            st_shared_v4(sb + OFF_PG + p * 8192 + sw128(r, ch), pack_h2(x[8 * ch], x[8 * ch + 1]),
                                         pack_h2(x[8 * ch + 2], x[8 * ch + 3]), pack_h2(x[8 * ch + 4], x[8 * ch + 5]),
                                         pack_h2(x[8 * ch + 6], x[8 * ch + 7]));
                    }
                }
                fence_proxy_async();
                named_bar(kBarM, 128);
                if (lead) mbar_arrive(&bars[B_ATRDY + p]);
                // ---- K and V: 2048 chunks of 16 B at [0,8K) [16K,24K) [32K,48K) -> fp16
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    uint4 xv[8];
                    uint32_t offs[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const uint32_t idx = static_cast<uint32_t>((part * 8 + i) * 128 + m);   // 0..2047
                        const uint32_t reg = idx >> 9;                                           // 0..3
                        offs[i] = (reg < 2 ? reg * 16384u : 32768u + (reg - 2) * 8192u) + (idx & 511u) * 16u;
                        xv[i] = *reinterpret_cast<const uint4 *>(st + offs[i]);
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        xv[i].x = pack_h2(bf_lo(xv[i].x), bf_hi(xv[i].x));
                        xv[i].y = pack_h2(bf_lo(xv[i].y), bf_hi(xv[i].y));
                        xv[i].z = pack_h2(bf_lo(xv[i].z), bf_hi(xv[i].z));
                        xv[i].w = pack_h2(bf_lo(xv[i].w), bf_hi(xv[i].w));
                        *reinterpret_cast<uint4 *>(st + offs[i]) = xv[i];
                    }
                }
                // ---- Q: 1024 chunks at [8K,16K) [24K,32K) -> -Q' = fp16(-scale gamma_r q_r)
                {
                    uint4 xv[8];
                    uint32_t offs[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const uint32_t idx = static_cast<uint32_t>(i * 128 + m);                 // 0..1023
                        offs[i] = ST_Q0 + (idx >> 9) * 16384u + (idx & 511u) * 16u;
                        xv[i] = *reinterpret_cast<const uint4 *>(st + offs[i]);
                    }
                    float fq[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) fq[i] = -scale * vec[V_GAM + ((offs[i] & 8191u) >> 7)];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float f = fq[i];
                        xv[i].x = pack_h2(f * bf_lo(xv[i].x), f * bf_hi(xv[i].x));
                        xv[i].y = pack_h2(f * bf_lo(xv[i].y), f * bf_hi(xv[i].y));
                        xv[i].z = pack_h2(f * bf_lo(xv[i].z), f * bf_hi(xv[i].z));
                        xv[i].w = pack_h2(f * bf_lo(xv[i].w), f * bf_hi(xv[i].w));
                        *reinterpret_cast<uint4 *>(st + offs[i]) = xv[i];
                    }
                }
                fence_proxy_async();
                named_bar(kBarM, 128);
                if (lead) mbar_arrive(&bars[B_CONV + s]);
            }
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

template <bool GATED, bool OPTS>
gdn_status_t launch_gdn_t(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv, const float *beta,
                          const float *g, const OutArgs &out, const float *s0, float *s_final, const int *cu,
                          int nctas, int H, int L, float scale, cudaStream_t stream) {
    auto kern = tc_gdn_kernel<GATED, OPTS>;
    if (!ensure_smem_limit(reinterpret_cast<const void *>(kern), kSmemAlloc)) return GDN_ERR_CUDA;
    unsigned *err = device_error_word();
    if (!err) return GDN_ERR_CUDA;
    kern<<<nctas, kThreads, kSmemAlloc, stream>>>(mq, mk, mv, beta, g, out, s0, s_final, cu, H, L, scale,
                                                  wait_limit_cycles(), err);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace

bool tc_supported(gdn_dtype_t in_dtype, int dk, int dv, int chunk) {
    return in_dtype == GDN_BF16 && dk == 128 && dv == 128 && chunk == 64 && encode_fn() != nullptr;
}

gdn_status_t launch_tc_gdn(const void *q, const void *k, const void *v, const float *beta, const float *g,
                           void *o, const float *s0, float *s_final, const int *cu, int B, int H, int L,
                           float scale, FwdOpts oo, cudaStream_t stream) {
    const int nctas = B * H;                 // one CTA per (sequence, head)
    // few (sequence, head) pairs: the cluster form spreads each chunk's prep over two more SMs
    if (tc_gdn_cluster_fits(nctas))
        return launch_tc_gdn_cluster(q, k, v, beta, g, o, s0, s_final, cu, B, H, L, scale, oo, stream);
    const OutArgs out = make_out_args(o, v, oo);
    const int rows = cu ? H : B * H;         // rows of the (rows, L) token grid
    CUtensorMap mq, mk, mv;
    if (!make_qkv_map(&mq, q, L, rows) || !make_qkv_map(&mk, k, L, rows) || !make_qkv_map(&mv, v, L, rows))
        return GDN_ERR_CUDA;
    const bool opts = oo.bf16 || oo.dskip != nullptr || oo.xnorm != kXNormNone;   // the general output epilogue
    if (g) return opts ? launch_gdn_t<true, true>(mq, mk, mv, beta, g, out, s0, s_final, cu, nctas, H, L, scale, stream)
                       : launch_gdn_t<true, false>(mq, mk, mv, beta, g, out, s0, s_final, cu, nctas, H, L, scale, stream);
    return opts ? launch_gdn_t<false, true>(mq, mk, mv, beta, g, out, s0, s_final, cu, nctas, H, L, scale, stream)
                : launch_gdn_t<false, false>(mq, mk, mv, beta, g, out, s0, s_final, cu, nctas, H, L, scale, stream);
}

}  // namespace gdn
