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
//   Gram   [K;Q] K^T (the Q K^T half is used)           one M=128 UMMA
//   state  S^T <- gamma_last S^T + V^T (diag(d) K)        M=128 (value rows)
//   out    O^T = S^T Q'^T + V^T P^T,  Q' = diag(scale gamma) Q,
//          P = scale (Q K^T o Gamma) (s <= r)
// One CTA per (batch, head) walks its chunks in order. The fp32 state S^T (lane =
// value column) and its fp16 copy (the A operand of S^T Q'^T) live in tensor memory
// for the whole sequence. The state chain per chunk is one fp32 -> fp16 pass over
// S^T (with the decay) and four state-update UMMAs; everything else (tile loads,
// the Gram, P, the fp16 operand conversion, the output products and the output
// stores) is pipelined around it by dedicated warps.
//
// Warp roles (640 threads):
//   warp 0      TMA producer (4-stage ring of Q, K, V tiles)
//   warp 1      Gram issuer
//   warp 2      gate warp (gated only): G, gamma, d, exp(-G) per chunk
//   warp 3      chain issuer: state update, then S^T Q'^T and V^T P^T
//   warps 4-7   state group: S^T -> fp16 copy, S^T <- gamma_last S^T
//   warps 8-11  output group: O^T -> o
//   warps 12-15 converter: Q -> Q', K -> diag(d) K, in place
//   warps 16-17 V -> fp16, in place
//   warps 18-19 P writers (Gram rows 64-127: Q K^T)
// Hand-offs are mbarriers with one arrival each; resources used by consecutive
// chunks (O^T, fp16 S, P, gate values) are double-buffered and their barriers are
// indexed by chunk parity, per-stage barriers by stage.
//
// UMMA operands are fp16: the bf16 tiles are converted in place once the Gram has
// read them (exact in fp16 range), the computed operands (S, P, Q', diag(d) K) are
// rounded to fp16. Shared-memory operands use the 128-byte swizzled layouts.
#include "tc_ctl.cuh"

namespace gdn {

namespace {
using namespace ptx;

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kThreads = 640;
constexpr int kStages = 4;
constexpr float kFastDecayLimit = -60.f;   // G_last >= this: Gamma = gamma_r * exp(-G_s)

// ---- shared memory map (byte offsets from a 1024-aligned base) ------------------
constexpr uint32_t kStageBytes = 49152;
// Each key half holds the 64 K rows directly followed by the 64 Q rows, so [K;Q] is
// one 128-row operand of the Gram.
constexpr uint32_t ST_K0 = 0, ST_Q0 = 8192, ST_K1 = 16384, ST_Q1 = 24576, ST_V0 = 32768, ST_V1 = 40960;
constexpr uint32_t OFF_PG = kStages * kStageBytes;   // 2 x P, K-major 64 x 64 fp16
constexpr uint32_t OFF_VEC = OFF_PG + 16384;         // 2 x {G, gamma, d, exp(-G), flag}
constexpr uint32_t kVecBytes = 1536;
constexpr int V_G = 0, V_GAM = 64, V_D = 128, V_IG = 192, V_FAST = 256;
constexpr uint32_t OFF_XN = OFF_VEC + 2 * kVecBytes;   // output-normalisation scratch (384 fp32)
constexpr uint32_t OFF_BAR = OFF_XN + 1536;
constexpr uint32_t kSmemBytes = OFF_BAR + 512;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;   // slack to align the base to 1024 B
static_assert(kSmemAlloc <= 232448, "shared memory budget");
static_assert(OFF_PG % 1024 == 0, "UMMA tiles need 1024-B alignment");

// ---- tensor memory columns (512 allocated) ----------------------------------------
constexpr uint32_t TM_S = 0;      // S^T fp32: lane = value v, 128 key columns
constexpr uint32_t TM_G = 128;    // 2 x [K;Q] K^T: lanes 64-127 Q K^T (row r, column s)
constexpr uint32_t TM_SH = 256;   // 2 x S^T fp16 (A operand): 64 columns of key pairs
constexpr uint32_t TM_O = 384;    // 2 x O^T: lane = value v, 64 columns r

constexpr uint32_t ID_GRAM = idesc_f16(128, 64, false, false, false, /*bf16=*/true);
constexpr uint32_t ID_SQ = idesc_f16(128, 64, false, false);
constexpr uint32_t ID_ST = idesc_f16(128, 128, true, true);
constexpr uint32_t ID_PV = idesc_f16(128, 64, true, false);

// mbarriers. A parity wait for phase k is only correct while the producer cannot
// complete phase k+1 first: per-stage barriers are waited with parity (c / 4) & 1,
// per-parity ones with (c >> 1) & 1, single ones with c & 1.
enum : int {
    B_FULL = 0,      // [4] TMA -> Gram issuer, converter
    B_GREAD = 4,     // [4] Gram has read the bf16 Q, K tiles of the stage -> converter
    B_CONV = 8,      // [4] Q', diag(d) K of the stage written -> chain issuer
    B_SFREE = 12,    // [4] last UMMA reading the stage done -> TMA
    B_GATE = 16,     // [2] gate values of the chunk ready -> converter, P writers, state group
    B_ODONE = 20,    // [2] O^T of the chunk complete -> output group, gate warp, P writer
    B_OFREE = 22,    // [2] output group has read O^T -> chain issuer
    B_PREP = 24,     // [2] P of the chunk written -> chain issuer
    B_GRAM = 26,     // [2] Gram of the chunk done -> P writer
    B_GFREE = 28,    // [2] P writer has read the Gram -> Gram issuer
    B_VCONV = 30,    // [4] V of the stage converted to fp16 -> chain issuer
    B_SRDY = 34,     // fp16 S written and S decayed -> chain issuer
    B_SDONE = 35,    // state update done -> state group
    kNumBars = 36
};
constexpr int kBarState = 1, kBarOut = 2, kBarP = 3, kBarConv = 4, kBarV = 5;   // named barriers

template <int N>
__device__ __forceinline__ void ld_cols(uint32_t taddr, float (&v)[N]) {
    static_assert(N % 16 == 0, "16-column pieces");
#pragma unroll
    for (int cc = 0; cc < N / 16; ++cc) tmem_ld16(taddr + cc * 16, *reinterpret_cast<float (*)[16]>(v + cc * 16));
    tmem_wait_ld();
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
// 8 bf16 (one 16-byte chunk) -> 8 fp16 scaled by f
__device__ __forceinline__ uint4 scale_chunk(uint4 x, float f) {
    x.x = pack_h2(f * bf_lo(x.x), f * bf_hi(x.x));
    x.y = pack_h2(f * bf_lo(x.y), f * bf_hi(x.y));
    x.z = pack_h2(f * bf_lo(x.z), f * bf_hi(x.z));
    x.w = pack_h2(f * bf_lo(x.w), f * bf_hi(x.w));
    return x;
}

// NARROW: head sizes dk_arg, dv_arg of 64 or 128 (tiles past them load as zeros; plain fp32
// output only); otherwise both are 128 and the arguments are ignored.
template <bool GATED, bool OPTS, bool NARROW>
__global__ void __launch_bounds__(kThreads, 1)
tc_la_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ g, const OutArgs out,
             const float *__restrict__ s0, float *__restrict__ s_final, const int *__restrict__ cu, int H,
             int Lrow, float scale, int dk_arg, int dv_arg, long long wait_limit, unsigned *__restrict__ err_word) {
    static_assert(!(NARROW && OPTS), "the output options need dv = 128");
    const int dk_in = NARROW ? dk_arg : kD, dv_in = NARROW ? dv_arg : kD;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base derived by pointer arithmetic on the shared array, so the
    // compiler keeps every access below in the shared address space (LDS/STS)
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kNumBars);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);   // CTA-wide abort flag
    const Ctl ctl{bars, abort_flag, err_word, wait_limit};

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // (sequence, head): state index; packed batches take their sequences longest first
    const int bh = cu ? longest_first(cu, blockIdx.x, H, gridDim.x / H) : blockIdx.x;
    const SeqSpan sp = seq_span(cu, bh, H, Lrow, err_word);
    const int L = sp.len;                               // tokens of this sequence
    const int zc = sp.head_row, ty0 = sp.t0;            // TMA head and first-token coordinates
    const int nchunks = (L + kC - 1) / kC;
    const size_t row0 = static_cast<size_t>(zc) * Lrow + ty0;   // first token row in the grid
    // extents the launch implies (bounds checks of the debug build): token rows of the grid, and
    // state elements
    const long long n_rows = static_cast<long long>(cu ? H : gridDim.x) * Lrow;
    const long long n_state = static_cast<long long>(gridDim.x) * dk_in * dv_in;

    if (tid == 0) {
        for (int b = 0; b < kNumBars; ++b) mbar_init(&bars[b], 1);
        abort_flag[0] = 0;
        fence_mbar_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    if (!GATED && tid < 128) {
        // constant gate values of the ungated case, in both buffers
        float *vec = reinterpret_cast<float *>(smem + OFF_VEC + (tid >> 6) * kVecBytes);
        const int i = tid & 63;
        vec[V_G + i] = 0.f;
        vec[V_GAM + i] = 1.f;
        vec[V_D + i] = 1.f;
        vec[V_IG + i] = 1.f;
        if (i == 0) reinterpret_cast<int *>(vec)[V_FAST] = 1;
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ================================================================ TMA producer
        if (lane == 0) {
            int last[kStages] = {-1, -1, -1, -1};
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % kStages;
                if (c >= kStages && !ctl.wait(B_SFREE + s, (c / kStages - 1) & 1)) break;
                uint8_t *st = smem + s * kStageBytes;
                uint64_t *fb = &bars[B_FULL + s];
                mbar_arrive_expect_tx(fb, kStageBytes);
                tma_load_3d(st + ST_Q0, &tm_q, fb, 0, ty0 + c * kC, zc);
                tma_load_3d(st + ST_K0, &tm_k, fb, 0, ty0 + c * kC, zc);
                tma_load_3d(st + ST_Q1, &tm_q, fb, 64, ty0 + c * kC, zc);
                tma_load_3d(st + ST_K1, &tm_k, fb, 64, ty0 + c * kC, zc);
                tma_load_3d(st + ST_V0, &tm_v, fb, 0, ty0 + c * kC, zc);
                tma_load_3d(st + ST_V1, &tm_v, fb, 64, ty0 + c * kC, zc);
                last[s] = c;
            }
            // never leave a copy in flight past the end of the CTA
            for (int s = 0; s < kStages; ++s)
                if (last[s] >= 0) ctl.drain(B_FULL + s, (last[s] / kStages) & 1);
        }
    } else if (warp == 1) {
        // ================================================================ Gram issuer
        if (lane == 0) {
            int last = -1;
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % kStages;
                const uint32_t stg = sb + s * kStageBytes;
                const int p = c & 1;
                if (!ctl.wait(B_FULL + s, (c / kStages) & 1)) break;
                if (c >= 2 && !ctl.wait(B_GFREE + p, ((c - 2) >> 1) & 1)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
                    mma_f16(tmem + TM_G + p * 64, sdesc_sw128(stg + ST_K0 + off, 16, 1024),
                            sdesc_sw128(stg + ST_K0 + off, 16, 1024), ID_GRAM, kk > 0);
                }
                mma_commit(&bars[B_GRAM + p]);
                mma_commit(&bars[B_GREAD + s]);
                last = c;
            }
            if (last >= 0) ctl.drain(B_GREAD + last % kStages, (last / kStages) & 1);
        }
    } else if (warp == 2) {
        // ================================================================ gate warp
        // lane l owns rows 2l, 2l+1 of each chunk; values of chunk c+1 are fetched one
        // chunk ahead to hide the HBM latency
        if (GATED) {
            float g_nx[2] = {0.f, 0.f};
#pragma unroll
            for (int e = 0; e < 2; ++e)
                if (2 * lane + e < L && in_bounds(static_cast<long long>(row0) + 2 * lane + e, n_rows, err_word))
                    g_nx[e] = g[row0 + 2 * lane + e];
#pragma unroll 1
            for (int c = 0; c < nchunks; ++c) {
                const int p = c & 1;
                float *vec = reinterpret_cast<float *>(smem + OFF_VEC + p * kVecBytes);
                // the gate values of parity p are free once chunk c-2 is complete
                if (c >= 2) {
                    int w = 1;
                    if (lane == 0) w = ctl.wait(B_ODONE + p, ((c - 2) >> 1) & 1) ? 1 : 0;
                    if (__shfl_sync(0xffffffffu, w, 0) == 0) break;
                }
                const float g0 = g_nx[0], g1 = g_nx[1];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int t = (c + 1) * kC + 2 * lane + e;
                    g_nx[e] = (c + 1 < nchunks && t < L && in_bounds(static_cast<long long>(row0) + t, n_rows, err_word))
                                  ? g[row0 + t] : 0.f;
                }
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
                vec[V_GAM + 2 * lane] = __expf(G0);
                vec[V_GAM + 2 * lane + 1] = __expf(G1);
                vec[V_D + 2 * lane] = __expf(Glast - G0);
                vec[V_D + 2 * lane + 1] = __expf(Glast - G1);
                vec[V_IG + 2 * lane] = fast ? __expf(-G0) : 1.f;
                vec[V_IG + 2 * lane + 1] = fast ? __expf(-G1) : 1.f;
                if (lane == 0) reinterpret_cast<int *>(vec)[V_FAST] = fast ? 1 : 0;
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_GATE + p]);
            }
        }
    } else if (warp == 3) {
        // ================================================================ chain issuer
        if (lane == 0) {
            int last_bar = -1, last_par = 0;
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % kStages, p = c & 1;
                const uint32_t stg = sb + s * kStageBytes;
                if (!ctl.wait(B_SRDY, c & 1)) break;
                if (!ctl.wait(B_CONV + s, (c / kStages) & 1)) break;
                if (!ctl.wait(B_VCONV + s, (c / kStages) & 1)) break;
                tc_fence_after();
                // S^T += V^T (diag(d) K): the serial state chain goes first
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f16(tmem + TM_S, sdesc_sw128(stg + ST_V0 + kk * 2048, 8192, 1024),
                            sdesc_sw128(stg + ST_K0 + kk * 2048, 16384, 1024), ID_ST, 1u);
                mma_commit(&bars[B_SDONE]);
                last_bar = B_SDONE;
                last_par = c & 1;
                // O^T = S^T Q'^T into the O buffer of parity p, once chunk c-2's output was read
                if (c >= 2 && !ctl.wait(B_OFREE + p, ((c - 2) >> 1) & 1)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
                    mma_f16_ts(tmem + TM_O + p * 64, tmem + TM_SH + p * 64 + kk * 8,
                               sdesc_sw128(stg + ST_Q0 + off, 16, 1024), ID_SQ, kk > 0);
                }
                if (!ctl.wait(B_PREP + p, (c >> 1) & 1)) {
                    // cover the UMMAs just issued by a commit, so the final drain waits for them
                    mma_commit(&bars[B_ODONE + p]);
                    last_bar = B_ODONE + p;
                    last_par = (c >> 1) & 1;
                    break;
                }
                tc_fence_after();
                // O^T += V^T P^T
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f16(tmem + TM_O + p * 64, sdesc_sw128(stg + ST_V0 + kk * 2048, 8192, 1024),
                            sdesc_sw128(sb + OFF_PG + p * 8192 + kk * 32, 16, 1024), ID_PV, 1u);
                mma_commit(&bars[B_ODONE + p]);
                mma_commit(&bars[B_SFREE + s]);
                last_bar = B_SFREE + s;
                last_par = (c / kStages) & 1;
            }
            // UMMAs complete in issue order: the last commit covers everything issued
            if (last_bar >= 0) ctl.drain(last_bar, last_par);
        }
    } else if (warp < 8) {
        // ================================================================ state group
        const int v = tid - 128;                          // TMEM lane = value column
        const bool lead = (v == 0);
        const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        float nf = 0.f;   // non-finite probe over the final state
        {
            // S^T row v = column v of the dk_in x dv_in initial state (a warp reads 32 consecutive
            // floats; rows and columns beyond it are zero)
            const float *src = s0 && v < dv_in ? s0 + static_cast<size_t>(bh) * dk_in * dv_in + v : nullptr;
#pragma unroll 1
            for (int cc = 0; cc < 8; ++cc) {
                float r[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    r[e] = src && cc * 16 < dk_in &&
                                   in_bounds(static_cast<long long>(bh) * dk_in * dv_in + static_cast<long long>(cc * 16 + e) * dv_in + v,
                                             n_state, err_word)
                               ? src[static_cast<size_t>(cc * 16 + e) * dv_in] : 0.f;
                tmem_st16(trow + TM_S + cc * 16, r);
            }
            tmem_wait_st();
        }
        int done = -1;   // last chunk whose state update this group has seen issued
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const int p = c & 1;
            const float *vec = reinterpret_cast<const float *>(smem + OFF_VEC + p * kVecBytes);
            if (c >= 1 && !ctl.group_wait(B_SDONE, (c - 1) & 1, kBarState, lead, 128)) break;
            if (GATED && !ctl.group_wait(B_GATE + p, (c >> 1) & 1, kBarState, lead, 128)) break;
            tc_fence_after();
            // S^T row v -> fp16 pairs (A operand of S^T Q'^T); S <- gamma_last S
            const float gl = GATED ? vec[V_GAM + 63] : 1.f;
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                float sv[32];
                ld_cols<32>(trow + TM_S + h * 32, sv);
                float hv[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) hv[e] = __uint_as_float(pack_h2(sv[2 * e], sv[2 * e + 1]));
                tmem_st16(trow + TM_SH + p * 64 + h * 16, hv);
                if (GATED) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) sv[e] *= gl;
                    tmem_st16(trow + TM_S + h * 32, *reinterpret_cast<float (*)[16]>(sv));
                    tmem_st16(trow + TM_S + h * 32 + 16, *reinterpret_cast<float (*)[16]>(sv + 16));
                }
            }
            tmem_wait_st();
            tc_fence_before();
            named_bar(kBarState, 128);
            if (lead) mbar_arrive(&bars[B_SRDY]);
            done = c;
        }
        // column v of the dk_in x dv_in final state (a warp writes 32 consecutive floats; lanes
        // v >= dv_in are whole warps and store nothing)
        if (s_final && nchunks == 0) {
            // empty sequence: the final state is the initial one (TMEM holds it)
            if (v < dv_in) {
                float *dst = s_final + static_cast<size_t>(bh) * dk_in * dv_in + v;
#pragma unroll 1
                for (int cc = 0; cc < dk_in / 16; ++cc) {
                    float sv[16];
                    tmem_ld16(trow + TM_S + cc * 16, sv);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        if (in_bounds(static_cast<long long>(bh) * dk_in * dv_in + static_cast<long long>(cc * 16 + e) * dv_in + v,
                                      n_state, err_word))
                            dst[static_cast<size_t>(cc * 16 + e) * dv_in] = sv[e];
                }
            }
        } else if (s_final && nchunks > 0 && done == nchunks - 1 &&
            ctl.group_wait(B_SDONE, (nchunks - 1) & 1, kBarState, lead, 128)) {
            tc_fence_after();
            if (v < dv_in) {
                float *dst = s_final + static_cast<size_t>(bh) * dk_in * dv_in + v;
#pragma unroll 1
                for (int cc = 0; cc < dk_in / 16; ++cc) {
                    float sv[16];
                    tmem_ld16(trow + TM_S + cc * 16, sv);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        probe_finite(nf, sv[e]);
                        if (in_bounds(static_cast<long long>(bh) * dk_in * dv_in + static_cast<long long>(cc * 16 + e) * dv_in + v,
                                      n_state, err_word))
                            dst[static_cast<size_t>(cc * 16 + e) * dv_in] = sv[e];
                    }
                }
            }
        }
        report_nonfinite(ctl.aborted() ? 0.f : nf, err_word);
    } else if (warp < 12) {
        // ================================================================ output group
        const int v = tid - 256;                          // TMEM lane = value column
        const bool lead = (v == 0);
        const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        const int head = zc % H;                          // head of this row (dense and packed grids)
        float *xn = reinterpret_cast<float *>(smem + OFF_XN);
        float nf = 0.f;   // non-finite probe over sampled output tiles
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const int p = c & 1;
            if (!ctl.group_wait(B_ODONE + p, (c >> 1) & 1, kBarOut, lead, 128)) break;
            tc_fence_after();
            float ov[64];
            ld_cols<64>(trow + TM_O + p * 64, ov);
            tc_fence_before();
            named_bar(kBarOut, 128);
            if (lead) mbar_arrive(&bars[B_OFREE + p]);
            const int n = min(kC, L - c * kC);
            if constexpr (OPTS) {
                store_out_rows_group(ov, out, (row0 + static_cast<size_t>(c) * kC) * kD + v, n, head, v, kBarOut, xn,
                                     xn + 256, probe_chunk(c, nchunks), nf);
            } else if (v < dv_in) {
                float *ocol = static_cast<float *>(out.o) + (row0 + static_cast<size_t>(c) * kC) * dv_in + v;
#pragma unroll
                for (int r = 0; r < 64; ++r)
                    if (r < n && in_bounds((static_cast<long long>(row0) + c * kC + r) * dv_in + v, n_rows * dv_in, err_word))
                        ocol[static_cast<size_t>(r) * dv_in] = ov[r];
                if (probe_chunk(c, nchunks)) probe_tile(nf, ov, n);
            }
        }
        report_nonfinite(ctl.aborted() ? 0.f : nf, err_word);
    } else if (warp >= 18) {
        // ================================================================ P writers
        // P = scale (Q K^T o Gamma), s <= r, row r (Gram lane 64 + r) -> PG (fp16)
        const int r = tid - 576;                          // 0..63
        const bool pl = (r == 0);
        const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const int p = c & 1;
            const float *vec = reinterpret_cast<const float *>(smem + OFF_VEC + p * kVecBytes);
            // PG of parity p is free once chunk c-2 is complete
            if (c >= 2 && !ctl.group_wait(B_ODONE + p, ((c - 2) >> 1) & 1, kBarP, pl, 64)) break;
            if (GATED && !ctl.group_wait(B_GATE + p, (c >> 1) & 1, kBarP, pl, 64)) break;
            if (!ctl.group_wait(B_GRAM + p, (c >> 1) & 1, kBarP, pl, 64)) break;
            tc_fence_after();
            const bool fast = !GATED || reinterpret_cast<const int *>(vec)[V_FAST] != 0;
            const float fr = scale * (GATED ? vec[V_GAM + r] : 1.f);
            const float Gr = GATED ? vec[V_G + r] : 0.f;
            const uint32_t prow = sb + OFF_PG + p * 8192;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float x[32];
                ld_cols<32>(trow + TM_G + p * 64 + h * 32, x);
                if (h == 1) {
                    // both halves of the Gram row are in registers: release the buffer
                    tc_fence_before();
                    named_bar(kBarP, 64);
                    if (pl) mbar_arrive(&bars[B_GFREE + p]);
                }
                if (fast) {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        x[e] = (32 * h + e <= r) ? fr * (GATED ? vec[V_IG + 32 * h + e] : 1.f) * x[e] : 0.f;
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        x[e] = (32 * h + e <= r) ? scale * __expf(Gr - vec[V_G + 32 * h + e]) * x[e] : 0.f;
                }
#pragma unroll
                for (int ch = 0; ch < 4; ++ch)
                    st_shared_v4(prow + sw128(r, 4 * h + ch), pack_h2(x[8 * ch], x[8 * ch + 1]),
                                 pack_h2(x[8 * ch + 2], x[8 * ch + 3]), pack_h2(x[8 * ch + 4], x[8 * ch + 5]),
                                 pack_h2(x[8 * ch + 6], x[8 * ch + 7]));
            }
            fence_proxy_async();
            named_bar(kBarP, 64);
            if (pl) mbar_arrive(&bars[B_PREP + p]);
        }
    } else if (warp >= 16) {
        // ================================================================ V converter
        // V (2 x 8 KB, 1024 chunks of 16 B) -> fp16 in place once the tiles have landed
        const int t = tid - 512;                          // 0..63
        const bool lead = (t == 0);
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kStages;
            if (!ctl.group_wait(B_FULL + s, (c / kStages) & 1, kBarV, lead, 64)) break;
            uint8_t *vt = smem + s * kStageBytes + ST_V0;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint4 x[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) x[i] = *reinterpret_cast<const uint4 *>(vt + ((h * 8 + i) * 64 + t) * 16);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    *reinterpret_cast<uint4 *>(vt + ((h * 8 + i) * 64 + t) * 16) = scale_chunk(x[i], 1.f);
            }
            fence_proxy_async();
            named_bar(kBarV, 64);
            if (lead) mbar_arrive(&bars[B_VCONV + s]);
        }
    } else {
        // ================================================================ Q / K converter
        // Q -> fp16(scale gamma_r q), K -> fp16(d_s k), V -> fp16, in place, once the Gram
        // has read the bf16 tiles
        const int t = tid - 384;                          // 0..127 (warps 12-15)
        const bool lead = (t == 0);
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kStages, p = c & 1;
            const float *vec = reinterpret_cast<const float *>(smem + OFF_VEC + p * kVecBytes);
            uint8_t *st = smem + s * kStageBytes;
            const int nvalid = min(kC, L - c * kC);
            if (!ctl.group_wait(B_FULL + s, (c / kStages) & 1, kBarConv, lead, 128)) break;
            if (GATED && !ctl.group_wait(B_GATE + p, (c >> 1) & 1, kBarConv, lead, 128)) break;
            if (!ctl.group_wait(B_GREAD + s, (c / kStages) & 1, kBarConv, lead, 128)) break;
            // 2 x 1024 chunks of 16 B; chunk i of a tensor sits in box i / 512 (key half),
            // row (i % 512) / 8 of that box (V is converted by the state group)
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                uint4 x[8];
                uint32_t off[8];
                float f[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint32_t idx = static_cast<uint32_t>(i * 128 + t);     // 0..1023
                    const uint32_t box = idx >> 9, row = (idx & 511u) >> 3;
                    if (part == 0) {
                        off[i] = ST_Q0 + box * 16384u + (idx & 511u) * 16u;
                        f[i] = scale * (GATED ? vec[V_GAM + row] : 1.f);
                    } else {
                        // rows past the end of the sequence (the next sequence of a packed
                        // batch, or TMA zero fill) must not reach the state
                        off[i] = ST_K0 + box * 16384u + (idx & 511u) * 16u;
                        f[i] = static_cast<int>(row) < nvalid ? (GATED ? vec[V_D + row] : 1.f) : 0.f;
                    }
                    x[i] = *reinterpret_cast<const uint4 *>(st + off[i]);
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) *reinterpret_cast<uint4 *>(st + off[i]) = scale_chunk(x[i], f[i]);
            }
            fence_proxy_async();
            named_bar(kBarConv, 128);
            if (lead) mbar_arrive(&bars[B_CONV + s]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <bool GATED, bool OPTS, bool NARROW = false>
gdn_status_t launch_la_t(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv, const float *g,
                         const OutArgs &out, const float *s0, float *s_final, const int *cu, int nctas, int H,
                         int L, float scale, cudaStream_t stream, int dk = kD, int dv = kD) {
    auto kern = tc_la_kernel<GATED, OPTS, NARROW>;
    if (!ensure_smem_limit(reinterpret_cast<const void *>(kern), kSmemAlloc)) return GDN_ERR_CUDA;
    unsigned *err = device_error_word();
    if (!err) return GDN_ERR_CUDA;
    kern<<<nctas, kThreads, kSmemAlloc, stream>>>(mq, mk, mv, g, out, s0, s_final, cu, H, L, scale, dk, dv,
                                                  wait_limit_cycles(), err);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace

gdn_status_t launch_tc_la(const void *q, const void *k, const void *v, const float *g, void *o,
                          const float *s0, float *s_final, const int *cu, int B, int H, int L, float scale,
                          FwdOpts oo, cudaStream_t stream) {
    const int nctas = B * H;                 // one CTA per (sequence, head)
    const OutArgs out = make_out_args(o, v, oo);
    const int rows = cu ? H : B * H;         // rows of the (rows, L) token grid
    CUtensorMap mq, mk, mv;
    if (!make_qkv_map(&mq, q, L, rows) || !make_qkv_map(&mk, k, L, rows) || !make_qkv_map(&mv, v, L, rows))
        return GDN_ERR_CUDA;
    const bool opts = oo.bf16 || oo.dskip != nullptr || oo.xnorm != kXNormNone;   // the general output epilogue
    if (g) return opts ? launch_la_t<true, true>(mq, mk, mv, g, out, s0, s_final, cu, nctas, H, L, scale, stream)
                       : launch_la_t<true, false>(mq, mk, mv, g, out, s0, s_final, cu, nctas, H, L, scale, stream);
    return opts ? launch_la_t<false, true>(mq, mk, mv, g, out, s0, s_final, cu, nctas, H, L, scale, stream)
                : launch_la_t<false, false>(mq, mk, mv, g, out, s0, s_final, cu, nctas, H, L, scale, stream);
}

// 64- or 128-wide bf16 row tensor maps (tc_gdn.cu)
bool make_rows_map(CUtensorMap *m, const void *ptr, int L, int BH, int width);

// Head sizes of 64 (dk or dv; the other 64 or 128) with the plain fp32 output: 64-wide tensor
// maps whose second 64-column box loads as zeros, so the kernel computes the zero-padded call
// and stores only dk x dv states and dv output columns.
gdn_status_t launch_tc_la_narrow(const void *q, const void *k, const void *v, const float *g, float *o,
                                 const float *s0, float *s_final, const int *cu, int B, int H, int L, int dk, int dv,
                                 float scale, cudaStream_t stream) {
    const int nctas = B * H;
    const FwdOpts plain{false, nullptr, false, kXNormNone, nullptr, 0.f};
    const OutArgs out = make_out_args(o, v, plain);
    const int rows = cu ? H : B * H;
    CUtensorMap mq, mk, mv;
    if (!make_rows_map(&mq, q, L, rows, dk) || !make_rows_map(&mk, k, L, rows, dk) ||
        !make_rows_map(&mv, v, L, rows, dv))
        return GDN_ERR_CUDA;
    return g ? launch_la_t<true, false, true>(mq, mk, mv, g, out, s0, s_final, cu, nctas, H, L, scale, stream, dk, dv)
             : launch_la_t<false, false, true>(mq, mk, mv, g, out, s0, s_final, cu, nctas, H, L, scale, stream, dk, dv);
}

}  // namespace gdn
