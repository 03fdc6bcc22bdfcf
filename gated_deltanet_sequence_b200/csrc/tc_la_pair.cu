// Pair form of the tensor-core linear-attention prefill for sm_100a (plain or with a
// scalar per-token decay; bf16 inputs, dk = dv = 128, chunk C = 64, fp32 accumulation,
// output and state), for batches with at most half as many (sequence, head) pairs as SMs:
// the one-CTA-per-head form would then leave most SMs idle while each CTA walks its
// chunks at the latency of its own pipeline. Here a cluster of two CTAs serves one
// (sequence, head) and splits the state by key rows: CTA h holds S^T_h = S[64h:64h+64, :]^T
// (TMEM lane = value column v, 64 key columns). Per chunk (page "混合注意力学习(1)",
// section "FWP分块并行机制"; page "LinearAttention 概述", sections "快速预览" and
// "Lightning Attention": O = (Q K^T o M) V, diagonal included), with G the within-chunk
// cumulative sum of g, gamma = exp(G), Gamma_rs = exp(G_r - G_s) (s <= r), d_s =
// exp(G_last - G_s), and s_h = rows 32h .. 32h+31 of the chunk:
//   Gram    [K;Q] K_{s_h}^T                                 M=128, N=32 (Q K^T half used)
//   state   S^T_h <- gamma_last S^T_h + V^T (diag(d) K)[:, 64h:64h+64]        M=128, N=64
//   out     O^T_h = S^T_h Q'_h^T + V_{s_h}^T P_{s_h}^T,  Q' = diag(scale gamma) Q,
//           P = scale (Q K^T o Gamma) (s <= r)                                M=128, N=64
// so O^T = O^T_0 + O^T_1. CTA h stores output rows 32h .. 32h+31: it sends the other
// half of its partial O^T to its peer through distributed shared memory and adds the
// peer's half of the same rows. Each CTA loads the full Q, K, V tiles (the peer's copy of
// a tile is read from L2). The state chain per chunk is half a state: one fp32 -> fp16
// pass over 64 key columns and four N=64 UMMAs.
//
// Warp roles (640 threads) as in the one-CTA form:
//   warp 0      TMA producer (3-stage ring of Q, K, V tiles)
//   warp 1      Gram issuer
//   warp 2      gate warp (gated only): G, gamma, d, exp(-G) per chunk
//   warp 3      chain issuer: state update, then S^T Q'^T and V^T P^T
//   warps 4-7   state group: S^T_h -> fp16 copy, S^T_h <- gamma_last S^T_h
//   warps 8-11  output group: O^T_h halves -> peer / own rows, sum, o
//   warps 12-15 converter: Q box h -> Q', K box h -> diag(d) K, in place
//   warps 16-17 V -> fp16, in place
//   warps 18-19 P writers (Gram rows 64-127: Q K_{s_h}^T)
#include "tc_ctl.cuh"

namespace gdn {

namespace {
using namespace ptx;

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kThreads = 640;
constexpr int kStages = 3;
constexpr int kPair = 2;                  // CTAs per (sequence, head)
constexpr float kFastDecayLimit = -60.f;  // G_last >= this: Gamma = gamma_r * exp(-G_s)

// ---- shared memory map (byte offsets from a 1024-aligned base; the same in both CTAs) --
constexpr uint32_t kStageBytes = 49152;
constexpr uint32_t ST_K0 = 0, ST_Q0 = 8192, ST_K1 = 16384, ST_Q1 = 24576, ST_V0 = 32768, ST_V1 = 40960;
constexpr uint32_t OFF_PG = kStages * kStageBytes;  // 2 x P_{s_h}, K-major 64 rows x 32 s (first 64 B of 128-B rows)
constexpr uint32_t OFF_RX = OFF_PG + 16384;         // 2 x the peer's half of O^T: [v][32 r] fp32 (16 KB each)
constexpr uint32_t kRxBytes = 16384;
constexpr uint32_t OFF_VEC = OFF_RX + 2 * kRxBytes; // 2 x {G, gamma, d, exp(-G), flag}
constexpr uint32_t kVecBytes = 1536;
constexpr int V_G = 0, V_GAM = 64, V_D = 128, V_IG = 192, V_FAST = 256;
constexpr uint32_t OFF_XN = OFF_VEC + 2 * kVecBytes; // output-normalisation scratch (384 fp32)
constexpr uint32_t OFF_BAR = OFF_XN + 1536;
constexpr uint32_t kSmemBytes = OFF_BAR + 512;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;
static_assert(kSmemAlloc <= 232448, "shared memory budget");
static_assert(OFF_PG % 1024 == 0 && OFF_RX % 16 == 0, "alignment");

// ---- tensor memory columns (512 allocated) ----------------------------------------
constexpr uint32_t TM_S = 0;      // S^T_h fp32: lane = value v, 64 key columns of this half
constexpr uint32_t TM_SH = 64;    // 2 x S^T_h fp16 (A operand): 32 columns of key pairs each
constexpr uint32_t TM_G = 128;    // 2 x [K;Q] K_{s_h}^T: lanes 64-127 Q K^T (row r, column s - 32h)
constexpr uint32_t TM_O = 256;    // 2 x O^T_h: lane = value v, 64 columns r

constexpr uint32_t ID_GRAM = idesc_f16(128, 32, false, false, false, /*bf16=*/true);
constexpr uint32_t ID_SQ = idesc_f16(128, 64, false, false);
constexpr uint32_t ID_ST = idesc_f16(128, 64, true, true);
constexpr uint32_t ID_PV = idesc_f16(128, 64, true, false);

enum : int {
    B_FULL = 0,      // [4] TMA -> Gram issuer, converters (3 used)
    B_GREAD = 4,     // [4] Gram has read the bf16 tiles of the stage -> Q/K converter
    B_CONV = 8,      // [4] Q', diag(d) K of box h written -> chain issuer
    B_SFREE = 12,    // [4] last UMMA reading the stage done -> TMA
    B_GATE = 16,     // [2] gate values ready
    B_ODONE = 18,    // [2] O^T_h of the chunk complete -> output group, gate warp, P writers
    B_OFREE = 20,    // [2] output group has read O^T_h -> chain issuer
    B_PREP = 22,     // [2] P written -> chain issuer
    B_GRAM = 24,     // [2] Gram done -> P writers
    B_GFREE = 26,    // [2] P writers have read the Gram -> Gram issuer
    B_VCONV = 28,    // [4] V of the stage converted -> chain issuer (3 used)
    B_SRDY = 32,     // fp16 S and decay done -> chain issuer
    B_SDONE = 33,    // state update done -> state group
    B_RXFULL = 34,   // [2] the peer's half for this CTA's rows is in RX (its asynchronous stores'
                     //     byte count, armed by this CTA one phase ahead)
    B_TXFREE = 36,   // [2] the peer has consumed what this CTA sent it (remote arrival)
    kNumBars = 38
};
constexpr int kBarState = 1, kBarOut = 2, kBarP = 3, kBarConv = 4, kBarV = 5;   // named barriers

template <bool GATED, bool OPTS>
__global__ void __launch_bounds__(kThreads, 1)
tc_la_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ g, const OutArgs out,
                  const float *__restrict__ s0, float *__restrict__ s_final, const int *__restrict__ cu, int H,
                  int Lrow, float scale, long long wait_limit, unsigned *__restrict__ err_word) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kNumBars);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
    const Ctl ctl{bars, abort_flag, err_word, wait_limit};

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t h = cluster_ctarank();               // key half of this CTA
    const uint32_t peer = h ^ 1u;
    const int bh = blockIdx.x / kPair;                  // (sequence, head): state index
    const SeqSpan sp = seq_span(cu, bh, H, Lrow, err_word);
    const int L = sp.len;
    const int zc = sp.head_row, ty0 = sp.t0;
    const int nchunks = (L + kC - 1) / kC;
    const size_t row0 = static_cast<size_t>(zc) * Lrow + ty0;

    if (tid == 0) {
        for (int b = 0; b < kNumBars; ++b) mbar_init(&bars[b], 1);
        abort_flag[0] = 0;
        // the receive buffers of chunks 0 and 1 expect the peer's 16 KB each
        for (int p = 0; p < 2; ++p)
            if (p < (sp.len + kC - 1) / kC) mbar_arrive_expect_tx(&bars[B_RXFULL + p], kRxBytes);
        fence_mbar_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    if (!GATED && tid < 128) {
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
    // both CTAs' barriers are initialised before any remote arrival or store
    cluster_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ================================================================ TMA producer
        if (lane == 0) {
            int last[kStages] = {-1, -1, -1};
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % kStages;
                if (c >= kStages && !ctl.wait_lazy(B_SFREE + s, (c / kStages - 1) & 1)) break;
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
            for (int s = 0; s < kStages; ++s)
                if (last[s] >= 0) ctl.drain(B_FULL + s, (last[s] / kStages) & 1);
        }
    } else if (warp == 1) {
        // ================================================================ Gram issuer
        // [K;Q] K_{s_h}^T: B = the 32 K rows of this CTA's half of the chunk
        if (lane == 0) {
            int last = -1;
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % kStages;
                const uint32_t stg = sb + s * kStageBytes;
                const int p = c & 1;
                if (!ctl.wait_lazy(B_FULL + s, (c / kStages) & 1)) break;
                if (c >= 2 && !ctl.wait_lazy(B_GFREE + p, ((c - 2) >> 1) & 1)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
                    mma_f16(tmem + TM_G + p * 32, sdesc_sw128(stg + ST_K0 + off, 16, 1024),
                            sdesc_sw128(stg + ST_K0 + h * 4096u + off, 16, 1024), ID_GRAM, kk > 0);
                }
                mma_commit(&bars[B_GRAM + p]);
                mma_commit(&bars[B_GREAD + s]);
                last = c;
            }
            if (last >= 0) ctl.drain(B_GREAD + last % kStages, (last / kStages) & 1);
        }
    } else if (warp == 2) {
        // ================================================================ gate warp
        if (GATED) {
            float g_nx[2] = {0.f, 0.f};
#pragma unroll
            for (int e = 0; e < 2; ++e)
                if (2 * lane + e < L) g_nx[e] = g[row0 + 2 * lane + e];
#pragma unroll 1
            for (int c = 0; c < nchunks; ++c) {
                const int p = c & 1;
                float *vec = reinterpret_cast<float *>(smem + OFF_VEC + p * kVecBytes);
                if (c >= 2) {
                    int w = 1;
                    if (lane == 0) w = ctl.wait_lazy(B_ODONE + p, ((c - 2) >> 1) & 1) ? 1 : 0;
                    if (__shfl_sync(0xffffffffu, w, 0) == 0) break;
                }
                const float g0 = g_nx[0], g1 = g_nx[1];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int t = (c + 1) * kC + 2 * lane + e;
                    g_nx[e] = (c + 1 < nchunks && t < L) ? g[row0 + t] : 0.f;
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
                // S^T_h += V^T (diag(d) K)[:, box h]: the serial state chain goes first
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f16(tmem + TM_S, sdesc_sw128(stg + ST_V0 + kk * 2048, 8192, 1024),
                            sdesc_sw128(stg + ST_K0 + h * 16384u + kk * 2048, 16384, 1024), ID_ST, 1u);
                mma_commit(&bars[B_SDONE]);
                last_bar = B_SDONE;
                last_par = c & 1;
                // O^T_h = S^T_h Q'_h^T into the O buffer of parity p, once chunk c-2's was read
                if (c >= 2 && !ctl.wait(B_OFREE + p, ((c - 2) >> 1) & 1)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f16_ts(tmem + TM_O + p * 64, tmem + TM_SH + p * 32 + kk * 8,
                               sdesc_sw128(stg + ST_Q0 + h * 16384u + kk * 32, 16, 1024), ID_SQ, kk > 0);
                if (!ctl.wait(B_PREP + p, (c >> 1) & 1)) {
                    mma_commit(&bars[B_ODONE + p]);
                    last_bar = B_ODONE + p;
                    last_par = (c >> 1) & 1;
                    break;
                }
                tc_fence_after();
                // O^T_h += V_{s_h}^T P_{s_h}^T (32 rows of V)
#pragma unroll
                for (int kk = 0; kk < 2; ++kk)
                    mma_f16(tmem + TM_O + p * 64, sdesc_sw128(stg + ST_V0 + h * 4096u + kk * 2048, 8192, 1024),
                            sdesc_sw128(sb + OFF_PG + p * 8192 + kk * 32, 16, 1024), ID_PV, 1u);
                mma_commit(&bars[B_ODONE + p]);
                mma_commit(&bars[B_SFREE + s]);
                last_bar = B_SFREE + s;
                last_par = (c / kStages) & 1;
            }
            if (last_bar >= 0) ctl.drain(last_bar, last_par);
        }
    } else if (warp < 8) {
        // ================================================================ state group
        const int v = tid - 128;                          // TMEM lane = value column
        const bool lead = (v == 0);
        const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        const float *vbase = nullptr;
        {
            // S^T_h row v = column v of key rows 64h .. 64h+63 of the initial state
            const float *src = s0 ? s0 + static_cast<size_t>(bh) * kD * kD + h * 64u * kD + v : nullptr;
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
                float r[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) r[e] = src ? src[static_cast<size_t>(cc * 16 + e) * kD] : 0.f;
                tmem_st16(trow + TM_S + cc * 16, r);
            }
            tmem_wait_st();
        }
        (void)vbase;
        int done = -1;
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const int p = c & 1;
            const float *vec = reinterpret_cast<const float *>(smem + OFF_VEC + p * kVecBytes);
            if (!ctl.group_wait_all({c >= 1 ? static_cast<int>(B_SDONE) : -1, GATED ? B_GATE + p : -1},
                                    {static_cast<uint32_t>(c - 1) & 1u, static_cast<uint32_t>(c >> 1) & 1u},
                                    kBarState, lead))
                break;
            tc_fence_after();
            const float gl = GATED ? vec[V_GAM + 63] : 1.f;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float sv[32];
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) tmem_ld16(trow + TM_S + hh * 32 + cc * 16, *reinterpret_cast<float (*)[16]>(sv + 16 * cc));
                tmem_wait_ld();
                float hv[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) hv[e] = __uint_as_float(pack_h2(sv[2 * e], sv[2 * e + 1]));
                tmem_st16(trow + TM_SH + p * 32 + hh * 16, hv);
                if (GATED) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) sv[e] *= gl;
                    tmem_st16(trow + TM_S + hh * 32, *reinterpret_cast<float (*)[16]>(sv));
                    tmem_st16(trow + TM_S + hh * 32 + 16, *reinterpret_cast<float (*)[16]>(sv + 16));
                }
            }
            tmem_wait_st();
            tc_fence_before();
            named_bar(kBarState, 128);
            if (lead) mbar_arrive(&bars[B_SRDY]);
            done = c;
        }
        if (s_final && (nchunks == 0 || (done == nchunks - 1 &&
                                         ctl.group_wait(B_SDONE, (nchunks - 1) & 1, kBarState, lead, 128)))) {
            if (nchunks > 0) tc_fence_after();
            // column v of key rows 64h .. 64h+63 of the final state
            float *dst = s_final + static_cast<size_t>(bh) * kD * kD + h * 64u * kD + v;
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
                float sv[16];
                tmem_ld16(trow + TM_S + cc * 16, sv);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) dst[static_cast<size_t>(cc * 16 + e) * kD] = sv[e];
            }
        }
    } else if (warp < 12) {
        // ================================================================ output group
        // O^T_h lane v, columns r: the other CTA's rows (32 (1-h) .. +31) go to the peer's RX,
        // the peer's partial of this CTA's rows (32 h .. +31) arrives in this CTA's RX
        const int v = tid - 256;
        const bool lead = (v == 0);
        const int head = zc % H;
        float *xn = reinterpret_cast<float *>(smem + OFF_XN);
        const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const int p = c & 1;
            if (!ctl.group_wait(B_ODONE + p, (c >> 1) & 1, kBarOut, lead, 128)) break;
            tc_fence_after();
            float mine[32], theirs[32];
            {
                float t0[16], t1[16];
                tmem_ld16(trow + TM_O + p * 64 + peer * 32, t0);
                tmem_ld16(trow + TM_O + p * 64 + peer * 32 + 16, t1);
                tmem_ld16(trow + TM_O + p * 64 + h * 32, *reinterpret_cast<float (*)[16]>(mine));
                tmem_ld16(trow + TM_O + p * 64 + h * 32 + 16, *reinterpret_cast<float (*)[16]>(mine + 16));
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) { theirs[e] = t0[e]; theirs[16 + e] = t1[e]; }
            }
            tc_fence_before();
            // the peer's RX of parity p is free once it consumed what this CTA sent for chunk c-2
            if (!ctl.group_wait_cluster(B_TXFREE + p, ((c - 2) >> 1) & 1, kBarOut, lead && c >= 2, 128)) break;
            if (lead) mbar_arrive(&bars[B_OFREE + p]);
            {
                // asynchronous stores into the peer's RX, counted in bytes on its RXFULL barrier
                const uint32_t rx = mapa_shared(sb + OFF_RX + p * kRxBytes + v * 128u, peer);
                const uint32_t rb = mapa_shared(smem_u32(&bars[B_RXFULL + p]), peer);
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    asm volatile(
                        "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                            rx + e * 4u),
                        "f"(theirs[e]), "f"(theirs[e + 1]), "f"(theirs[e + 2]), "f"(theirs[e + 3]), "r"(rb)
                        : "memory");
            }
            // the peer's partial of this CTA's rows
            if (!ctl.group_wait_cluster(B_RXFULL + p, (c >> 1) & 1, kBarOut, lead, 128)) break;
            {
                const float4 *rx = reinterpret_cast<const float4 *>(smem + OFF_RX + p * kRxBytes + v * 128u);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float4 x = rx[e];
                    mine[4 * e] += x.x; mine[4 * e + 1] += x.y; mine[4 * e + 2] += x.z; mine[4 * e + 3] += x.w;
                }
            }
            named_bar(kBarOut, 128);
            if (lead) {
                // RX of parity p expects the peer's half of chunk c + 2, then goes back to the peer
                if (c + 2 < nchunks) mbar_arrive_expect_tx(&bars[B_RXFULL + p], kRxBytes);
                mbar_arrive_cluster(mapa_shared(smem_u32(&bars[B_TXFREE + p]), peer));
            }
            // rows 32h .. 32h+31 of the chunk (rows >= n are padding)
            const int n = min(kC, L - c * kC) - static_cast<int>(h) * 32;
            const size_t elem0 = (row0 + static_cast<size_t>(c) * kC + h * 32u) * kD + v;
            if constexpr (OPTS) {
                float ov[64];
#pragma unroll
                for (int e = 0; e < 32; ++e) { ov[e] = mine[e]; ov[32 + e] = 0.f; }
                store_out_rows_group(ov, out, elem0, n < 32 ? n : 32, head, v, kBarOut, xn, xn + 256);
            } else {
                float *ocol = static_cast<float *>(out.o) + elem0;
#pragma unroll
                for (int r = 0; r < 32; ++r)
                    if (r < n) ocol[static_cast<size_t>(r) * kD] = mine[r];
            }
        }
    } else if (warp >= 18) {
        // ================================================================ P writers
        // P[r][s] = scale (Q K^T o Gamma)[r][s], s in this CTA's half (s <= r); Gram lane 64 + r
        const int r = tid - 576;                          // 0..63
        const bool pl = (r == 0);
        const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const int p = c & 1;
            const float *vec = reinterpret_cast<const float *>(smem + OFF_VEC + p * kVecBytes);
            if (!ctl.group_wait_all({c >= 2 ? B_ODONE + p : -1, GATED ? B_GATE + p : -1, B_GRAM + p},
                                    {static_cast<uint32_t>((c - 2) >> 1) & 1u, static_cast<uint32_t>(c >> 1) & 1u,
                                     static_cast<uint32_t>(c >> 1) & 1u},
                                    kBarP, pl, 64))
                break;
            tc_fence_after();
            float x[32];
            {
                float t0[16], t1[16];
                tmem_ld16(trow + TM_G + p * 32, t0);
                tmem_ld16(trow + TM_G + p * 32 + 16, t1);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) { x[e] = t0[e]; x[16 + e] = t1[e]; }
            }
            tc_fence_before();
            named_bar(kBarP, 64);
            if (pl) mbar_arrive(&bars[B_GFREE + p]);
            const bool fast = !GATED || reinterpret_cast<const int *>(vec)[V_FAST] != 0;
            const float fr = scale * (GATED ? vec[V_GAM + r] : 1.f);
            const float Gr = GATED ? vec[V_G + r] : 0.f;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int sabs = 32 * static_cast<int>(h) + e;
                if (fast) x[e] = (sabs <= r) ? fr * (GATED ? vec[V_IG + sabs] : 1.f) * x[e] : 0.f;
                else x[e] = (sabs <= r) ? scale * __expf(Gr - vec[V_G + sabs]) * x[e] : 0.f;
            }
            const uint32_t prow = sb + OFF_PG + p * 8192;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch)
                st_shared_v4(prow + sw128(r, ch), pack_h2(x[8 * ch], x[8 * ch + 1]), pack_h2(x[8 * ch + 2], x[8 * ch + 3]),
                             pack_h2(x[8 * ch + 4], x[8 * ch + 5]), pack_h2(x[8 * ch + 6], x[8 * ch + 7]));
            fence_proxy_async();
            named_bar(kBarP, 64);
            if (pl) mbar_arrive(&bars[B_PREP + p]);
        }
    } else if (warp >= 16) {
        // ================================================================ V converter
        const int t = tid - 512;                          // 0..63
        const bool lead = (t == 0);
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kStages;
            if (!ctl.group_wait(B_FULL + s, (c / kStages) & 1, kBarV, lead, 64)) break;
            uint8_t *vt = smem + s * kStageBytes + ST_V0;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint4 x[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) x[i] = *reinterpret_cast<const uint4 *>(vt + ((hh * 8 + i) * 64 + t) * 16);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    uint4 y = x[i];
                    y.x = bf16x2_to_h2(y.x);
                    y.y = bf16x2_to_h2(y.y);
                    y.z = bf16x2_to_h2(y.z);
                    y.w = bf16x2_to_h2(y.w);
                    *reinterpret_cast<uint4 *>(vt + ((hh * 8 + i) * 64 + t) * 16) = y;
                }
            }
            fence_proxy_async();
            named_bar(kBarV, 64);
            if (lead) mbar_arrive(&bars[B_VCONV + s]);
        }
    } else {
        // ================================================================ Q / K converter
        // box h of Q -> fp16(scale gamma_r q), box h of K -> fp16(d_s k), in place, once the
        // Gram has read the bf16 tiles
        const int t = tid - 384;                          // 0..127
        const bool lead = (t == 0);
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kStages, p = c & 1;
            const float *vec = reinterpret_cast<const float *>(smem + OFF_VEC + p * kVecBytes);
            uint8_t *st = smem + s * kStageBytes;
            const int nvalid = min(kC, L - c * kC);
            if (!ctl.group_wait_all({B_FULL + s, GATED ? B_GATE + p : -1, B_GREAD + s},
                                    {static_cast<uint32_t>(c / kStages) & 1u, static_cast<uint32_t>(c >> 1) & 1u,
                                     static_cast<uint32_t>(c / kStages) & 1u},
                                    kBarConv, lead, 128))
                break;
            // box h of Q then of K: 2 x 512 chunks of 16 B, row = chunk / 8
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                uint4 x[4];
                uint32_t off[4];
                float f[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t idx = static_cast<uint32_t>(i * 128 + t);       // 0..511
                    const uint32_t row = idx >> 3;
                    off[i] = (part == 0 ? ST_Q0 : ST_K0) + h * 16384u + idx * 16u;
                    if (part == 0) f[i] = scale * (GATED ? vec[V_GAM + row] : 1.f);
                    else f[i] = static_cast<int>(row) < nvalid ? (GATED ? vec[V_D + row] : 1.f) : 0.f;
                    x[i] = *reinterpret_cast<const uint4 *>(st + off[i]);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint4 y = x[i];
                    y.x = pack_h2(f[i] * __uint_as_float(y.x << 16), f[i] * __uint_as_float(y.x & 0xFFFF0000u));
                    y.y = pack_h2(f[i] * __uint_as_float(y.y << 16), f[i] * __uint_as_float(y.y & 0xFFFF0000u));
                    y.z = pack_h2(f[i] * __uint_as_float(y.z << 16), f[i] * __uint_as_float(y.z & 0xFFFF0000u));
                    y.w = pack_h2(f[i] * __uint_as_float(y.w << 16), f[i] * __uint_as_float(y.w & 0xFFFF0000u));
                    *reinterpret_cast<uint4 *>(st + off[i]) = y;
                }
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
    // no CTA leaves while its peer may still store to its shared memory or arrive on its barriers
    cluster_sync();
}

template <bool GATED, bool OPTS>
gdn_status_t launch_pair_t(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv, const float *g,
                           const OutArgs &out, const float *s0, float *s_final, const int *cu, int nheads, int H,
                           int L, float scale, cudaStream_t stream) {
    auto kern = tc_la_pair_kernel<GATED, OPTS>;
    if (!ensure_smem_limit(reinterpret_cast<const void *>(kern), kSmemAlloc)) return GDN_ERR_CUDA;
    unsigned *err = device_error_word();
    if (!err) return GDN_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(nheads) * kPair);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemAlloc;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kPair;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const long long limit = wait_limit_cycles();
    return cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, g, out, s0, s_final, cu, H, L, scale, limit, err) == cudaSuccess
               ? GDN_OK
               : GDN_ERR_CUDA;
}

}  // namespace

gdn_status_t launch_tc_la_pair(const void *q, const void *k, const void *v, const float *g, void *o,
                               const float *s0, float *s_final, const int *cu, int B, int H, int L, float scale,
                               FwdOpts oo, cudaStream_t stream) {
    const int nheads = B * H;
    const OutArgs out = make_out_args(o, v, oo);
    const int rows = cu ? H : B * H;
    CUtensorMap mq, mk, mv;
    if (!make_qkv_map(&mq, q, L, rows) || !make_qkv_map(&mk, k, L, rows) || !make_qkv_map(&mv, v, L, rows))
        return GDN_ERR_CUDA;
    const bool opts = oo.bf16 || oo.dskip != nullptr || oo.xnorm != kXNormNone;
    if (g) return opts ? launch_pair_t<true, true>(mq, mk, mv, g, out, s0, s_final, cu, nheads, H, L, scale, stream)
                       : launch_pair_t<true, false>(mq, mk, mv, g, out, s0, s_final, cu, nheads, H, L, scale, stream);
    return opts ? launch_pair_t<false, true>(mq, mk, mv, g, out, s0, s_final, cu, nheads, H, L, scale, stream)
                : launch_pair_t<false, false>(mq, mk, mv, g, out, s0, s_final, cu, nheads, H, L, scale, stream);
}

}  // namespace gdn
