// Cluster form of the tensor-core Gated DeltaNet / DeltaNet prefill for sm_100a, for
// batches with few (sequence, head) pairs and long sequences: the one-CTA-per-head kernel
// then leaves most SMs idle while each CTA walks its chunks at the latency of the
// state-independent prep (Gram, A / P masks, UT solve). Here a cluster of three CTAs
// serves one (sequence, head): CTA 0 runs the serial state chain; CTAs 1 and 2 each run
// the prep of every other chunk (chunks 0, 2, 4, ... and 1, 3, 5, ...) and write its
// results (T diag(beta gamma), T diag(beta), P = scale (Q K^T o Gamma) as fp16 operands
// in the 128-byte swizzled layouts, and the chunk's gate values) straight into a
// three-slot ring in CTA 0's shared memory (chunk c in slot c mod 3) through
// distributed shared memory, handing each slot over with a remote mbarrier arrival
// (release / acquire at cluster scope). Once a chunk's last UMMA has completed, CTA 0
// hands its slot to the prep CTA that fills it next (the one of chunk c + 3), so the
// prep runs up to three chunks ahead of the chain.
//
// The arithmetic is the one-CTA kernel's (same operands, same UMMAs, same order of
// operations per chunk), so both forms give the same bits. Per chunk, with G the
// within-chunk cumulative sum of g, gamma = exp(G), Gamma_rs = exp(G_r - G_s) (s <= r),
// d_s = exp(G_last - G_s) (page "混合注意力学习(1)", sections "DeltaNet 分块并行机制",
// "重新定义降低内存占用", "HouseHolder变换和WY表示"; page "LinearAttention 概述", "FLASH"):
//   prep CTA   Gram [K;Q] K^T; A = tril(diag(beta) K K^T o Gamma, -1); T = (I + A)^-1;
//              T1 = T diag(beta gamma), T2 = T diag(beta); P
//   chain CTA  W^T = K^T T1^T, U^T = V^T T2^T; Ut^T = U^T - S^T W^T; O^T = S^T Q'^T + Ut^T P^T;
//              S <- gamma_last S + (diag(d) K)^T Ut
//
// Warp roles. Chain CTA (rank 0): warp 0 TMA (Q, K, V, 2 stages), warp 2 UMMA issuer,
// warps 4-7 state group, warps 8-11 tile converter (K, V -> fp16, Q -> Q'). Prep CTAs:
// warp 0 TMA (K, Q), warp 1 Gram issuer, warp 3 gate warp, warps 8-15 prep group.
#include "tc_gdn_parts.cuh"

namespace gdn {

namespace {
using namespace ptx;
using namespace tcgdn;

constexpr int kCluster = 3;       // chain CTA + two prep CTAs
constexpr int kThreads = 512;
constexpr int kGroupS = 4;        // first warp of the chain CTA's state group
constexpr int kGroupP = 8;        // first warp of the prep CTA's prep group / the converter
constexpr int kNP = 256;          // prep group threads
constexpr int kBarS = 1, kBarP = 2, kBarC = 4;   // named barriers: state, prep (256), converter
constexpr float kFastDecayLimit = -60.f;          // G_last >= this: Gamma = gamma_r * exp(-G_s)

// ---- chain CTA shared memory (byte offsets from a 1024-aligned base) --------------
constexpr uint32_t kStageBytes = 49152;   // one chunk of K, Q, V
constexpr uint32_t ST_K0 = 0, ST_Q0 = 8192, ST_K1 = 16384, ST_Q1 = 24576, ST_V0 = 32768, ST_V1 = 40960;
constexpr uint32_t ST_W = ST_V0;          // W (MN-major) replaces V once U has been formed
constexpr uint32_t C_S = 2 * kStageBytes; // S as MN-major A: 2 x (128 key rows x 64 v)
constexpr uint32_t C_UB = C_S + 32768;    // Ut, K-major: 128 value rows x 64 s
constexpr uint32_t C_SLOT = C_UB + 16384; // kSlots slots filled by the prep CTAs
constexpr int kSlots = 3;
constexpr uint32_t SL_T1 = 0, SL_T2 = 8192, SL_PG = 16384, SL_VEC = 24576;   // within a slot
constexpr uint32_t kSlotBytes = 26624;
constexpr uint32_t kVecBytes = 1536;      // {G, beta, gamma, d, exp(-G), flag}: 64 fp32 each
constexpr int V_G = 0, V_B = 64, V_GAM = 128, V_D = 192, V_IG = 256, V_FAST = 320;
// ---- prep CTA shared memory --------------------------------------------------------
constexpr uint32_t kPStageBytes = 32768;  // one chunk of K, Q ([K;Q] per key half)
constexpr uint32_t P_AT = 2 * kPStageBytes;   // A^T fp32 64 x 64
constexpr uint32_t P_TF = P_AT + 16384;       // T fp32 64 x 68 (pitch 68)
constexpr int kTP = 68;
constexpr uint32_t P_R = P_TF + 64 * kTP * 4; // 4 x 16 x 16 fp32 per-warp block scratch
constexpr uint32_t P_VEC = P_R + 4096;        // 2 x gate values
// ---- both: barriers at the same offset (remote arrivals address them by offset) -----
constexpr uint32_t C_XN = C_SLOT + kSlots * kSlotBytes;   // chain CTA: output-normalisation scratch
constexpr uint32_t OFF_BAR = C_XN + 1536;
constexpr uint32_t kSmemBytes = OFF_BAR + 512;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;  // slack to align the base to 1024 B
static_assert(kSmemAlloc <= 232448, "shared memory budget");
static_assert(C_SLOT % 1024 == 0 && kSlotBytes % 1024 == 0 && C_S % 1024 == 0 && C_UB % 1024 == 0, "alignment");
static_assert(P_VEC + 2 * kVecBytes <= OFF_BAR, "prep CTA map");

// ---- tensor memory ---------------------------------------------------------------------
constexpr uint32_t TM_S = 0;      // chain CTA: state S, lane = key row j, 128 value columns
constexpr uint32_t TM_W = 128;    // W^T: lane = key j, 64 columns r
constexpr uint32_t TM_U = 192;    // U^T then Ut^T: lane = value v, 64 columns r
constexpr uint32_t TM_O = 256;    // 2 x O^T: lane = value v, 64 columns r
constexpr uint32_t TM_G = 0;      // prep CTA: [K;Q] K^T, lanes 0-63 K K^T, 64-127 Q K^T

constexpr uint32_t ID_GRAM = idesc_f16(128, 64, false, false, false, /*bf16=*/true);
constexpr uint32_t ID_WU = idesc_f16(128, 64, true, false);
constexpr uint32_t ID_SW = idesc_f16(128, 64, true, true, /*neg_a=*/true);
constexpr uint32_t ID_SQ = idesc_f16(128, 64, true, false);
constexpr uint32_t ID_ST = idesc_f16(128, 128, true, false);
constexpr uint32_t ID_O = idesc_f16(128, 64, false, false);

// mbarriers (every CTA initialises all of them; each role uses its own). A parity wait
// for phase k is only correct while the producer cannot complete phase k+1 first.
enum : int {
    // chain CTA
    B_FULL = 0,      // [2] TMA -> converter
    B_CDONE = 2,     // [2] chunk's UMMAs done (frees the stage, returns the slot)
    B_SLOT = 4,      // [3] slot filled by a prep CTA (remote arrival) -> converter, issuer, state
    B_CONV = 7,      // [2] K, V fp16 and Q' written -> issuer
    B_WU = 9,        // W/U done -> state group (W epilogue)
    B_XFREE = 10,    // state group has read W^T -> issuer (next W/U)
    B_WRDY = 11,     // W operand written -> issuer
    B_SRDY = 12,     // fp16 S written, S scaled -> issuer
    B_ADONE = 13,    // U - W S and S Q' done -> state group (Ut epilogue)
    B_URDY = 14,     // Ut operand written -> issuer
    // prep CTA
    B_PFULL = 15,    // [2] TMA (K, Q) -> Gram issuer
    B_GREAD = 17,    // [2] Gram has read the stage -> TMA
    B_GRAM = 19,     // Gram done -> prep group
    B_GFREE = 20,    // prep group has read the Gram -> Gram issuer
    B_PGATE = 21,    // [2] gate values ready -> prep group
    B_PDONE = 23,    // [2] prep group done with a chunk (gate values free) -> gate warp
    B_SFREE = 25,    // [2] the chain CTA has finished with the slot this CTA fills next (remote
                     //     arrival); this CTA's k-th slot reuse waits on [k & 1]
    // chain CTA (continued)
    B_SDONE = 27,    // state-update UMMAs done -> state group (next fp16 S)
    B_KRDY = 28,     // [2] K <- diag(d) K done (converter, after W/U read K) -> issuer
    kNumBars = 30
};

template <bool GATED, bool OPTS>
__global__ void __launch_bounds__(kThreads, 1)
tc_gdn_cl_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ beta,
                 const float *__restrict__ g, const OutArgs out, const float *__restrict__ s0,
                 float *__restrict__ s_final, const int *__restrict__ cu, int H, int Lrow, float scale,
                 long long wait_limit, unsigned *__restrict__ err_word) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base derived by pointer arithmetic on the shared array (the same
    // offset in every CTA of the cluster, so remote addresses match local ones)
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kNumBars);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
    const Ctl ctl{bars, abort_flag, err_word, wait_limit};

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();
    const int bh = blockIdx.x / kCluster;               // (sequence, head): state index
    const SeqSpan sp = seq_span(cu, bh, H, Lrow, err_word);
    const int L = sp.len;                               // tokens of this sequence
    const int zc = sp.head_row, ty0 = sp.t0;            // TMA head and first-token coordinates
    const int nchunks = (L + kC - 1) / kC;
    const size_t row0 = static_cast<size_t>(zc) * Lrow + ty0;   // first token row in the grid
    const uint32_t ncols = rank == 0 ? 512u : 64u;      // TMEM columns of this CTA

    if (tid == 0) {
        for (int b = 0; b < kNumBars; ++b) mbar_init(&bars[b], 1);
        abort_flag[0] = 0;
        fence_mbar_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, ncols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // every CTA's barriers are initialised before any remote arrival or store
    cluster_sync();
    const uint32_t tmem = *tmem_slot;

    if (rank == 0) {
        // ==================================================================== chain CTA
        if (warp == 0) {
            // ------------------------------------------------------------ TMA producer
            if (lane == 0) {
                int last[2] = {-1, -1};
                for (int c = 0; c < nchunks; ++c) {
                    const int s = c & 1;
                    if (c >= 2 && !ctl.wait_lazy(B_CDONE + s, ((c - 2) >> 1) & 1)) break;
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
                for (int s = 0; s < 2; ++s)
                    if (last[s] >= 0) ctl.drain(B_FULL + s, (last[s] >> 1) & 1);
            }
        } else if (warp == 2) {
            // ================================================================ chain UMMA issuer
            // per chunk: U - W S and S Q' ; state update and P Ut ; then W/U of the next chunk
            if (lane == 0) {
                // the slot of chunk c (written by a prep CTA, cluster acquire) and its converted tiles
                auto ready = [&](int c) -> bool {
                    return ctl.wait_cluster(B_SLOT + c % kSlots, (c / kSlots) & 1) &&
                           ctl.wait(B_CONV + (c & 1), (c >> 1) & 1);
                };
                auto wu = [&](int c) {
                    const uint32_t stg = sb + (c & 1) * kStageBytes;
                    const uint32_t slot = sb + C_SLOT + (c % kSlots) * kSlotBytes;
                    fence_proxy_async();
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16(tmem + TM_W, sdesc_sw128(stg + ST_K0 + kk * 2048, 16384, 1024),
                                sdesc_sw128(slot + SL_T1 + kk * 32, 16, 1024), ID_WU, kk > 0);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16(tmem + TM_U, sdesc_sw128(stg + ST_V0 + kk * 2048, 8192, 1024),
                                sdesc_sw128(slot + SL_T2 + kk * 32, 16, 1024), ID_WU, kk > 0);
                    mma_commit(&bars[B_WU]);
                };
                int last_bar = -1, last_par = 0;   // last commit, for the final drain
                if (nchunks > 0 && ready(0)) {
                    wu(0);
                    last_bar = B_WU;
                    last_par = 0;
                }
                for (int c = 0; last_bar >= 0 && c < nchunks; ++c) {
                    const int s = c & 1;
                    const uint32_t stg = sb + s * kStageBytes;
                    if (!ctl.wait(B_SRDY, c & 1)) break;
                    tc_fence_after();
                    // O^T = S^T Q'^T (needs only the fp16 state and Q')
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
                        mma_f16(tmem + TM_O + s * 64, sdesc_sw128(sb + C_S + kk * 2048, 16384, 1024),
                                sdesc_sw128(stg + ST_Q0 + off, 16, 1024), ID_SQ, kk > 0);
                    }
                    if (!ctl.wait(B_WRDY, c & 1)) {
                        // cover the UMMAs just issued by a commit, so the final drain waits for them
                        mma_commit(&bars[B_ADONE]);
                        last_bar = B_ADONE;
                        last_par = c & 1;
                        break;
                    }
                    tc_fence_after();
                    // Ut^T = U^T - S^T W^T
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_f16(tmem + TM_U, sdesc_sw128(sb + C_S + kk * 2048, 16384, 1024),
                                sdesc_sw128(stg + ST_W + kk * 2048, 8192, 1024), ID_SW, 1u);
                    mma_commit(&bars[B_ADONE]);
                    last_bar = B_ADONE;
                    last_par = c & 1;
                    if (!ctl.wait(B_URDY, c & 1)) break;
                    if (!ctl.wait(B_KRDY + s, (c >> 1) & 1)) break;
                    tc_fence_after();
                    // S += (diag(d) K)^T Ut ;  O^T += Ut^T PG^T
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16(tmem + TM_S, sdesc_sw128(stg + ST_K0 + kk * 2048, 16384, 1024),
                                sdesc_sw128(sb + C_UB + kk * 32, 16, 1024), ID_ST, 1u);
                    mma_commit(&bars[B_SDONE]);
                    last_bar = B_SDONE;
                    last_par = c & 1;
                    // W/U of the next chunk ahead of this chunk's output product, so it runs
                    // while the next fp16 state is formed (Ut^T was read by the Ut epilogue,
                    // W^T by the W epilogue)
                    if (c + 1 < nchunks) {
                        if (!ready(c + 1)) break;
                        if (!ctl.wait(B_XFREE, c & 1)) break;
                        wu(c + 1);
                        last_bar = B_WU;
                        last_par = (c + 1) & 1;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16(tmem + TM_O + s * 64, sdesc_sw128(sb + C_UB + kk * 32, 16, 1024),
                                sdesc_sw128(sb + C_SLOT + (c % kSlots) * kSlotBytes + SL_PG + kk * 32, 16, 1024), ID_O, 1u);
                    mma_commit(&bars[B_CDONE + s]);
                    last_bar = B_CDONE + s;
                    last_par = (c >> 1) & 1;
                }
                // UMMAs complete in issue order: the last commit covers everything issued
                if (last_bar >= 0) ctl.drain(last_bar, last_par);
            }
        } else if (warp >= kGroupS && warp < kGroupS + 4) {
            // ================================================================ state group
            const int j = tid - kGroupS * 32;                // = TMEM lane (key row j / value column v)
            const bool lead = (j == 0);
            const int head = zc % H;                     // head of this row (dense and packed grids)
            float *xn = reinterpret_cast<float *>(smem + C_XN);
            const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
            {
                const float *src = s0 ? s0 + (static_cast<size_t>(bh) * kD + j) * kD : nullptr;
#pragma unroll 1
                for (int cc = 0; cc < 8; ++cc) {
                    float r[16];
#pragma unroll
                    for (int e = 0; e < 16; e += 4) {
                        const float4 x = src ? *reinterpret_cast<const float4 *>(src + cc * 16 + e)
                                             : make_float4(0.f, 0.f, 0.f, 0.f);
                        r[e] = x.x; r[e + 1] = x.y; r[e + 2] = x.z; r[e + 3] = x.w;
                    }
                    tmem_st16(trow + TM_S + cc * 16, r);
                }
                tmem_wait_st();
            }
            int done = 0;   // chunks whose output tile has been stored
            float nf = 0.f;  // non-finite probe over sampled output tiles and the final state
#pragma unroll 1
            for (int c = 0; c < nchunks; ++c) {
                const int s = c & 1;
                const float *vec = reinterpret_cast<const float *>(smem + C_SLOT + (c % kSlots) * kSlotBytes + SL_VEC);
                // S(c) complete (state-update UMMAs of chunk c-1), and this chunk's gate values
                if (!ctl.group_wait_all({c >= 1 ? static_cast<int>(B_SDONE) : -1, B_SLOT + c % kSlots},
                                        {static_cast<uint32_t>(c - 1) & 1u, static_cast<uint32_t>(c / kSlots) & 1u},
                                        kBarS, lead, 128, 2u))
                    break;
                tc_fence_after();
                // ---- S row j -> fp16 MN-major operand; S <- gamma_last S (ahead of the update)
                {
                    const float gl = GATED ? vec[V_GAM + 63] : 1.f;
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        float sv[32];
                        ld_cols<32>(trow + TM_S + h * 32, sv);
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc)
                            st_row16_h(sb + C_S + (h >> 1) * 16384u, j, (h & 1) * 4 + cc * 2, sv + 16 * cc);
                        if (GATED) {
#pragma unroll
                            for (int e = 0; e < 32; ++e) sv[e] *= gl;
#pragma unroll
                            for (int cc = 0; cc < 2; ++cc)
                                tmem_st16(trow + TM_S + h * 32 + cc * 16, *reinterpret_cast<float (*)[16]>(sv + 16 * cc));
                        }
                    }
                    if (GATED) tmem_wait_st();
                }
                fence_proxy_async();
                tc_fence_before();
                named_bar(kBarS, 128);
                if (lead) mbar_arrive(&bars[B_SRDY]);
                // ---- W operand of this chunk (its V slot is consumed); the converter scales K
                if (!ctl.group_wait(B_WU, c & 1, kBarS, lead)) break;
                tc_fence_after();
                {
                    float w[64];
                    ld_cols<64>(trow + TM_W, w);
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) st_row16_h(sb + s * kStageBytes + ST_W, j, 2 * cc, w + 16 * cc);
                }
                fence_proxy_async();
                tc_fence_before();
                named_bar(kBarS, 128);
                if (lead) {
                    mbar_arrive(&bars[B_WRDY]);
                    mbar_arrive(&bars[B_XFREE]);
                }
                // ---- output of the previous chunk (its O tile is complete); its slot goes to the
                //      prep CTA of chunk c+2, the next chunk in that slot (that CTA's
                //      ((c - 1) >> 1)-th slot reuse)
                if (c >= 1) {
                    const int cp = c - 1;
                    if (!ctl.group_wait(B_CDONE + (cp & 1), (cp >> 1) & 1, kBarS, lead)) break;
                    if (c + 2 < nchunks && lead)
                        mbar_arrive_cluster(mapa_shared(smem_u32(&bars[B_SFREE + (((c - 1) >> 1) & 1)]), 1 + (c & 1)));
                    tc_fence_after();
                    store_out_col<OPTS>(trow + TM_O + (cp & 1) * 64, out, (row0 + static_cast<size_t>(cp) * kC) * kD + j, kC, head, j, kBarS, xn,
                                    false, nf);   // the last tile is stored (and probed) after the loop
                    done = c;
                }
                // ---- Ut^T row v -> Ut operand (K-major, rows v)
                if (!ctl.group_wait(B_ADONE, c & 1, kBarS, lead)) break;
                tc_fence_after();
                {
                    float u[64];
                    ld_cols<64>(trow + TM_U, u);
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) st_row16_h(sb + C_UB, j, 2 * cc, u + 16 * cc);
                }
                fence_proxy_async();
                tc_fence_before();
                named_bar(kBarS, 128);
                if (lead) mbar_arrive(&bars[B_URDY]);
            }
            // ---- last output tile and the final state
            if (nchunks > 0 && done == nchunks - 1) {
                const int cp = nchunks - 1;
                if (ctl.group_wait(B_CDONE + (cp & 1), (cp >> 1) & 1, kBarS, lead)) {
                    tc_fence_after();
                    store_out_col<OPTS>(trow + TM_O + (cp & 1) * 64, out, (row0 + static_cast<size_t>(cp) * kC) * kD + j,
                                  L - cp * kC, head, j, kBarS, xn, true, nf);
                    done = nchunks;
                }
            }
            if (s_final && done == nchunks) {
                float *dst = s_final + (static_cast<size_t>(bh) * kD + j) * kD;
#pragma unroll 1
                for (int cc = 0; cc < 8; ++cc) {
                    float sv[16];
                    tmem_ld16(trow + TM_S + cc * 16, sv);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; e += 4) {
                        probe_finite(nf, sv[e] + sv[e + 1] + sv[e + 2] + sv[e + 3]);
                        *reinterpret_cast<float4 *>(dst + cc * 16 + e) = make_float4(sv[e], sv[e + 1], sv[e + 2], sv[e + 3]);
                    }
                }
            }
            report_nonfinite(ctl.aborted() ? 0.f : nf, err_word);
        } else if (warp >= kGroupP && warp < kGroupP + 4) {
            // ------------------------------------------------------------ tile converter
            // K, V bf16 -> fp16 and Q -> Q' = fp16(scale gamma q), in place, once the tiles
            // have landed and the chunk's gate values are in its slot
            const int t4 = tid - kGroupP * 32;               // 0..127
            const bool lead = (t4 == 0);
#pragma unroll 1
            for (int c = 0; c < nchunks; ++c) {
                const int s = c & 1;
                uint8_t *st = smem + s * kStageBytes;
                const float *vec = reinterpret_cast<const float *>(smem + C_SLOT + (c % kSlots) * kSlotBytes + SL_VEC);
                if (!ctl.group_wait_all({B_FULL + s, B_SLOT + c % kSlots},
                                        {static_cast<uint32_t>(c >> 1) & 1u, static_cast<uint32_t>(c / kSlots) & 1u},
                                        kBarC, lead, 128, 2u))
                    break;
                // K and V: 2048 chunks of 16 B at [0,8K) [16K,24K) [32K,48K)
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    uint4 x[8];
                    uint32_t offs[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const uint32_t idx = static_cast<uint32_t>((part * 8 + i) * 128 + t4);   // 0..2047
                        const uint32_t reg = idx >> 9;                                            // 0..3
                        offs[i] = (reg < 2 ? reg * 16384u : 32768u + (reg - 2) * 8192u) + (idx & 511u) * 16u;
                        x[i] = *reinterpret_cast<const uint4 *>(st + offs[i]);
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        x[i].x = pack_h2(bf_lo(x[i].x), bf_hi(x[i].x));
                        x[i].y = pack_h2(bf_lo(x[i].y), bf_hi(x[i].y));
                        x[i].z = pack_h2(bf_lo(x[i].z), bf_hi(x[i].z));
                        x[i].w = pack_h2(bf_lo(x[i].w), bf_hi(x[i].w));
                        *reinterpret_cast<uint4 *>(st + offs[i]) = x[i];
                    }
                }
                // Q: 1024 chunks at [8K,16K) [24K,32K), row r = (offset within the box) / 128
                {
                    uint4 x[8];
                    uint32_t offs[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const uint32_t idx = static_cast<uint32_t>(i * 128 + t4);                 // 0..1023
                        offs[i] = ST_Q0 + (idx >> 9) * 16384u + (idx & 511u) * 16u;
                        x[i] = *reinterpret_cast<const uint4 *>(st + offs[i]);
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float f = scale * vec[V_GAM + ((offs[i] & 8191u) >> 7)];
                        x[i].x = pack_h2(f * bf_lo(x[i].x), f * bf_hi(x[i].x));
                        x[i].y = pack_h2(f * bf_lo(x[i].y), f * bf_hi(x[i].y));
                        x[i].z = pack_h2(f * bf_lo(x[i].z), f * bf_hi(x[i].z));
                        x[i].w = pack_h2(f * bf_lo(x[i].w), f * bf_hi(x[i].w));
                        *reinterpret_cast<uint4 *>(st + offs[i]) = x[i];
                    }
                }
                fence_proxy_async();
                named_bar(kBarC, 128);
                if (lead) mbar_arrive(&bars[B_CONV + s]);
                // K <- diag(d) K for the state update, once W/U (its last reader) is done
                if (GATED) {
                    if (!ctl.group_wait(B_WU, c & 1, kBarC, lead)) break;
                    uint4 x[8];
                    __half2 f[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const uint32_t idx = static_cast<uint32_t>(i * 128 + t4);               // 0..1023
                        f[i] = __float2half2_rn(vec[V_D + ((idx & 511u) >> 3)]);
                        x[i] = *reinterpret_cast<const uint4 *>(st + ST_K0 + (idx >> 9) * 16384u + (idx & 511u) * 16u);
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const uint32_t idx = static_cast<uint32_t>(i * 128 + t4);
                        __half2 *hp = reinterpret_cast<__half2 *>(&x[i]);
#pragma unroll
                        for (int e = 0; e < 4; ++e) hp[e] = __hmul2(hp[e], f[i]);
                        *reinterpret_cast<uint4 *>(st + ST_K0 + (idx >> 9) * 16384u + (idx & 511u) * 16u) = x[i];
                    }
                    fence_proxy_async();
                    named_bar(kBarC, 128);
                }
                if (lead) mbar_arrive(&bars[B_KRDY + s]);
            }
        }
    } else {
        // ==================================================================== prep CTA
        const int pc = static_cast<int>(rank) - 1;         // this CTA's chunks: pc, pc + 2, ...
        const int nmine = nchunks > pc ? (nchunks - pc + 1) / 2 : 0;
        // its first chunk that reuses a slot (c >= kSlots): waits on B_SFREE count from there
        const int i_reuse = (kSlots - pc + 1) / 2;
        if (warp == 0) {
            // ------------------------------------------------------------ TMA producer (K, Q)
            if (lane == 0) {
                int last[2] = {-1, -1};
                for (int i = 0; i < nmine; ++i) {
                    const int s = i & 1, c = pc + 2 * i;
                    if (i >= 2 && !ctl.wait_lazy(B_GREAD + s, ((i - 2) >> 1) & 1)) break;
                    uint8_t *st = smem + s * kPStageBytes;
                    uint64_t *fb = &bars[B_PFULL + s];
                    mbar_arrive_expect_tx(fb, kPStageBytes);
                    tma_load_3d(st + ST_K0, &tm_k, fb, 0, ty0 + c * kC, zc);
                    tma_load_3d(st + ST_Q0, &tm_q, fb, 0, ty0 + c * kC, zc);
                    tma_load_3d(st + ST_K1, &tm_k, fb, 64, ty0 + c * kC, zc);
                    tma_load_3d(st + ST_Q1, &tm_q, fb, 64, ty0 + c * kC, zc);
                    last[s] = i;
                }
                for (int s = 0; s < 2; ++s)
                    if (last[s] >= 0) ctl.drain(B_PFULL + s, (last[s] >> 1) & 1);
            }
        } else if (warp == 1) {
            // ------------------------------------------------------------ Gram issuer
            if (lane == 0) {
                int last = -1;
                for (int i = 0; i < nmine; ++i) {
                    const int s = i & 1;
                    const uint32_t stg = sb + s * kPStageBytes;
                    if (!ctl.wait_lazy(B_PFULL + s, (i >> 1) & 1)) break;
                    if (i >= 1 && !ctl.wait_lazy(B_GFREE, (i - 1) & 1)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
                        mma_f16(tmem + TM_G, sdesc_sw128(stg + ST_K0 + off, 16, 1024),
                                sdesc_sw128(stg + ST_K0 + off, 16, 1024), ID_GRAM, kk > 0);
                    }
                    mma_commit(&bars[B_GRAM]);
                    mma_commit(&bars[B_GREAD + s]);
                    last = i;
                }
                if (last >= 0) ctl.drain(B_GREAD + (last & 1), (last >> 1) & 1);
            }
        } else if (warp == 3) {
            // ------------------------------------------------------------ gate warp
            // lane l owns rows 2l, 2l+1 of each chunk; the next chunk's values are fetched
            // one chunk ahead
            float g_nx[2] = {0.f, 0.f}, b_nx[2] = {0.f, 0.f};
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int t = pc * kC + 2 * lane + e;
                if (nmine > 0 && t < L) {
                    if (GATED) g_nx[e] = g[row0 + t];
                    b_nx[e] = beta[row0 + t];
                }
            }
#pragma unroll 1
            for (int i = 0; i < nmine; ++i) {
                const int s = i & 1, c = pc + 2 * i;
                float *vec = reinterpret_cast<float *>(smem + P_VEC + s * kVecBytes);
                // gate values of parity s are free once the prep group finished local chunk i-2
                if (i >= 2) {
                    int w = 1;
                    if (lane == 0) w = ctl.wait_lazy(B_PDONE + s, ((i - 2) >> 1) & 1) ? 1 : 0;
                    if (__shfl_sync(0xffffffffu, w, 0) == 0) break;
                }
                const float g0 = g_nx[0], g1 = g_nx[1], b0 = b_nx[0], b1 = b_nx[1];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int t = (c + 2) * kC + 2 * lane + e;
                    g_nx[e] = (GATED && i + 1 < nmine && t < L) ? g[row0 + t] : 0.f;
                    b_nx[e] = (i + 1 < nmine && t < L) ? beta[row0 + t] : 0.f;
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
                if (lane == 0) mbar_arrive(&bars[B_PGATE + s]);
            }
        } else if (warp >= kGroupP) {
            // ------------------------------------------------------------ prep group
            const int p = tid - kGroupP * 32;                // 0..255
            const int w8 = warp - kGroupP;                   // 0..7
            const int sub = warp & 3;                        // TMEM lane quarter of this warp
            const int hh = w8 >> 2;                          // which 32 of the 64 Gram columns
            const uint32_t trow = tmem + (static_cast<uint32_t>(sub * 32) << 16);
            // the upper blocks of T1/T2 of every slot stay zero (CTA 1 clears slots 0 and 2, the
            // first used by its chunks 0 and 2; CTA 2 clears slot 1)
            for (int sl = pc; sl < kSlots; sl += 2) {
                const uint32_t zs = mapa_shared(sb + C_SLOT + sl * kSlotBytes, 0);
                for (int i = p; i < 16384 / 16; i += kNP) st_cluster_v4(zs + SL_T1 + i * 16, 0u, 0u, 0u, 0u);
            }
            // order these stores before the T-factor stores of other threads of the group
            asm volatile("fence.acq_rel.cluster;" ::: "memory");
            float *At = reinterpret_cast<float *>(smem + P_AT);   // At[s * 64 + r] = A[r][s]
            float *Tf = reinterpret_cast<float *>(smem + P_TF);   // Tf[r * kTP + c] = T[r][c]
#pragma unroll 1
            for (int i = 0; i < nmine; ++i) {
                const int s = i & 1, c = pc + 2 * i;
                const float *vec = reinterpret_cast<const float *>(smem + P_VEC + s * kVecBytes);
                const uint32_t rslot = mapa_shared(sb + C_SLOT + (c % kSlots) * kSlotBytes, 0);   // in CTA 0
                // gate values, the Gram, and the slot (free once the chain CTA finished the
                // chunk it held, kSlots chunks earlier)
                if (!ctl.group_wait_all({B_PGATE + s, static_cast<int>(B_GRAM),
                                         i >= i_reuse ? B_SFREE + ((i - i_reuse) & 1) : -1},
                                        {static_cast<uint32_t>(i >> 1) & 1u, static_cast<uint32_t>(i) & 1u,
                                         static_cast<uint32_t>((i - i_reuse) >> 1) & 1u},
                                        kBarP, p == 0, kNP, 4u))
                    break;
                // gate values -> slot (96 chunks of 16 B)
                if (p < 96) {
                    const uint4 x = *reinterpret_cast<const uint4 *>(smem + P_VEC + s * kVecBytes + p * 16);
                    st_cluster_v4(rslot + SL_VEC + p * 16, x.x, x.y, x.z, x.w);
                }
                tc_fence_after();
                const bool fast = !GATED || reinterpret_cast<const int *>(vec)[V_FAST] != 0;
                // ---- Gram rows (lane quarter `sub`, columns 32 hh .. 32 hh + 31):
                //      rows 0-63 -> A^T (fp32, UT-solve input), rows 64-127 -> scale Gamma o Q K^T
                {
                    float v[32];
                    ld_cols<32>(trow + TM_G + 32 * hh, v);
                    tc_fence_before();
                    named_bar(kBarP, kNP);                       // every Gram row has been read
                    if (p == 0) mbar_arrive(&bars[B_GFREE]);
                    const int R = sub * 32 + lane;
                    float ig[32];
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4) {
                        const float4 t = *reinterpret_cast<const float4 *>(vec + V_IG + 32 * hh + 4 * q4);
                        ig[4 * q4] = t.x; ig[4 * q4 + 1] = t.y; ig[4 * q4 + 2] = t.z; ig[4 * q4 + 3] = t.w;
                    }
                    if (!fast) {
                        // strong decay: exp(G_r - G_s) per element (ig holds G_s here)
#pragma unroll
                        for (int q4 = 0; q4 < 8; ++q4) {
                            const float4 t = *reinterpret_cast<const float4 *>(vec + V_G + 32 * hh + 4 * q4);
                            ig[4 * q4] = t.x; ig[4 * q4 + 1] = t.y; ig[4 * q4 + 2] = t.z; ig[4 * q4 + 3] = t.w;
                        }
                    }
                    if (R < 64) {
                        const int r = R;
                        float av[32];
                        if (fast) {
                            const float lead = vec[V_B + r] * vec[V_GAM + r];
#pragma unroll
                            for (int e = 0; e < 32; ++e) av[e] = (32 * hh + e < r) ? lead * ig[e] * v[e] : 0.f;
                        } else {
                            const float br = vec[V_B + r], Gr = vec[V_G + r];
#pragma unroll
                            for (int e = 0; e < 32; ++e) av[e] = (32 * hh + e < r) ? br * __expf(Gr - ig[e]) * v[e] : 0.f;
                        }
#pragma unroll
                        for (int e = 0; e < 32; ++e) At[(32 * hh + e) * 64 + r] = av[e];
                    } else {
                        const int r = R - 64;
                        float pv[32];
                        if (fast) {
                            const float lead = scale * vec[V_GAM + r];
#pragma unroll
                            for (int e = 0; e < 32; ++e) pv[e] = (32 * hh + e <= r) ? lead * ig[e] * v[e] : 0.f;
                        } else {
                            const float Gr = vec[V_G + r];
#pragma unroll
                            for (int e = 0; e < 32; ++e) pv[e] = (32 * hh + e <= r) ? scale * __expf(Gr - ig[e]) * v[e] : 0.f;
                        }
#pragma unroll
                        for (int ch = 0; ch < 4; ++ch)
                            st_cluster_v4(rslot + SL_PG + sw128(r, 4 * hh + ch), pack_h2(pv[8 * ch], pv[8 * ch + 1]),
                                         pack_h2(pv[8 * ch + 2], pv[8 * ch + 3]), pack_h2(pv[8 * ch + 4], pv[8 * ch + 5]),
                                         pack_h2(pv[8 * ch + 6], pv[8 * ch + 7]));
                    }
                }
                named_bar(kBarP, kNP);                           // A^T complete
                if (w8 < 4) {
                    // ---- UT solve on warps 8-11. Blocks of T are kept in fp32 (Tf) for the
                    //      products that follow and copied, once final, into the fp16 factors
                    //      T1 = T diag(beta gamma), T2 = T diag(beta) (K-major rows r).
                    //      The upper blocks of T1/T2 are zero from the start.
                    const uint32_t sb = smem_u32(smem);
                    // one 16 x 16 block (bi, bj) of Tf -> T1/T2; lane: row lane / 2, 8 columns
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
                        st_cluster_v4(rslot + SL_T2 + off, pack_h2(u[0], u[1]), pack_h2(u[2], u[3]), pack_h2(u[4], u[5]),
                                     pack_h2(u[6], u[7]));
                        st_cluster_v4(rslot + SL_T1 + off, pack_h2(u[0] * gg[0], u[1] * gg[1]),
                                     pack_h2(u[2] * gg[2], u[3] * gg[3]), pack_h2(u[4] * gg[4], u[5] * gg[5]),
                                     pack_h2(u[6] * gg[6], u[7] * gg[7]));
                    };
                    // diagonal blocks of 16: D_i = (I + A_ii)^-1 by right-looking substitution
                    // (warp i, lane = column; lanes 16-31 mirror 0-15)
                    const int bi = w8, cl = lane & 15;
                    {
                        float acc[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) acc[i] = (i == cl) ? 1.f : 0.f;
#pragma unroll
                        for (int s2 = 0; s2 < 15; ++s2) {
                            const float xs = acc[s2];
                            const float *arow = At + (16 * bi + s2) * 64 + 16 * bi;
#pragma unroll
                            for (int k4 = 0; k4 < 4; ++k4) {
                                if (4 * k4 + 3 <= s2) continue;          // rows of this group are not below s2
                                const float4 a4 = *reinterpret_cast<const float4 *>(arow + 4 * k4);
                                acc[4 * k4 + 0] = fmaf(-a4.x, xs, acc[4 * k4 + 0]);
                                acc[4 * k4 + 1] = fmaf(-a4.y, xs, acc[4 * k4 + 1]);
                                acc[4 * k4 + 2] = fmaf(-a4.z, xs, acc[4 * k4 + 2]);
                                acc[4 * k4 + 3] = fmaf(-a4.w, xs, acc[4 * k4 + 3]);
                            }
                        }
                        if (lane < 16) {
#pragma unroll
                            for (int i = 0; i < 16; ++i) Tf[(16 * bi + i) * kTP + 16 * bi + cl] = acc[i];
                        }
                    }
                    // T1/T2 of chunk c-1 must have been read by its W/U before they are overwritten
                    asm volatile("bar.sync 3, 128;" ::: "memory");
                    {
                        emit(bi, bi);
                        float *Rw = reinterpret_cast<float *>(smem + P_R);
                        // level 1 (warps 0, 1): T_10 = -D_1 (A_10 D_0), T_32 = -D_3 (A_32 D_2)
                        if (bi < 2) {
                            const int i = 2 * bi + 1, j = 2 * bi;
                            float *R = Rw + bi * 256;
                            float acc2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                            block_mm<2>(acc2, [&](int r, int k) { return At[(16 * j + k) * 64 + 16 * i + r]; },
                                        [&](int k, int n) { return Tf[(16 * j + k) * kTP + 16 * j + n]; }, lane);
                            block_store(acc2, [&](int r, int n, float x) { R[r * 16 + n] = x; }, lane, 1.f);
                            __syncwarp();
                            float acc3[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                            block_mm<2>(acc3, [&](int r, int k) { return Tf[(16 * i + r) * kTP + 16 * i + k]; },
                                        [&](int k, int n) { return R[k * 16 + n]; }, lane);
                            block_store(acc3, [&](int r, int n, float x) { Tf[(16 * i + r) * kTP + 16 * j + n] = x; },
                                        lane, -1.f);
                            emit(i, j);
                        }
                        asm volatile("bar.sync 3, 128;" ::: "memory");
                        // level 2 (warp w -> block (i, j) = (2 + w / 2, w % 2)): X_ij = A_{i,0..1} T_{0..1,j}
                        const int ii = 2 + (bi >> 1), jj = bi & 1;
                        {
                            float acc2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                            if (jj == 0)
                                block_mm<4>(acc2, [&](int r, int k) { return At[k * 64 + 16 * ii + r]; },
                                            [&](int k, int n) { return Tf[k * kTP + n]; }, lane);
                            else
                                block_mm<2>(acc2, [&](int r, int k) { return At[(16 + k) * 64 + 16 * ii + r]; },
                                            [&](int k, int n) { return Tf[(16 + k) * kTP + 16 + n]; }, lane);
                            float *R = Rw + bi * 256;
                            block_store(acc2, [&](int r, int n, float x) { R[r * 16 + n] = x; }, lane, 1.f);
                        }
                        asm volatile("bar.sync 3, 128;" ::: "memory");
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
                }
                // hand the slot to the chain CTA
                fence_proxy_async_cluster();
                named_bar(kBarP, kNP);
                if (p == 0) {
                    mbar_arrive_cluster(mapa_shared(smem_u32(&bars[B_SLOT + c % kSlots]), 0));
                    mbar_arrive(&bars[B_PDONE + s]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, ncols);
    }
    // no CTA leaves while another one may still store to its shared memory or arrive on
    // its barriers
    cluster_sync();
}

template <bool GATED, bool OPTS>
gdn_status_t launch_cl_t(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv, const float *beta,
                         const float *g, const OutArgs &out, const float *s0, float *s_final, const int *cu,
                         int nctas, int H, int L, float scale, cudaStream_t stream) {
    auto kern = tc_gdn_cl_kernel<GATED, OPTS>;
    if (!ensure_smem_limit(reinterpret_cast<const void *>(kern), kSmemAlloc)) return GDN_ERR_CUDA;
    unsigned *err = device_error_word();
    if (!err) return GDN_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(nctas) * kCluster);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemAlloc;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const long long limit = wait_limit_cycles();
    return cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, beta, g, out, s0, s_final, cu, H, L, scale, limit, err) ==
                   cudaSuccess
               ? GDN_OK
               : GDN_ERR_CUDA;
}

}  // namespace

bool tc_gdn_cluster_fits(int nctas) { return static_cast<long long>(nctas) * kCluster <= sm_count(); }

gdn_status_t launch_tc_gdn_cluster(const void *q, const void *k, const void *v, const float *beta, const float *g,
                                   void *o, const float *s0, float *s_final, const int *cu, int B, int H, int L,
                                   float scale, FwdOpts oo, cudaStream_t stream) {
    const int nctas = B * H;                 // one cluster per (sequence, head)
    const OutArgs out = make_out_args(o, v, oo);
    const int rows = cu ? H : B * H;         // rows of the (rows, L) token grid
    CUtensorMap mq, mk, mv;
    if (!make_qkv_map(&mq, q, L, rows) || !make_qkv_map(&mk, k, L, rows) || !make_qkv_map(&mv, v, L, rows))
        return GDN_ERR_CUDA;
    const bool opts = oo.bf16 || oo.dskip != nullptr || oo.xnorm != kXNormNone;   // the general output epilogue
    if (g) return opts ? launch_cl_t<true, true>(mq, mk, mv, beta, g, out, s0, s_final, cu, nctas, H, L, scale, stream)
                       : launch_cl_t<true, false>(mq, mk, mv, beta, g, out, s0, s_final, cu, nctas, H, L, scale, stream);
    return opts ? launch_cl_t<false, true>(mq, mk, mv, beta, g, out, s0, s_final, cu, nctas, H, L, scale, stream)
                : launch_cl_t<false, false>(mq, mk, mv, beta, g, out, s0, s_final, cu, nctas, H, L, scale, stream);
}

}  // namespace gdn
