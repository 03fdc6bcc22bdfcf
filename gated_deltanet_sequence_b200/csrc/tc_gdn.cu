// Tensor-core chunkwise DeltaNet / Gated DeltaNet prefill for sm_100a
// (bf16 inputs, dk = dv = 128, chunk C = 64; fp32 accumulation, output and state).
//
// One CTA per (batch, head) walks the chunks in order; the fp32 state S (dk x dv)
// lives in tensor memory for the whole sequence and goes to HBM only at the end.
// Per chunk of C rows (page "混合注意力学习(1)", sections "DeltaNet 分块并行机制",
// "重新定义降低内存占用", "HouseHolder变换和WY表示"; page "LinearAttention 概述", section
// "FLASH"), with G the within-chunk cumulative sum of g, gamma = exp(G),
// Gamma_rs = exp(G_r - G_s) (s <= r) and d_s = exp(G_last - G_s):
//   Gram   [K;Q] K^T                     one M=128 UMMA (rows: K K^T, then Q K^T)
//   UT     A = tril(diag(beta) KK^T o Gamma, -1), T = (I + A)^-1   (forward subst.)
//   W, U   W^T = K^T (T diag(beta gamma))^T, U^T = V^T (T diag(beta))^T
//   Ut/out [O^T | Ut^T] += S^T [Q'^T | -W^T]   (one N=128 product: O^T starts at zero, Ut^T
//          at U^T), Q' = diag(scale gamma) Q
//   out    O^T += Ut^T (scale Q K^T o Gamma)^T
//   state  S <- gamma_last S + (diag(d) K)^T Ut   (K scaled in place once W/U has read it)
// Every product has dk or dv (= 128) as the UMMA M dimension, so each tcgen05.mma
// is a full 128-lane instruction and TMEM lane = row of the result. An M=128, K=16
// tcgen05.mma issued back to back takes about 49 cycles at N=64 and 65 at N=128 on this
// part (measured), so the state's two products above, which share their A operand, run as
// one N=128 product: the serial chain issues 8 instructions for them instead of 16 (Q'^T
// and -W are stored MN-major, one operand stride apart in each key half).
//
// Warp roles (512 threads):
//   warp 0      TMA producer (2-stage ring of Q, K, V tiles)
//   warp 1      issues the Gram UMMA of each chunk as soon as its tiles land
//   warp 2      issues the chain UMMAs (U - W S, output, state) and the next W/U
//   warp 3      gate warp: cumulative log-decay G, gamma = exp(G), d, exp(-G), beta
//   warps 4-7   "state" group: S -> fp16 operand, Ut epilogue, output stores, and
//               the W epilogue of the next chunk (in its idle slot)
//   warps 8-15  "prep" group, one chunk ahead of the state chain: A / P masks, the
//               blocked UT solve on warps 8-11 (16 x 16 diagonal blocks by substitution,
//               off-diagonal blocks by warp-level tf32 MMA) while warps 12-15 convert the
//               tiles with the Q scaling, then the fp16 T factors
// so the state-independent work of chunk c+1 overlaps the serial state chain of
// chunk c. Hand-offs are mbarriers with one arrival each.
//
// Decay factors: Gamma_rs = exp(G_r - G_s) is formed as gamma_r * exp(-G_s) when the
// chunk's total log-decay G_last >= -60 (both factors then stay far inside fp32
// range); chunks with stronger decay take one exp per element instead.
//
// Precision: the Gram product runs on the bf16 input tiles (exact products, fp32
// sums). Every other UMMA takes fp16 operands (10-bit mantissa): K, V are converted
// in place after the Gram has read them, Q is replaced by Q' in fp16, and every
// computed operand (T, P, W, S, Ut) is rounded to fp16, which keeps the rounding of
// the chunk intermediates ~8x below what bf16 operands give. Shared-memory
// operands use the 128-byte swizzled canonical layouts.
#include "tc_gdn_parts.cuh"

namespace gdn {

namespace {
using namespace ptx;
using namespace tcgdn;
constexpr int kThreads = 512;
constexpr int kGroupS = 4;       // first warp of the state group (4 warps)
constexpr int kGroupP = 8;       // first warp of the prep group (8 warps)
constexpr int kNP = 256;         // prep group threads
constexpr int kBarS = 1, kBarP = 2;   // named barriers of the state (128) and prep (256) groups
constexpr int kBarQ = 4;              // the prep group's four converter warps (id 3: its solve warps)
constexpr float kFastDecayLimit = -60.f;   // G_last >= this: Gamma = gamma_r * exp(-G_s)

// ---- shared memory map (byte offsets from a 1024-aligned base) ------------------
constexpr uint32_t kStageBytes = 49152;   // one chunk of K, Q, V; per key half h: [K_h Q_h V_h]
constexpr uint32_t ST_K0 = 0;             // K, key columns 0-63   (64 rows x 128 B)
constexpr uint32_t ST_Q0 = 8192;          // Q, key columns 0-63   (directly after K: [K;Q]); then Q'^T
constexpr uint32_t ST_V0 = 16384;         // V, value columns 0-63; then -W, key rows 0-63
constexpr uint32_t ST_K1 = 24576;         // K, key columns 64-127
constexpr uint32_t ST_Q1 = 32768;         // Q, key columns 64-127; then Q'^T
constexpr uint32_t ST_V1 = 40960;         // V, value columns 64-127; then -W, key rows 64-127
constexpr uint32_t kHalf = ST_K1 - ST_K0;  // stride between the key (or value) halves of a tensor
static_assert(ST_V0 - ST_Q0 == ST_V1 - ST_Q1, "Q'^T and W of a key half must be one operand stride apart");
constexpr uint32_t OFF_AT = 2 * kStageBytes;        // A^T fp32 64 x 64 (UT-solve input)
constexpr uint32_t OFF_TF = OFF_AT + 16384;         // T fp32 64 x 68 (pitch 68)
constexpr int kTP = 68;
constexpr uint32_t OFF_R = OFF_TF + 64 * kTP * 4;   // 4 x 16 x 16 fp32 per-warp block scratch
constexpr uint32_t OFF_PG = OFF_R + 4096;           // 2 x scale (Q K^T o Gamma), K-major 64 x 64
constexpr uint32_t OFF_S = OFF_PG + 16384;          // S as MN-major A: 2 x (128 key rows x 64 v)
constexpr uint32_t OFF_UB = OFF_S + 32768;          // Ut, K-major: 128 value rows x 64 s
constexpr uint32_t OFF_T1 = OFF_UB + 16384;         // T diag(beta gamma), K-major 64 x 64 fp16
constexpr uint32_t OFF_T2 = OFF_T1 + 8192;          // T diag(beta)
constexpr uint32_t OFF_VEC = OFF_T2 + 8192;        // 2 x {G, beta, gamma, d, exp(-G), flag}
constexpr uint32_t kVecBytes = 1536;                //   (64 fp32 each; flag = fast decay path)
constexpr int V_G = 0, V_B = 64, V_GAM = 128, V_D = 192, V_IG = 256, V_FAST = 320;
constexpr uint32_t OFF_XN = OFF_VEC + 2 * kVecBytes;    // output-normalisation scratch (384 fp32)
constexpr uint32_t OFF_BAR = OFF_XN + 1536;             // mbarriers, TMEM base, abort flags
constexpr uint32_t kSmemBytes = OFF_BAR + 512;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;  // slack to align the base to 1024 B
static_assert(kSmemAlloc <= 232448, "shared memory budget");
static_assert(OFF_T1 % 1024 == 0 && OFF_PG % 1024 == 0 && OFF_S % 1024 == 0 && OFF_UB % 1024 == 0,
              "UMMA tiles need 1024-B alignment");

// ---- tensor memory columns (512 allocated) ----------------------------------------
constexpr uint32_t TM_S = 0;      // state S: lane = key row j, 128 value columns
constexpr uint32_t TM_G = 128;    // [K;Q] K^T: lanes 0-63 K K^T, 64-127 Q K^T; 64 columns s
constexpr uint32_t TM_W = 192;    // W^T: lane = key j, 64 columns r
constexpr uint32_t TM_OU = 256;   // 2 x [O^T | U^T then Ut^T]: lane = value v, 64 + 64 columns r

constexpr uint32_t ID_GRAM = idesc_f16(128, 64, false, false, false, /*bf16=*/true);
constexpr uint32_t ID_WU = idesc_f16(128, 64, true, false);
// [O^T | Ut^T] += S^T [Q'^T | -W^T]: one N=128 product for both uses of the state (B = Q'^T and
// -W, MN-major, one operand stride apart)
constexpr uint32_t ID_SQW = idesc_f16(128, 128, true, true);
constexpr uint32_t ID_ST = idesc_f16(128, 128, true, false);
constexpr uint32_t ID_O = idesc_f16(128, 64, false, false);

// mbarriers (index into the barrier array). A parity wait for phase k is only
// correct while the producer cannot complete phase k+1 first; hand-offs whose
// producer may run two chunks ahead of the consumer use one barrier per chunk
// parity (waited with parity (c >> 1) & 1).
enum : int {
    B_FULL = 0,      // [2] TMA -> prep issuer (Gram) and prep group
    B_CDONE = 2,     // [2] state-update UMMAs of chunk c done (frees stage, PG, vec of parity c)
    B_GATE = 4,      // [2] gate warp: vec ready           -> state group
    B_GATEP = 6,     // [2] gate warp: vec ready           -> prep group
    B_PREP = 8,      // [2] prep: P, Q' ready               -> state issuer
    B_TRDY = 10,     // [2] prep: T1/T2, K/V fp16 written  -> prep issuer (W/U)
    B_GRAM = 12,     // Gram done                          -> prep group
    B_GFREE = 13,    // prep group has read the Gram       -> prep issuer (next Gram)
    B_WU = 14,       // W/U done                           -> state group (W epilogue)
    B_XFREE = 15,    // state group has read W^T           -> prep issuer (next W/U)
    B_WRDY = 16,     // state group: W operand written     -> state issuer
    B_SRDY = 17,     // state group: S operand written, S scaled -> state issuer
    B_ADONE = 18,    // U - W S and S Q' done              -> state group (Ut epilogue)
    B_URDY = 19,     // state group: Ut operand ready (U^T read) -> chain issuer
    kNumBars = 20
};

// NARROW: head sizes dk_in, dv_in of 64 or 128 (tiles past them load as zeros; plain fp32
// output only); otherwise both are 128 and the arguments are ignored.
template <bool GATED, bool OPTS, bool NARROW>
__global__ void __launch_bounds__(kThreads, 1)
tc_gdn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ beta,
              const float *__restrict__ g, const OutArgs out, const float *__restrict__ s0,
              float *__restrict__ s_final, const int *__restrict__ cu, int H, int Lrow, float scale, int dk_arg,
              int dv_arg, long long wait_limit, unsigned *__restrict__ err_word) {
    static_assert(!(NARROW && OPTS), "the output options need dv = 128");
    const int dk_in = NARROW ? dk_arg : kD, dv_in = NARROW ? dv_arg : kD;
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
            int last[2] = {-1, -1};   // last chunk loaded into each stage
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
            // never leave a copy in flight past the end of the CTA
            for (int s = 0; s < 2; ++s)
                if (last[s] >= 0) ctl.drain(B_FULL + s, (last[s] >> 1) & 1);
        }
    } else if (warp == 1) {
        // ================================================================ Gram issuer
        // [K;Q] K^T of each chunk on its bf16 tiles, as soon as the tiles have landed and
        // the previous Gram has been read
        if (lane == 0) {
            int gram_last = -1;
            for (int c = 0; c < nchunks; ++c) {
                const int s = c & 1;
                const uint32_t stg = sb + s * kStageBytes;
                if (!ctl.wait_lazy(B_FULL + s, (c >> 1) & 1)) break;
                if (c >= 1 && !ctl.wait_lazy(B_GFREE, (c - 1) & 1)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32u;
                    mma_f16(tmem + TM_G, sdesc_sw128(stg + ST_K0 + off, 16, 1024),
                            sdesc_sw128(stg + ST_K0 + off, 16, 1024), ID_GRAM, kk > 0);
                }
                mma_commit(&bars[B_GRAM]);
                gram_last = c;
            }
            if (gram_last >= 0) ctl.drain(B_GRAM, gram_last & 1);
        }
    } else if (warp == 2) {
        // ================================================================ chain UMMA issuer
        // per chunk: U - W S and S Q' ; state update and P Ut ; then W/U of the next chunk
        if (lane == 0) {
            auto wu = [&](int c) {
                const uint32_t stg = sb + (c & 1) * kStageBytes;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f16(tmem + TM_W, sdesc_sw128(stg + ST_K0 + kk * 2048, kHalf, 1024),
                            sdesc_sw128(sb + OFF_T1 + kk * 32, 16, 1024), ID_WU, kk > 0);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f16(tmem + TM_OU + (c & 1) * 128 + 64, sdesc_sw128(stg + ST_V0 + kk * 2048, kHalf, 1024),
                            sdesc_sw128(sb + OFF_T2 + kk * 32, 16, 1024), ID_WU, kk > 0);
                mma_commit(&bars[B_WU]);
            };
            int last_bar = -1, last_par = 0;   // last commit, for the final drain
            if (nchunks > 0 && ctl.wait(B_TRDY, 0)) {
                wu(0);
                last_bar = B_WU;
                last_par = 0;
            }
            for (int c = 0; last_bar >= 0 && c < nchunks; ++c) {
                const int s = c & 1;
                const uint32_t stg = sb + s * kStageBytes;
                if (!ctl.wait(B_PREP + s, (c >> 1) & 1)) break;
                if (!ctl.wait(B_WRDY, c & 1)) break;
                if (!ctl.wait(B_SRDY, c & 1)) break;
                tc_fence_after();
                // [O^T | Ut^T] += S^T [Q'^T | -W^T]  (O^T starts zeroed, Ut^T holds U^T): the
                // output's state part and U - W S in one N=128 product
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_f16(tmem + TM_OU + s * 128, sdesc_sw128(sb + OFF_S + kk * 2048, 16384, 1024),
                            sdesc_sw128(stg + (kk >> 2) * kHalf + ST_Q0 + (kk & 3) * 2048, ST_V0 - ST_Q0, 1024),
                            ID_SQW, 1u);
                mma_commit(&bars[B_ADONE]);
                last_bar = B_ADONE;
                last_par = c & 1;
                if (!ctl.wait(B_URDY, c & 1)) break;
                tc_fence_after();
                // S += (diag(d) K)^T Ut ;  O^T += Ut^T PG^T
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f16(tmem + TM_S, sdesc_sw128(stg + ST_K0 + kk * 2048, kHalf, 1024),
                            sdesc_sw128(sb + OFF_UB + kk * 32, 16, 1024), ID_ST, 1u);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f16(tmem + TM_OU + s * 128, sdesc_sw128(sb + OFF_UB + kk * 32, 16, 1024),
                            sdesc_sw128(sb + OFF_PG + s * 8192 + kk * 32, 16, 1024), ID_O, 1u);
                mma_commit(&bars[B_CDONE + s]);
                last_bar = B_CDONE + s;
                last_par = (c >> 1) & 1;
                if (c + 1 < nchunks) {
                    // W/U of the next chunk: its T factors, and W^T of this chunk read
                    if (!ctl.wait(B_TRDY + ((c + 1) & 1), ((c + 1) >> 1) & 1)) break;
                    if (!ctl.wait(B_XFREE, c & 1)) break;
                    wu(c + 1);
                    last_bar = B_WU;
                    last_par = (c + 1) & 1;
                }
            }
            // UMMAs complete in issue order: the last commit covers everything issued
            if (last_bar >= 0) ctl.drain(last_bar, last_par);
        }
    } else if (warp >= kGroupS && warp < kGroupS + 4) {
        // ================================================================ state group
        const int j = tid - kGroupS * 32;                // = TMEM lane (key row j / value column v)
        const bool lead = (j == 0);
        const int head = zc % H;                         // head of this row (dense and packed grids)
        float *xn = reinterpret_cast<float *>(smem + OFF_XN);
        const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        {
            // row j of S0 (dk_in x dv_in; rows and columns beyond them are zero)
            const float *src = s0 && j < dk_in ? s0 + (static_cast<size_t>(bh) * dk_in + j) * dv_in : nullptr;
#pragma unroll 1
            for (int cc = 0; cc < 8; ++cc) {
                float r[16];
#pragma unroll
                for (int e = 0; e < 16; e += 4) {
                    const bool in = src && cc * 16 < dv_in &&
                                    in_bounds((static_cast<long long>(bh) * dk_in + j) * dv_in + cc * 16 + e + 3, n_state,
                                              err_word);
                    const float4 x = in ? *reinterpret_cast<const float4 *>(src + cc * 16 + e)
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                    r[e] = x.x; r[e + 1] = x.y; r[e + 2] = x.z; r[e + 3] = x.w;
                }
                tmem_st16(trow + TM_S + cc * 16, r);
            }
            // the O^T tiles start at zero (the merged state product accumulates onto them)
            float z[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) z[e] = 0.f;
#pragma unroll 1
            for (int cc = 0; cc < 8; ++cc) tmem_st16(trow + TM_OU + (cc >> 2) * 128 + (cc & 3) * 16, z);
            tmem_wait_st();
        }
        int done = 0;   // chunks whose output tile has been stored
        float nf = 0.f;  // non-finite probe over sampled output tiles and the final state
        // output tile of chunk cp (n rows): the general epilogue (dv = 128) with the output
        // options, else fp32 rows of dv_in columns (lanes j >= dv_in are whole warps: no store)
        auto store_tile = [&](int cp, int n, bool probe) {
            const uint32_t taddr = trow + TM_OU + (cp & 1) * 128;
            if constexpr (OPTS) {
                store_out_col<OPTS>(taddr, out, (row0 + static_cast<size_t>(cp) * kC) * kD + j, n, head, j, kBarS, xn,
                                    probe, nf);
            } else if (j < dv_in) {
                float ov[64];
                ld_cols<64>(taddr, ov);
                float *ocol = static_cast<float *>(out.o) + (row0 + static_cast<size_t>(cp) * kC) * dv_in + j;
#pragma unroll
                for (int r = 0; r < 64; ++r)
                    if (r < n && in_bounds((static_cast<long long>(row0) + cp * kC + r) * dv_in + j, n_rows * dv_in,
                                           err_word))
                        ocol[static_cast<size_t>(r) * dv_in] = ov[r];
                if (probe) probe_tile(nf, ov, n);
            }
        };
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            const float *vec = reinterpret_cast<const float *>(smem + OFF_VEC + s * kVecBytes);
            uint8_t *st = smem + s * kStageBytes;
            // S(c) complete, and this chunk's gate values
            if (!ctl.group_wait_all({c >= 1 ? B_CDONE + ((c - 1) & 1) : -1, B_GATE + s},
                                    {static_cast<uint32_t>((c - 1) >> 1) & 1u, static_cast<uint32_t>(c >> 1) & 1u},
                                    kBarS, lead))
                break;
            tc_fence_after();
            // ---- S row j -> fp16 MN-major operand; S <- gamma_last S (ahead of the update)
            {
                const float gl = GATED ? vec[V_GAM + 63] : 1.f;
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    float sv[16];
                    tmem_ld16(trow + TM_S + cc * 16, sv);
                    tmem_wait_ld();
                    st_row16_h(sb + OFF_S + (cc >> 2) * 16384u, j, (cc & 3) * 2, sv);
                    if (GATED) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) sv[e] *= gl;
                        tmem_st16(trow + TM_S + cc * 16, sv);
                    }
                }
                if (GATED) tmem_wait_st();
            }
            fence_proxy_async();
            tc_fence_before();
            named_bar(kBarS, 128);
            if (lead) mbar_arrive(&bars[B_SRDY]);
            // ---- W operand of this chunk (its V slot is consumed) and K <- diag(d) K
            //      (K's last reader before the state update was W/U)
            if (!ctl.group_wait(B_WU, c & 1, kBarS, lead)) break;
            tc_fence_after();
            {
                // W^T row j -> -W, MN-major: row j % 64 of the V slot of key half j / 64
                const uint32_t wtile = sb + s * kStageBytes + (j >> 6) * kHalf + ST_V0;
#pragma unroll 1
                for (int cc = 0; cc < 4; ++cc) {
                    float w[16];
                    tmem_ld16(trow + TM_W + cc * 16, w);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) w[e] = -w[e];
                    st_row16_h(wtile, j & 63, 2 * cc, w);
                }
            }
            if (GATED) {
                // K tiles: 2 x 8 KB at ST_K0 / ST_K1, 64 rows of 128 B each; 1024 chunks of 16 B
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint32_t idx = static_cast<uint32_t>(i * 128 + j);
                    const uint32_t off = (idx >> 9) * kHalf + ST_K0 + (idx & 511u) * 16u;
                    const __half2 f = __float2half2_rn(vec[V_D + ((idx & 511u) >> 3)]);
                    uint4 x = *reinterpret_cast<const uint4 *>(st + off);
                    __half2 *hh = reinterpret_cast<__half2 *>(&x);
#pragma unroll
                    for (int e = 0; e < 4; ++e) hh[e] = __hmul2(hh[e], f);
                    *reinterpret_cast<uint4 *>(st + off) = x;
                }
            }
            fence_proxy_async();
            tc_fence_before();
            named_bar(kBarS, 128);
            if (lead) {
                mbar_arrive(&bars[B_WRDY]);
                mbar_arrive(&bars[B_XFREE]);
            }
            // ---- output of the previous chunk (its O tile is complete)
            if (c >= 1) {
                const int cp = c - 1;
                store_tile(cp, kC, false);   // the last tile is stored (and probed) after the loop
                // chunk c + 1 accumulates onto this tile: zero it (ordered before that chunk's
                // product by this group's state-ready hand-off)
                float z[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) z[e] = 0.f;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) tmem_st16(trow + TM_OU + (cp & 1) * 128 + cc * 16, z);
                tmem_wait_st();
                done = c;
            }
            // ---- Ut^T row v -> Ut operand (K-major, rows v)
            if (!ctl.group_wait(B_ADONE, c & 1, kBarS, lead)) break;
            tc_fence_after();
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                float u[16];
                tmem_ld16(trow + TM_OU + s * 128 + 64 + cc * 16, u);
                tmem_wait_ld();
                st_row16_h(sb + OFF_UB, j, 2 * cc, u);
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
                store_tile(cp, L - cp * kC, true);
                done = nchunks;
            }
        }
        if (s_final && done == nchunks && j < dk_in) {
            // row j of the dk_in x dv_in final state (lanes j >= dk_in are whole warps)
            float *dst = s_final + (static_cast<size_t>(bh) * dk_in + j) * dv_in;
#pragma unroll 1
            for (int cc = 0; cc < dv_in / 16; ++cc) {
                float sv[16];
                tmem_ld16(trow + TM_S + cc * 16, sv);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; e += 4) {
                    probe_finite(nf, sv[e] + sv[e + 1] + sv[e + 2] + sv[e + 3]);
                    if (in_bounds((static_cast<long long>(bh) * dk_in + j) * dv_in + cc * 16 + e + 3, n_state, err_word))
                        *reinterpret_cast<float4 *>(dst + cc * 16 + e) = make_float4(sv[e], sv[e + 1], sv[e + 2], sv[e + 3]);
                }
            }
        }
        report_nonfinite(ctl.aborted() ? 0.f : nf, err_word);
    } else if (warp >= kGroupP) {
        // ================================================================ prep group
        const int p = tid - kGroupP * 32;                // 0..255
        const int w8 = warp - kGroupP;                   // 0..7
        const int sub = warp & 3;                        // TMEM lane quarter of this warp
        const int hh = w8 >> 2;                          // which 32 of the 64 Gram columns
        const uint32_t trow = tmem + (static_cast<uint32_t>(sub * 32) << 16);
        for (int i = p; i < 16384 / 16; i += kNP)          // T1/T2: upper blocks stay zero
            *reinterpret_cast<uint4 *>(smem + OFF_T1 + i * 16) = make_uint4(0u, 0u, 0u, 0u);
        float *At = reinterpret_cast<float *>(smem + OFF_AT);   // At[s * 64 + r] = A[r][s]
        float *Tf = reinterpret_cast<float *>(smem + OFF_TF);   // Tf[r * kTP + c] = T[r][c]
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            const float *vec = reinterpret_cast<const float *>(smem + OFF_VEC + s * kVecBytes);
            uint8_t *st = smem + s * kStageBytes;
            // PG of parity s is free once chunk c-2 is complete; then this chunk's gate
            // values, its tiles and its Gram
            if (!ctl.group_wait_all({c >= 2 ? B_CDONE + s : -1, B_GATEP + s, B_FULL + s, B_GRAM},
                                    {static_cast<uint32_t>((c - 2) >> 1) & 1u, static_cast<uint32_t>(c >> 1) & 1u,
                                     static_cast<uint32_t>(c >> 1) & 1u, static_cast<uint32_t>(c) & 1u},
                                    kBarP, p == 0, kNP))
                break;
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
                        st_shared_v4(sb + OFF_PG + s * 8192 + sw128(r, 4 * hh + ch), pack_h2(pv[8 * ch], pv[8 * ch + 1]),
                                     pack_h2(pv[8 * ch + 2], pv[8 * ch + 3]), pack_h2(pv[8 * ch + 4], pv[8 * ch + 5]),
                                     pack_h2(pv[8 * ch + 6], pv[8 * ch + 7]));
                }
            }
            named_bar(kBarP, kNP);                           // A^T complete
            bool solve_ok = true;                            // the solve warps' wait for W/U (c-1)
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
                    st_shared_v4(sb + OFF_T2 + off, pack_h2(u[0], u[1]), pack_h2(u[2], u[3]), pack_h2(u[4], u[5]),
                                 pack_h2(u[6], u[7]));
                    st_shared_v4(sb + OFF_T1 + off, pack_h2(u[0] * gg[0], u[1] * gg[1]),
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
                if (c >= 1) solve_ok = ctl.group_wait(B_WU, (c - 1) & 1, 3, p == 0, 128);
                else asm volatile("bar.sync 3, 128;" ::: "memory");
                if (solve_ok) {
                    emit(bi, bi);
                    float *Rw = reinterpret_cast<float *>(smem + OFF_R);
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
            } else {
                // ---- meanwhile (the Gram has read the tiles): K, V bf16 -> fp16 in place and
                //      Q -> Q'^T = fp16(scale gamma q)^T into the Q slots (128 threads)
                const int t4 = p - 128;                      // 0..127
                // K and V: 2048 chunks of 16 B in the K0, K1, V0, V1 slots
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    uint4 x[8];
                    uint32_t offs[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const uint32_t idx = static_cast<uint32_t>((part * 8 + i) * 128 + t4);   // 0..2047
                        const uint32_t reg = idx >> 9;                                            // 0..3
                        offs[i] = (reg & 1u) * kHalf + (reg < 2 ? ST_K0 : ST_V0) + (idx & 511u) * 16u;
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
                // Q -> Q'^T = fp16(scale gamma_r q_r)^T, transposed in place into the Q slots
                // (MN-major: row k % 64 of the slot of key half k / 64 holds the 64 values r).
                // Thread t4 takes row r = t4 % 64 and the logical 16-byte chunks kc = t4 / 64 + 2i
                // (i < 4) of both key halves; all eight are read before any is overwritten, and a
                // warp's threads then write consecutive r of one row (no bank conflicts)
                {
                    const int r = t4 & 63, kc0 = t4 >> 6;
                    const float f = scale * vec[V_GAM + r];
                    uint4 x[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int h = i >> 2, kc = kc0 + 2 * (i & 3);
                        x[i] = *reinterpret_cast<const uint4 *>(st + h * kHalf + ST_Q0 + r * 128 + ((kc ^ (r & 7)) << 4));
                    }
                    named_bar(kBarQ, 128);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int h = i >> 2, kc = kc0 + 2 * (i & 3);
                        const uint32_t w[4] = {x[i].x, x[i].y, x[i].z, x[i].w};
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float q = (e & 1) ? bf_hi(w[e >> 1]) : bf_lo(w[e >> 1]);
                            const int kr = 8 * kc + e;                   // key row within the half
                            __half *dst = reinterpret_cast<__half *>(st + h * kHalf + ST_Q0 + kr * 128 +
                                                                     ((((r >> 3) ^ kr) & 7) << 4)) + (r & 7);
                            *dst = __float2half_rn(f * q);
                        }
                    }
                }
            }
            fence_proxy_async();
            if (named_bar_any(kBarP, kNP, !solve_ok)) break;   // the solve warps gave up waiting
            if (p == 0) {
                mbar_arrive(&bars[B_TRDY + s]);
                mbar_arrive(&bars[B_PREP + s]);
            }
        }
    } else if (warp == 3) {
        // ================================================================ gate warp
        // lane l owns rows 2l, 2l+1 of each chunk; values of chunk c+1 are fetched one
        // chunk ahead to hide the HBM latency
        float g_nx[2] = {0.f, 0.f}, b_nx[2] = {0.f, 0.f};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int t = 2 * lane + e;
            if (t < L && in_bounds(static_cast<long long>(row0) + t, n_rows, err_word)) {
                if (GATED) g_nx[e] = g[row0 + t];
                b_nx[e] = beta[row0 + t];
            }
        }
        bool ok = true;
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            float *vec = reinterpret_cast<float *>(smem + OFF_VEC + s * kVecBytes);
            // vec of parity s is free once chunk c-2 is complete
            if (c >= 2) {
                int w = 1;
                if (lane == 0) w = ctl.wait_lazy(B_CDONE + s, ((c - 2) >> 1) & 1) ? 1 : 0;
                ok = __shfl_sync(0xffffffffu, w, 0) != 0;
                if (!ok) break;
            }
            const float g0 = g_nx[0], g1 = g_nx[1], b0 = b_nx[0], b1 = b_nx[1];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int t = (c + 1) * kC + 2 * lane + e;
                const bool in = c + 1 < nchunks && t < L && in_bounds(static_cast<long long>(row0) + t, n_rows, err_word);
                g_nx[e] = (GATED && in) ? g[row0 + t] : 0.f;
                b_nx[e] = in ? beta[row0 + t] : 0.f;
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
            if (lane == 0) {
                mbar_arrive(&bars[B_GATE + s]);
                mbar_arrive(&bars[B_GATEP + s]);
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
// (BH, L, width) bf16 rows, width 64 or 128, in 64 x 64 boxes: a box past the width (x = 64 of a
// 64-wide tensor) loads as zeros (also used by the linear-attention kernel's narrow launch)
bool make_rows_map(CUtensorMap *m, const void *ptr, int L, int BH, int width) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t row_bytes = static_cast<cuuint64_t>(width) * 2;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(width), static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(BH)};
    const cuuint64_t strides[2] = {row_bytes, static_cast<cuuint64_t>(L) * row_bytes};
    const cuuint32_t box[3] = {64, 64, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_qkv_map(CUtensorMap *m, const void *ptr, int L, int BH) { return make_rows_map(m, ptr, L, BH, 128); }

namespace {

template <bool GATED, bool OPTS, bool NARROW = false>
gdn_status_t launch_gdn_t(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv, const float *beta,
                          const float *g, const OutArgs &out, const float *s0, float *s_final, const int *cu,
                          int nctas, int H, int L, float scale, cudaStream_t stream, int dk = kD, int dv = kD) {
    auto kern = tc_gdn_kernel<GATED, OPTS, NARROW>;
    if (!ensure_smem_limit(reinterpret_cast<const void *>(kern), kSmemAlloc)) return GDN_ERR_CUDA;
    unsigned *err = device_error_word();
    if (!err) return GDN_ERR_CUDA;
    kern<<<nctas, kThreads, kSmemAlloc, stream>>>(mq, mk, mv, beta, g, out, s0, s_final, cu, H, L, scale, dk, dv,
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

bool tc_gdn_takes_narrow(int nctas) { return encode_fn() != nullptr && nctas > 0 && !tc_gdn_cluster_fits(nctas); }

gdn_status_t launch_tc_gdn_narrow(const void *q, const void *k, const void *v, const float *beta, const float *g,
                                  float *o, const float *s0, float *s_final, const int *cu, int B, int H, int L,
                                  int dk, int dv, float scale, cudaStream_t stream) {
    const int nctas = B * H;
    const int rows = cu ? H : B * H;
    const FwdOpts plain{false, nullptr, false, kXNormNone, nullptr, 0.f};
    const OutArgs out = make_out_args(o, v, plain);
    CUtensorMap mq, mk, mv;
    if (!make_rows_map(&mq, q, L, rows, dk) || !make_rows_map(&mk, k, L, rows, dk) ||
        !make_rows_map(&mv, v, L, rows, dv))
        return GDN_ERR_CUDA;
    return g ? launch_gdn_t<true, false, true>(mq, mk, mv, beta, g, out, s0, s_final, cu, nctas, H, L, scale, stream,
                                               dk, dv)
             : launch_gdn_t<false, false, true>(mq, mk, mv, beta, g, out, s0, s_final, cu, nctas, H, L, scale, stream,
                                                dk, dv);
}

}  // namespace gdn
