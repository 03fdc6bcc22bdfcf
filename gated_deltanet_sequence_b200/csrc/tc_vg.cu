// Tensor-core chunkwise prefill with vector-valued gates (one log-decay per token and key
// coordinate) for sm_100a: Gated DeltaNet and gated linear attention, bf16 inputs,
// dk = dv = 128, chunk C = 64, fp32 accumulation, output and state.
//
// The recurrence (page "混合注意力学习(1)", section "Gated DeltaNet", with the decay read per
// key coordinate, a GLA-style gate): row j of the state decays by exp(g_t[j]) before the
// token's read and write,
//   S_t = (I - beta_t k_t k_t^T) diag(exp(g_t)) S_{t-1} + beta_t k_t v_t^T,   o_t = scale S_t^T q_t
// (linear attention: S_t = diag(exp(g_t)) S_{t-1} + k_t v_t^T). Per chunk of C rows, with
// G_r[j] the within-chunk cumulative log-decay of coordinate j up to row r and GL = G of the
// chunk's last row (sections "DeltaNet 分块并行机制" and "HouseHolder变换和WY表示" of the same
// page, with the scalar decay factors replaced by per-coordinate ones):
//   A_rs = beta_r sum_j k_r[j] k_s[j] exp(G_r[j] - G_s[j])    (s < r)
//   P_rs = scale sum_j q_r[j] k_s[j] exp(G_r[j] - G_s[j])      (s <= r)
//   T = (I + A)^-1,  W = T diag(beta) (K o exp(G)),  U = T diag(beta) V
//   Ut = U - W S,   O = (scale Q o exp(G)) S + P Ut,   S <- diag(exp(GL)) S + (K o exp(GL - G))^T Ut
// (linear attention: T = I, W = 0, U = V). Only the last line and the two products with S
// before it depend on the previous chunk, so a call runs as two kernels:
//
//   vg_prep_kernel   one CTA per chunk of every head (two CTAs per SM): the per-coordinate
//                    gate sums, the decay-weighted Gram on the tensor cores, the UT solve and
//                    the W / U products. It writes one record per chunk to a workspace:
//                    Q'^T = (scale Q o exp(G))^T, -W^T, Kd^T = (K o exp(GL - G))^T, U^T and P
//                    (fp16, 128-byte rows), plus exp(GL) (fp32).
//   vg_chain_kernel  one CTA per (sequence, head): the fp32 state lives in tensor memory; per
//                    chunk the record arrives by bulk copies and the chain takes three products,
//                    [O^T | Ut^T] += S^T [Q'^T | -W^T] (Ut^T preloaded with U^T),
//                    S <- exp(GL) o S + Kd^T Ut and O^T += Ut^T P^T.
//
// The decay-weighted Gram: exp(G_r - G_s) = exp(G_r - c) exp(c - G_s) with c[j] the midpoint
// of coordinate j's range of G over the chunk, so the UMMA takes [K o e; Q o e] (K o 1/e)^T
// with fp16 factors within [e^-6, e^6] whenever that range is at most 12 ("fast"
// coordinates). The other coordinates are zero in those tiles and their exact terms,
// one exp per element, are added on the CUDA cores; when more than 32 coordinates of a chunk
// are such, the whole Gram of that chunk is formed that way. Every other factor (exp(G),
// exp(GL - G), exp(GL)) is at most 1 for non-positive log-decays and is formed directly.
#include <algorithm>
#include <mutex>
#include <vector>

#include "tc_gdn_parts.cuh"

namespace gdn {

namespace {
using namespace ptx;
using namespace tcgdn;

__device__ __forceinline__ void st_shared_b32(uint32_t addr, uint32_t a) {
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(a) : "memory");
}
__device__ __forceinline__ float h_lo(uint32_t w) { return __low2float(*reinterpret_cast<const __half2 *>(&w)); }
__device__ __forceinline__ float h_hi(uint32_t w) { return __high2float(*reinterpret_cast<const __half2 *>(&w)); }

// ---- the per-chunk record: fp16 tiles of 128-byte rows, stored as the image of a shared-memory
//      tile in the 128-byte swizzled layout (16-byte chunk c of row R at chunk c ^ (R mod 8)),
//      so that a plain bulk copy into a 1024-aligned buffer yields the UMMA operand layout
constexpr int kRQ = 0;        // Q'^T: row j holds scale q_r[j] exp(G_r[j]), r = 0..63
constexpr int kRW = 128;      // -W^T: row j holds -W[r][j]
constexpr int kRKD = 256;     // Kd^T: row j holds k_r[j] exp(GL[j] - G_r[j])
constexpr int kRU = 384;      // U^T: row v holds U[r][v]
constexpr int kRP = 512;      // P: row r holds P[r][s], s = 0..63
constexpr int kRecRows = 576;
constexpr uint32_t kRecBytes = kRecRows * 128u;   // 73728 (a multiple of 1024)
constexpr uint32_t kRecPiece = kRecBytes / 3;     // one record arrives as three bulk copies
constexpr float kSpanFast = 12.f;                 // coordinate's range of G within a chunk, factored Gram
constexpr int kSlowCap = 32;                      // at most this many exact coordinates next to the UMMA Gram

__device__ __forceinline__ void bulk_s2g(void *gdst, uint32_t ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(ssrc), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_g2s(uint32_t sdst, const void *gsrc, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(sdst),
                 "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// ================================================================== prep kernel
constexpr int kVPThreads = 256;
// shared memory (byte offsets from a 1024-aligned base); regions and their successive uses
constexpr uint32_t X0 = 0;        // per key half h at h * 16384: [K o e^(G-c) rows | Q o e^(G-c) rows];
                                  // the K rows stay (A operand of W^T); the Q rows then hold V (TMA)
constexpr uint32_t X1 = 32768;    // K o e^(c-G), per key half at h * 8192; then T diag(beta) (8 KB);
                                  // then -W^T (16 KB)
constexpr uint32_t X2 = 49152;    // gate sums, exact-coordinate data (up to 32), A^T fp32; then U^T
constexpr uint32_t X3 = 65536;    // Q'^T and Kd^T (32 KB); then T fp32 (pitch 68), the solve's block
                                  // scratch and P (8 KB)
constexpr uint32_t XS = X1;       // every coordinate exact: G fp32 32 KB, k and q bf16 16 KB each (X1-X3)
constexpr uint32_t VP_TF = X3, VP_RS = X3 + 17408, VP_P = X3 + 22528;
constexpr int kTP = 68;
constexpr uint32_t VP_VEC = 98304;   // beta[64] | c[128] | slot u8[128] | count | bars | tmem | abort |
                                     // scalar gate: G[64], exp(G)[64], exp(-G)[64], factored flag
constexpr uint32_t kVPSmem = VP_VEC + 2048;
constexpr uint32_t kVPAlloc = kVPSmem + 1024;
static_assert(kVPAlloc * 2 + 2048 <= 233472, "two prep CTAs per SM");
static_assert(VP_P + 8192 <= X3 + 32768, "P after T and the block scratch");
constexpr uint32_t V_BETA = 0, V_C = 256, V_SLOT = 768, V_NSLOW = 896, V_BARS = 928, V_TMEM = 960, V_ABORT = 964;
constexpr uint32_t V_GROW = 1024, V_GAM = 1280, V_IG = 1536, V_FACT = 1792;
constexpr float kFastDecayLimit = -60.f;   // scalar gate, G_last >= this: exp(G_r - G_s) = exp(G_r) exp(-G_s)
// tensor memory (256 columns)
constexpr uint32_t TMV_G = 0, TMV_W = 64, TMV_U = 128;
constexpr uint32_t ID_G16 = idesc_f16(128, 64, false, false);   // Gram: both K-major, fp16
constexpr uint32_t ID_WU = idesc_f16(128, 64, true, false);     // W^T, U^T: A MN-major
enum : int { VB_V = 0, VB_G = 1, VB_WU = 2, kVPBars = 3 };

// SCALAR: g holds one log-decay per token (or is null); the Gram then runs on the plain tiles and
// the masks take exp(G_r - G_s) per element. CTA i takes chunk cbase + i % nseg of head i / nseg
// and writes record i.
template <bool DELTA, bool SCALAR>
__global__ void __launch_bounds__(kVPThreads, 2)
vg_prep_kernel(const __grid_constant__ CUtensorMap tm_v, const __nv_bfloat16 *__restrict__ q,
               const __nv_bfloat16 *__restrict__ k, const float *__restrict__ beta, const float *__restrict__ g,
               uint8_t *__restrict__ recs, float *__restrict__ egl, int L, int cbase, int nseg, float scale,
               long long wait_limit, unsigned *__restrict__ err_word) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(smem);
    uint8_t *vec = smem + VP_VEC;
    uint64_t *bars = reinterpret_cast<uint64_t *>(vec + V_BARS);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(vec + V_TMEM);
    int *abort_flag = reinterpret_cast<int *>(vec + V_ABORT);
    const Ctl ctl{bars, abort_flag, err_word, wait_limit};
    float *betav = reinterpret_cast<float *>(vec + V_BETA);
    float *cv = reinterpret_cast<float *>(vec + V_C);
    uint8_t *slot = vec + V_SLOT;
    int *nslow_p = reinterpret_cast<int *>(vec + V_NSLOW);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long rec_id = blockIdx.x;
    const int bh = static_cast<int>(rec_id / nseg);
    const int c = cbase + static_cast<int>(rec_id - static_cast<long long>(bh) * nseg);
    const int nvalid = min(kC, L - c * kC);
    const size_t row0 = static_cast<size_t>(bh) * L + static_cast<size_t>(c) * kC;
    uint8_t *rec = recs + static_cast<size_t>(rec_id) * kRecBytes;

    if (tid == 0) {
        for (int b = 0; b < kVPBars; ++b) mbar_init(&bars[b], 1);
        *abort_flag = 0;
        *nslow_p = 0;
        fence_mbar_init();
        prefetch_tmap(&tm_v);
    }
    if (tid < kC) betav[tid] = (DELTA && tid < nvalid) ? beta[row0 + tid] : 0.f;
    if (warp == 0) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }

    // ---- gate sums and the operand tiles: thread (p, h) takes coordinates 2p, 2p+1 and
    //      rows 16h .. 16h+15
    const int p = tid & 63, h = tid >> 6;
    const int j0 = 2 * p, kh = j0 >> 6, jc = j0 & 63, r0 = 16 * h;
    float G0[16], G1[16];
    uint32_t kw[16], qw[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int r = r0 + i;
        if (r < nvalid) {
            const size_t e = (row0 + r) * kD + j0;
            if constexpr (SCALAR) {
                G0[i] = G1[i] = g ? g[row0 + r] : 0.f;
            } else {
                const float2 gg = *reinterpret_cast<const float2 *>(g + e);
                G0[i] = gg.x;
                G1[i] = gg.y;
            }
            kw[i] = *reinterpret_cast<const uint32_t *>(k + e);
            qw[i] = *reinterpret_cast<const uint32_t *>(q + e);
        } else {
            G0[i] = G1[i] = 0.f;
            kw[i] = qw[i] = 0u;
        }
    }
#pragma unroll
    for (int i = 1; i < 16; ++i) {
        G0[i] += G0[i - 1];
        G1[i] += G1[i - 1];
    }
    float *tot = reinterpret_cast<float *>(smem + X2);   // [4][128] quarter sums, then min, max
    tot[h * 128 + j0] = G0[15];
    tot[h * 128 + j0 + 1] = G1[15];
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    float o0 = 0.f, o1 = 0.f, gl0 = 0.f, gl1 = 0.f;
#pragma unroll
    for (int hh = 0; hh < 4; ++hh) {
        const float a = tot[hh * 128 + j0], b = tot[hh * 128 + j0 + 1];
        if (hh < h) {
            o0 += a;
            o1 += b;
        }
        gl0 += a;
        gl1 += b;
    }
    float mn0 = 3.0e38f, mx0 = -3.0e38f, mn1 = 3.0e38f, mx1 = -3.0e38f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        G0[i] += o0;
        G1[i] += o1;
        mn0 = fminf(mn0, G0[i]);
        mx0 = fmaxf(mx0, G0[i]);
        mn1 = fminf(mn1, G1[i]);
        mx1 = fmaxf(mx1, G1[i]);
    }
    tot[512 + h * 128 + j0] = mn0;
    tot[512 + h * 128 + j0 + 1] = mn1;
    tot[1024 + h * 128 + j0] = mx0;
    tot[1024 + h * 128 + j0 + 1] = mx1;
    __syncthreads();
    float lo0 = tot[512 + j0], lo1 = tot[512 + j0 + 1], hi0 = tot[1024 + j0], hi1 = tot[1024 + j0 + 1];
#pragma unroll
    for (int hh = 1; hh < 4; ++hh) {
        lo0 = fminf(lo0, tot[512 + hh * 128 + j0]);
        lo1 = fminf(lo1, tot[512 + hh * 128 + j0 + 1]);
        hi0 = fmaxf(hi0, tot[1024 + hh * 128 + j0]);
        hi1 = fmaxf(hi1, tot[1024 + hh * 128 + j0 + 1]);
    }
    // factored Gram coordinates (false for NaN ranges); the scalar gate takes the plain tiles
    const bool f0 = SCALAR || hi0 - lo0 <= kSpanFast, f1 = SCALAR || hi1 - lo1 <= kSpanFast;
    if (h == 0) {
        if (!f0) slot[j0] = static_cast<uint8_t>(atomicAdd(nslow_p, 1));
        if (!f1) slot[j0 + 1] = static_cast<uint8_t>(atomicAdd(nslow_p, 1));
        egl[static_cast<size_t>(rec_id) * kD + j0] = __expf(gl0);
        egl[static_cast<size_t>(rec_id) * kD + j0 + 1] = __expf(gl1);
    }
    __syncthreads();   // gate sums read; the exact-coordinate slots are assigned
    const int nslow = *nslow_p;
    const bool allslow = nslow > kSlowCap;
    const bool fa0 = !SCALAR && f0 && !allslow, fa1 = !SCALAR && f1 && !allslow;
    // reference c of the factors: the midpoint of the range for factored coordinates, else 0
    const float c0 = fa0 ? 0.5f * (lo0 + hi0) : 0.f, c1 = fa1 ? 0.5f * (lo1 + hi1) : 0.f;
    if (h == 0) {
        cv[j0] = c0;
        cv[j0 + 1] = c1;
    }
    if (SCALAR && tid == 0) *reinterpret_cast<int *>(vec + V_FACT) = gl0 >= kFastDecayLimit ? 1 : 0;
    const float ec0 = fa0 ? __expf(c0) : 0.f, ec1 = fa1 ? __expf(c1) : 0.f;
    const float edc0 = fa0 ? __expf(gl0 - c0) : 0.f, edc1 = fa1 ? __expf(gl1 - c1) : 0.f;
    uint32_t qT0[8], qT1[8], dT0[8], dT1[8];   // fp16 pairs along r for the transposed rows
    float pq0 = 0.f, pq1 = 0.f, pd0 = 0.f, pd1 = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int r = r0 + i;
        const float k0 = bf_lo(kw[i]), k1 = bf_hi(kw[i]), q0 = bf_lo(qw[i]), q1 = bf_hi(qw[i]);
        // K o e^(G-c) (Gram A rows, and W's operand), Q o e^(G-c), K o e^(c-G) (Gram B rows)
        float ka0, qa0 = 0.f, kb0 = 0.f, eg0, ed0, ka1, qa1 = 0.f, kb1 = 0.f, eg1, ed1;
        if constexpr (SCALAR) {
            // plain tiles; exp(G_r) and exp(GL - G_r) once per row
            eg0 = eg1 = __expf(G0[i]);
            ed0 = ed1 = __expf(gl0 - G0[i]);
            ka0 = kb0 = k0;
            ka1 = kb1 = k1;
            qa0 = q0;
            qa1 = q1;
            if (p == 0) {
                reinterpret_cast<float *>(vec + V_GROW)[r] = G0[i];
                reinterpret_cast<float *>(vec + V_GAM)[r] = eg0;
                reinterpret_cast<float *>(vec + V_IG)[r] = gl0 >= kFastDecayLimit ? __expf(-G0[i]) : 0.f;
            }
        } else if (fa0) {
            const float e1 = __expf(G0[i] - c0), e2 = __expf(c0 - G0[i]);
            ka0 = k0 * e1;
            qa0 = q0 * e1;
            kb0 = k0 * e2;
            eg0 = e1 * ec0;
            ed0 = e2 * edc0;
        } else {
            eg0 = __expf(G0[i]);
            ed0 = __expf(gl0 - G0[i]);
            ka0 = k0 * eg0;
        }
        if (SCALAR) {
        } else if (fa1) {
            const float e1 = __expf(G1[i] - c1), e2 = __expf(c1 - G1[i]);
            ka1 = k1 * e1;
            qa1 = q1 * e1;
            kb1 = k1 * e2;
            eg1 = e1 * ec1;
            ed1 = e2 * edc1;
        } else {
            eg1 = __expf(G1[i]);
            ed1 = __expf(gl1 - G1[i]);
            ka1 = k1 * eg1;
        }
        const uint32_t sw = sw128(r, jc >> 3) + (jc & 7) * 2;
        st_shared_b32(sb + X0 + kh * 16384 + sw, pack_h2(ka0, ka1));
        if (!allslow) {
            st_shared_b32(sb + X0 + kh * 16384 + 8192 + sw, pack_h2(qa0, qa1));
            st_shared_b32(sb + X1 + kh * 8192 + sw, pack_h2(kb0, kb1));
        }
        const float qp0 = scale * q0 * eg0, qp1 = scale * q1 * eg1, kd0 = k0 * ed0, kd1 = k1 * ed1;
        if (i & 1) {
            qT0[i >> 1] = pack_h2(pq0, qp0);
            qT1[i >> 1] = pack_h2(pq1, qp1);
            dT0[i >> 1] = pack_h2(pd0, kd0);
            dT1[i >> 1] = pack_h2(pd1, kd1);
        } else {
            pq0 = qp0;
            pq1 = qp1;
            pd0 = kd0;
            pd1 = kd1;
        }
        if ((i & 7) == 7) {
            // rows j0, j0+1 of Q'^T and Kd^T: the 8 values r = r0 + i - 7 .. r0 + i (one chunk)
            const int b = (i >> 3) * 4;
            const uint32_t ch = 2 * h + (i >> 3);
            st_shared_v4(sb + X3 + sw128(kRQ + j0, ch), qT0[b], qT0[b + 1], qT0[b + 2], qT0[b + 3]);
            st_shared_v4(sb + X3 + sw128(kRQ + j0 + 1, ch), qT1[b], qT1[b + 1], qT1[b + 2], qT1[b + 3]);
            st_shared_v4(sb + X3 + 16384 + sw128(j0, ch), dT0[b], dT0[b + 1], dT0[b + 2], dT0[b + 3]);
            st_shared_v4(sb + X3 + 16384 + sw128(j0 + 1, ch), dT1[b], dT1[b + 1], dT1[b + 2], dT1[b + 3]);
        }
    }
    // exact coordinates next to the UMMA Gram: G (fp32), k and q (bf16) by slot, rows contiguous
    auto put_exact = [&](uint32_t base, int NF) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            if (!allslow && (e ? f1 : f0)) continue;
            const int j = j0 + e;
            const int f = allslow ? j : slot[j];
            const float *Gv = e ? G1 : G0;
            float *sg = reinterpret_cast<float *>(smem + base) + f * 64 + r0;
#pragma unroll
            for (int i = 0; i < 16; i += 4)
                *reinterpret_cast<float4 *>(sg + i) = make_float4(Gv[i], Gv[i + 1], Gv[i + 2], Gv[i + 3]);
            uint32_t kk[8], qq[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t a = kw[2 * i], b = kw[2 * i + 1], x = qw[2 * i], y = qw[2 * i + 1];
                kk[i] = e ? ((a >> 16) | (b & 0xFFFF0000u)) : ((a & 0xFFFFu) | (b << 16));
                qq[i] = e ? ((x >> 16) | (y & 0xFFFF0000u)) : ((x & 0xFFFFu) | (y << 16));
            }
            uint8_t *sk = smem + base + NF * 256 + f * 128 + r0 * 2;
            uint8_t *sq = smem + base + NF * 384 + f * 128 + r0 * 2;
            *reinterpret_cast<uint4 *>(sk) = make_uint4(kk[0], kk[1], kk[2], kk[3]);
            *reinterpret_cast<uint4 *>(sk + 16) = make_uint4(kk[4], kk[5], kk[6], kk[7]);
            *reinterpret_cast<uint4 *>(sq) = make_uint4(qq[0], qq[1], qq[2], qq[3]);
            *reinterpret_cast<uint4 *>(sq + 16) = make_uint4(qq[4], qq[5], qq[6], qq[7]);
        }
    };
    if (!allslow && nslow > 0) put_exact(X2, kSlowCap);
    fence_proxy_async();
    __syncthreads();
    // Q'^T and Kd^T go out; the Gram starts; V is fetched into the Q rows once the Gram has read them
    bool ok = true, issued_v = false;   // issued_v: thread 0's own record of the V copy
    if (tid == 0) {
        bulk_s2g(rec + kRQ * 128, sb + X3, 16384);
        bulk_s2g(rec + kRKD * 128, sb + X3 + 16384, 16384);
        bulk_commit();
        if (!allslow) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_f16(tmem + TMV_G, sdesc_sw128(sb + X0 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                        sdesc_sw128(sb + X1 + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), ID_G16, kk > 0);
            mma_commit(&bars[VB_G]);
            ok = ctl.wait(VB_G, 0);
        } else {
            bulk_wait_read();   // X3 takes the exact-coordinate data next
        }
        if (ok) {
            mbar_arrive_expect_tx(&bars[VB_V], 16384);
            tma_load_3d(smem + X0 + 8192, &tm_v, &bars[VB_V], 0, c * kC, bh);
            tma_load_3d(smem + X0 + 24576, &tm_v, &bars[VB_V], 64, c * kC, bh);
            issued_v = true;
        }
    }
    if (allslow) {
        __syncthreads();
        put_exact(XS, kD);
        __syncthreads();
    } else {
        ok = ctl.wait(VB_G, 0);
        tc_fence_after();
    }
    const bool v_issued = !__syncthreads_or(!ok);   // thread 0 issued V iff every wait so far held
    ok = v_issued;
    const int sub = warp & 3, hh = warp >> 2, R = sub * 32 + lane;
    const int r = R & 63;
    const bool isP = R >= 64;
    const uint32_t trow = tmem + (static_cast<uint32_t>(sub * 32) << 16);
    float v[32];
    if (!allslow && ok) {
        ld_cols<32>(trow + TMV_G + 32 * hh, v);
    } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0.f;
    }
    if (ok && nslow > 0 && r >= 32 * hh && (DELTA || isP)) {
        // exact terms of the coordinates left out of the factored Gram
        const uint32_t sbase = allslow ? XS : X2;
        const int NF = allslow ? kD : kSlowCap;
        const float *SG = reinterpret_cast<const float *>(smem + sbase);
        const __nv_bfloat16 *SK = reinterpret_cast<const __nv_bfloat16 *>(smem + sbase + NF * 256);
        const __nv_bfloat16 *SX = reinterpret_cast<const __nv_bfloat16 *>(smem + sbase + NF * (isP ? 384 : 256));
        const int nf = allslow ? kD : nslow;
#pragma unroll 1
        for (int f = 0; f < nf; ++f) {
            const float Gr = SG[f * 64 + r], xr = __bfloat162float(SX[f * 64 + r]);
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int s = 32 * hh + e;
                if (s < r || (isP && s == r))
                    v[e] = fmaf(xr * __bfloat162float(SK[f * 64 + s]), __expf(Gr - SG[f * 64 + s]), v[e]);
            }
        }
    }
    if (tid == 0) bulk_wait_read();   // Q'^T / Kd^T have left X3 (P and T go there)
    tc_fence_before();
    __syncthreads();   // Gram and exact-coordinate data read: A^T and P may overwrite them
    if constexpr (SCALAR) {
        // the decay of the plain Gram: Gamma_rs = exp(G_r - G_s), factored when G_last >= -60
        const float *Gw = reinterpret_cast<const float *>(vec + V_GROW);
        const float *gam = reinterpret_cast<const float *>(vec + V_GAM);
        const float *ig = reinterpret_cast<const float *>(vec + V_IG);
        const bool fact = *reinterpret_cast<const int *>(vec + V_FACT) != 0;
        const float gr = gam[r], Gr = Gw[r];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const int s2 = 32 * hh + e;
            v[e] *= fact ? gr * ig[s2] : (s2 <= r ? __expf(Gr - Gw[s2]) : 0.f);
        }
    }
    if (!isP) {
        if (DELTA) {
            float *At = reinterpret_cast<float *>(smem + X2);   // At[s * 64 + r] = A[r][s]
            const float br = betav[r];
#pragma unroll
            for (int e = 0; e < 32; ++e) At[(32 * hh + e) * 64 + r] = (32 * hh + e < r) ? br * v[e] : 0.f;
        }
    } else {
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
            float pv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) pv[e] = (32 * hh + 8 * ch + e <= r) ? scale * v[8 * ch + e] : 0.f;
            st_shared_v4(sb + VP_P + sw128(r, 4 * hh + ch), pack_h2(pv[0], pv[1]), pack_h2(pv[2], pv[3]),
                         pack_h2(pv[4], pv[5]), pack_h2(pv[6], pv[7]));
        }
    }
    fence_proxy_async();
    __syncthreads();   // A^T and P complete
    if (tid == 0) {
        bulk_s2g(rec + kRP * 128, sb + VP_P, 8192);
        bulk_commit();
    }

    // ---- UT solve (warps 0-3) while warps 4-7 convert V to fp16
    if (warp < 4) {
        const float *At = reinterpret_cast<const float *>(smem + X2);
        float *Tf = reinterpret_cast<float *>(smem + VP_TF);    // Tf[r * kTP + c] = T[r][c]
        for (int i = tid; i < (SCALAR ? 16384 : 8192) / 16; i += 128)   // T factors: upper blocks stay zero
            *reinterpret_cast<uint4 *>(smem + X1 + i * 16) = make_uint4(0u, 0u, 0u, 0u);
        if (!DELTA) {
            // linear attention: T = I, so T diag(beta) is the identity (U = V)
            asm volatile("bar.sync 3, 128;" ::: "memory");
            if (tid < 64)
                *reinterpret_cast<__half *>(smem + X1 + sw128(tid, tid >> 3) + (tid & 7) * 2) = __float2half_rn(1.f);
        } else {
            // one 16 x 16 block (bi, bj) of Tf -> T diag(beta) (K-major rows r)
            auto emit = [&](int bi2, int bj2) {
                __syncwarp();
                const int rr = 16 * bi2 + (lane >> 1), cc0 = 16 * bj2 + 8 * (lane & 1);
                const float4 b0 = *reinterpret_cast<const float4 *>(betav + cc0);
                const float4 b1 = *reinterpret_cast<const float4 *>(betav + cc0 + 4);
                const float4 t0 = *reinterpret_cast<const float4 *>(Tf + rr * kTP + cc0);
                const float4 t1 = *reinterpret_cast<const float4 *>(Tf + rr * kTP + cc0 + 4);
                st_shared_v4(sb + X1 + sw128(rr, cc0 >> 3), pack_h2(t0.x * b0.x, t0.y * b0.y),
                             pack_h2(t0.z * b0.z, t0.w * b0.w), pack_h2(t1.x * b1.x, t1.y * b1.y),
                             pack_h2(t1.z * b1.z, t1.w * b1.w));
                if constexpr (SCALAR) {
                    // T diag(beta gamma) for W = T diag(beta gamma) K (the plain K tile)
                    const float *gm = reinterpret_cast<const float *>(vec + V_GAM) + cc0;
                    st_shared_v4(sb + X1 + 8192 + sw128(rr, cc0 >> 3), pack_h2(t0.x * b0.x * gm[0], t0.y * b0.y * gm[1]),
                                 pack_h2(t0.z * b0.z * gm[2], t0.w * b0.w * gm[3]),
                                 pack_h2(t1.x * b1.x * gm[4], t1.y * b1.y * gm[5]),
                                 pack_h2(t1.z * b1.z * gm[6], t1.w * b1.w * gm[7]));
                }
            };
            const int bi = warp, cl = lane & 15;
            if (ok) {
                // diagonal block D_i = (I + A_ii)^-1 by right-looking substitution (lane = column)
                float acc[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) acc[i] = (i == cl) ? 1.f : 0.f;
#pragma unroll
                for (int s2 = 0; s2 < 15; ++s2) {
                    const float xs = acc[s2];
                    const float *arow = At + (16 * bi + s2) * 64 + 16 * bi;
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        if (4 * k4 + 3 <= s2) continue;
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
            asm volatile("bar.sync 3, 128;" ::: "memory");
            if (ok) emit(bi, bi);
            float *Rw = reinterpret_cast<float *>(smem + VP_RS);
            // T_10 = -D_1 (A_10 D_0), T_32 = -D_3 (A_32 D_2)
            if (ok && bi < 2) {
                const int i = 2 * bi + 1, j = 2 * bi;
                float *Rb = Rw + bi * 256;
                float acc2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                block_mm<2>(acc2, [&](int rr, int kx) { return At[(16 * j + kx) * 64 + 16 * i + rr]; },
                            [&](int kx, int n) { return Tf[(16 * j + kx) * kTP + 16 * j + n]; }, lane);
                block_store(acc2, [&](int rr, int n, float x) { Rb[rr * 16 + n] = x; }, lane, 1.f);
                __syncwarp();
                float acc3[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                block_mm<2>(acc3, [&](int rr, int kx) { return Tf[(16 * i + rr) * kTP + 16 * i + kx]; },
                            [&](int kx, int n) { return Rb[kx * 16 + n]; }, lane);
                block_store(acc3, [&](int rr, int n, float x) { Tf[(16 * i + rr) * kTP + 16 * j + n] = x; }, lane,
                            -1.f);
                emit(i, j);
            }
            asm volatile("bar.sync 3, 128;" ::: "memory");
            // X_ij = A_{i,0..1} T_{0..1,j} for (i, j) = (2 + w / 2, w % 2)
            const int ii = 2 + (bi >> 1), jj = bi & 1;
            if (ok) {
                float acc2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                if (jj == 0)
                    block_mm<4>(acc2, [&](int rr, int kx) { return At[kx * 64 + 16 * ii + rr]; },
                                [&](int kx, int n) { return Tf[kx * kTP + n]; }, lane);
                else
                    block_mm<2>(acc2, [&](int rr, int kx) { return At[(16 + kx) * 64 + 16 * ii + rr]; },
                                [&](int kx, int n) { return Tf[(16 + kx) * kTP + 16 + n]; }, lane);
                float *Rb = Rw + bi * 256;
                block_store(acc2, [&](int rr, int n, float x) { Rb[rr * 16 + n] = x; }, lane, 1.f);
            }
            asm volatile("bar.sync 3, 128;" ::: "memory");
            // T_2j = -D_2 X_2j,  T_3j = -(T_32 X_2j + D_3 X_3j)
            if (ok) {
                const float *X2p = Rw + jj * 256, *X3p = Rw + (2 + jj) * 256;
                float acc3[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                if (ii == 2)
                    block_mm<2>(acc3, [&](int rr, int kx) { return Tf[(32 + rr) * kTP + 32 + kx]; },
                                [&](int kx, int n) { return X2p[kx * 16 + n]; }, lane);
                else
                    block_mm<4>(acc3, [&](int rr, int kx) { return Tf[(48 + rr) * kTP + 32 + kx]; },
                                [&](int kx, int n) { return kx < 16 ? X2p[kx * 16 + n] : X3p[(kx - 16) * 16 + n]; },
                                lane);
                block_store(acc3, [&](int rr, int n, float x) { Tf[(16 * ii + rr) * kTP + 16 * jj + n] = x; }, lane,
                            -1.f);
                emit(ii, jj);
            }
        }
    } else if (ok) {
        const int t4 = tid - 128;
        bool vok = true;
        if (t4 == 0) vok = ctl.wait(VB_V, 0);
        asm volatile("bar.sync 4, 128;" ::: "memory");
        vok = !ctl.aborted();   // the wait that gave up set the abort flag
        if (vok) {
            convert_tile_bf16_to_f16(smem + X0 + 8192, 8192, t4, 128);
            convert_tile_bf16_to_f16(smem + X0 + 24576, 8192, t4, 128);
        }
        ok = vok;
    }
    fence_proxy_async();
    ok = !__syncthreads_or(!ok);

    // ---- W^T = diag(e^c) (K o e^(G-c))^T (T diag(beta))^T and U^T = V^T (T diag(beta))^T
    const bool wu_issued = ok;
    if (ok && tid == 0) {
        tc_fence_after();
        if (DELTA) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(tmem + TMV_W, sdesc_sw128(sb + X0 + kk * 2048, 16384, 1024),
                        sdesc_sw128(sb + X1 + (SCALAR ? 8192u : 0u) + kk * 32, 16, 1024), ID_WU, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            mma_f16(tmem + TMV_U, sdesc_sw128(sb + X0 + 8192 + kk * 2048, 16384, 1024),
                    sdesc_sw128(sb + X1 + kk * 32, 16, 1024), ID_WU, kk > 0);
        mma_commit(&bars[VB_WU]);
    }
    if (ok) ok = ctl.wait(VB_WU, 0);
    tc_fence_after();
    if (!__syncthreads_or(!ok)) {
        // warps 0-3: -W^T rows j (times e^(c_j)) into X1; warps 4-7: U^T rows v into X2
        if (warp >= 4 || DELTA) {
            const float sg = warp >= 4 ? 1.f : -__expf(cv[R]);
            const uint32_t dst = sb + (warp >= 4 ? X2 : X1);
            float x[64];
            ld_cols<64>(trow + (warp >= 4 ? TMV_U : TMV_W), x);
#pragma unroll
            for (int ch = 0; ch < 8; ++ch)
                st_shared_v4(dst + sw128(R, ch), pack_h2(sg * x[8 * ch], sg * x[8 * ch + 1]),
                             pack_h2(sg * x[8 * ch + 2], sg * x[8 * ch + 3]), pack_h2(sg * x[8 * ch + 4], sg * x[8 * ch + 5]),
                             pack_h2(sg * x[8 * ch + 6], sg * x[8 * ch + 7]));
        }
        fence_proxy_async();
        __syncthreads();
        if (tid == 0) {
            if (DELTA) bulk_s2g(rec + kRW * 128, sb + X1, 16384);
            bulk_s2g(rec + kRU * 128, sb + X2, 16384);
            bulk_commit();
        }
    }
    // never leave a copy or a UMMA in flight past the end of the CTA (the shared memory the
    // bulk stores read stays until they have read it)
    if (tid == 0) {
        bulk_wait_read();
        if (issued_v) ctl.drain(VB_V, 0);
        if (!allslow) ctl.drain(VB_G, 0);
        if (wu_issued) ctl.drain(VB_WU, 0);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ================================================================== chain kernel
// The state is kept transposed, S^T (TMEM lane = value column v, one column per key row j), so
// that both state-side products take their A operand from tensor memory: the fp16 copy of S^T
// for [O^T | Ut^T] += S^T [Q'^T | -W^T], and the fp16 copy of Ut^T for S^T += Ut^T Kd and
// O^T += Ut^T P^T. Only the record tiles (the B operands) are read from shared memory; at N = 128
// a UMMA with both operands in shared memory reads about as many bytes per cycle as shared
// memory delivers, so every other access there slowed the chain.
constexpr int kVCThreads = 448;   // record-load warp, an idle warp, 8 state warps (two per TMEM lane quarter),
                                  // 4 output warps
constexpr int kVCStages = 3;      // records in flight: one SM's bulk loads take about a chunk's time each
constexpr uint32_t VC_EGL = kVCStages * kRecBytes;   // exp(GL) of each stage's chunk (128 fp32 each)
constexpr uint32_t VC_XN = VC_EGL + 512 * kVCStages;  // output-normalisation scratch (384 fp32)
constexpr uint32_t VC_BAR = VC_XN + 1536;       // mbarriers, TMEM base, abort flag
constexpr uint32_t kVCSmem = VC_BAR + 256;
constexpr uint32_t kVCAlloc = kVCSmem + 1024;
static_assert(kVCAlloc <= 232448, "shared memory budget");
constexpr uint32_t TMC_S = 0;      // S^T fp32: lane = v, 128 columns j
constexpr uint32_t TMC_SH = 128;   // S^T fp16 (A operand): 64 columns of key pairs
constexpr uint32_t TMC_OU = 192;   // 2 x [O^T | -(W S)^T; its first 32 columns then Ut^T fp16]
constexpr uint32_t ID_SQW = idesc_f16(128, 128, false, true);  // [O^T | Ut^T] += S^T [Q'^T | -W^T]
constexpr uint32_t ID_SQ = idesc_f16(128, 64, false, true);    // O^T += S^T Q'^T (linear attention)
constexpr uint32_t ID_ST = idesc_f16(128, 128, false, false);  // S^T += Ut^T Kd
constexpr uint32_t ID_O = idesc_f16(128, 64, false, false);    // O^T += Ut^T P^T
constexpr int kBarS = 1;   // the 8 state warps
constexpr int kBarO = 2;   // the 4 output warps
constexpr int kBarU = 3;   // the 4 state warps of the Ut epilogue (half 1)
constexpr int kBarH = 4;   // the 4 state warps that write back the decayed half of S^T first (half 0)
// mbarriers: FULL / ODONE per record stage (chunk c takes stage c % 3; ODONE also marks its
// output tile, parity c & 1, complete); ADONE: the [O^T | Ut^T] product is done; DEC: half 0
// has written its decayed half of S^T; SDONE: the state update of the last chunk is done (the
// next chunk may read S, and every UMMA lead1 issued before it is complete); OFREE per output
// tile: the output warps have read it (the product of chunk c + 2 may write it)
enum : int { CB_FULL = 0, CB_ODONE = 3, CB_ADONE = 6, CB_DEC = 7, CB_SDONE = 8, CB_OFREE = 9, kVCBars = 11 };

template <bool DELTA, bool OPTS>
__global__ void __launch_bounds__(kVCThreads, 1)
vg_chain_kernel(const uint8_t *__restrict__ recs, const float *__restrict__ egl, const OutArgs out,
                const float *__restrict__ s0, float *__restrict__ s_final, int H, int L, int cbase, int nch,
                long long wait_limit, unsigned *__restrict__ err_word) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + VC_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kVCBars);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
    const Ctl ctl{bars, abort_flag, err_word, wait_limit};

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x;
    // this launch takes chunks cbase .. cbase + nch - 1 of the head (records bh * nch ..); rows of
    // the chunk with index c of the launch start at row0 + c * C
    const size_t row0 = static_cast<size_t>(bh) * L + static_cast<size_t>(cbase) * kC;
    const int Lrem = L - cbase * kC;                         // tokens from the launch's first chunk on
    // extents the launch implies (bounds checks of the debug build): output and state elements
    const long long n_out = static_cast<long long>(gridDim.x) * L * kD;
    const long long n_state = static_cast<long long>(gridDim.x) * kD * kD;
    const bool seq_end = cbase + nch == (L + kC - 1) / kC;   // the launch ends the sequence
    const long long rec0 = static_cast<long long>(bh) * nch;

    if (tid == 0) {
        for (int b = 0; b < kVCBars; ++b) mbar_init(&bars[b], 1);
        abort_flag[0] = 0;
        fence_mbar_init();
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
        // ================================================================ record loads
        if (lane == 0) {
            int last[kVCStages] = {-1, -1, -1};
            for (int c = 0; c < nch; ++c) {
                const int st = c % kVCStages;
                if (c >= kVCStages && !ctl.wait_lazy(CB_ODONE + st, ((c - kVCStages) / kVCStages) & 1)) break;
                uint64_t *fb = &bars[CB_FULL + st];
                mbar_arrive_expect_tx(fb, kRecBytes + kD * 4);
                const uint8_t *src = recs + static_cast<size_t>(rec0 + c) * kRecBytes;
#pragma unroll
                for (int b = 0; b < 3; ++b) bulk_g2s(sb + st * kRecBytes + b * kRecPiece, src + b * kRecPiece, kRecPiece, fb);
                bulk_g2s(sb + VC_EGL + st * 512, egl + static_cast<size_t>(rec0 + c) * kD, kD * 4, fb);
                last[st] = c;
            }
            for (int st = 0; st < kVCStages; ++st)
                if (last[st] >= 0) ctl.drain(CB_FULL + st, (last[st] / kVCStages) & 1);
        }
    } else if (warp >= 2 && warp < 10) {
        // ================================================================ state group (warps 2-9)
        // thread (v, half): TMEM lane v (value column v of S^T, O and Ut). Both halves copy
        // S^T (key columns 64 * half ..) and write back its decayed half; half 1 then takes the
        // Ut epilogue of this chunk. The output warps store the output tiles, so the chain
        // carries no output stores. The group issues the chain's UMMAs itself: thread `lead`
        // the [O^T | Ut^T] product once the fp16 copy of S^T is complete (and the output tile
        // it writes has been read), thread `lead1` the state update and the output product once
        // the fp16 copy of Ut^T is complete.
        const int half = (warp - 2) >> 2;
        const int v = (warp & 3) * 32 + lane;
        const bool lead = (v == 0 && half == 0);    // polls for the whole group and for half 0
        const bool lead1 = (v == 0 && half == 1);   // polls for half 1
        const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        {
            // S^T[v][j] = S0[j][v] for this thread's 64 key rows j (a warp reads 128 bytes per j)
            const float *src = s0 ? s0 + static_cast<size_t>(bh) * kD * kD + static_cast<size_t>(64 * half) * kD + v
                                  : nullptr;
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
                float rr[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    rr[e] = src && in_bounds((static_cast<long long>(bh) * kD + 64 * half + cc * 16 + e) * kD + v, n_state,
                                             err_word)
                                ? src[static_cast<size_t>(cc * 16 + e) * kD] : 0.f;
                tmem_st16(trow + TMC_S + 64 * half + cc * 16, rr);
            }
            tmem_wait_st();
        }
        int issued_a = -1, issued_o = -1;   // last chunk whose products lead / lead1 committed
        float nf = 0.f;
        bool stop = false;   // this half gave up waiting; the group stops at its next meeting
#pragma unroll 1
        for (int c = 0; c < nch; ++c) {
            const int s = c & 1, st = c % kVCStages;
            const uint8_t *stg = smem + st * kRecBytes;
            const uint32_t stg_a = sb + st * kRecBytes;
            // S(c) complete (state update of c-1 done), this chunk's record landed and the output
            // tile of chunk c - 2 read (this chunk's product writes it)
            {
                bool fail = stop;
                if (lead && !fail) fail = (c >= 1 && !ctl.wait(CB_SDONE, static_cast<uint32_t>(c - 1) & 1u)) ||
                                          !ctl.wait(CB_FULL + st, static_cast<uint32_t>(c / kVCStages) & 1u) ||
                                          (c >= 2 && !ctl.wait(CB_OFREE + s, static_cast<uint32_t>((c - 2) >> 1) & 1u));
                if (named_bar_any(kBarS, 256, fail)) break;
            }
            tc_fence_after();
            // ---- this thread's 64 columns of S^T -> fp16 operand (the critical path), then
            //      S^T <- S^T diag(exp(GL)) while the product runs
            float sv[64];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                float t[16];
                tmem_ld16(trow + TMC_S + 64 * half + cc * 16, t);
#pragma unroll
                for (int e = 0; e < 16; ++e) sv[16 * cc + e] = t[e];
            }
            tmem_wait_ld();
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                float hv[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) hv[e] = __uint_as_float(pack_h2(sv[32 * cc + 2 * e], sv[32 * cc + 2 * e + 1]));
                tmem_st16(trow + TMC_SH + 32 * half + 16 * cc, hv);
            }
            tmem_wait_st();
            tc_fence_before();
            named_bar(kBarS, 256);
            if (lead) {
                // [O^T | -(W S)^T] = S^T [Q'^T | -W^T] into a fresh tile (U^T is added by the Ut
                // epilogue; linear attention: O^T = S^T Q'^T, Ut = U)
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_f16_ts(tmem + TMC_OU + s * 128, tmem + TMC_SH + kk * 8,
                               sdesc_sw128(stg_a + kRQ * 128 + kk * 2048, (kRW - kRQ) * 128, 1024),
                               DELTA ? ID_SQW : ID_SQ, kk > 0 ? 1u : 0u);
                mma_commit(&bars[CB_ADONE]);
                issued_a = c;
            }
            {
                const float *eg = reinterpret_cast<const float *>(smem + VC_EGL + st * 512) + 64 * half;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    float t[16];
#pragma unroll
                    for (int e = 0; e < 16; e += 4) {
                        const float4 f = *reinterpret_cast<const float4 *>(eg + 16 * cc + e);
                        t[e] = sv[16 * cc + e] * f.x;
                        t[e + 1] = sv[16 * cc + e + 1] * f.y;
                        t[e + 2] = sv[16 * cc + e + 2] * f.z;
                        t[e + 3] = sv[16 * cc + e + 3] * f.w;
                    }
                    tmem_st16(trow + TMC_S + 64 * half + cc * 16, t);
                }
                tmem_wait_st();
            }
            if (half == 0) {
                // the decayed half of S^T is in place: hand it to the state update
                tc_fence_before();
                named_bar(kBarH, 128);
                if (lead) mbar_arrive(&bars[CB_DEC]);
            } else {
                // ---- Ut^T row v -> fp16 pairs over its first 32 columns (A operand of the
                //      state update and of the output product)
                if (!ctl.group_wait(CB_ADONE, c & 1, kBarU, lead1, 128)) {
                    stop = true;
                    continue;
                }
                tc_fence_after();
                {
                    // Ut^T = U^T - (W S)^T: U^T row v from the record (GDN); linear attention
                    // has no W, so Ut^T = U^T
                    float u[64];
                    if (DELTA) {
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) {
                            float t[16];
                            tmem_ld16(trow + TMC_OU + s * 128 + 64 + cc * 16, t);
#pragma unroll
                            for (int e = 0; e < 16; ++e) u[16 * cc + e] = t[e];
                        }
                        tmem_wait_ld();
                    } else {
#pragma unroll
                        for (int e = 0; e < 64; ++e) u[e] = 0.f;
                    }
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        const uint4 a = *reinterpret_cast<const uint4 *>(stg + sw128(kRU + v, ch));
                        u[8 * ch] += h_lo(a.x);
                        u[8 * ch + 1] += h_hi(a.x);
                        u[8 * ch + 2] += h_lo(a.y);
                        u[8 * ch + 3] += h_hi(a.y);
                        u[8 * ch + 4] += h_lo(a.z);
                        u[8 * ch + 5] += h_hi(a.z);
                        u[8 * ch + 6] += h_lo(a.w);
                        u[8 * ch + 7] += h_hi(a.w);
                    }
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        float hv[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) hv[e] = __uint_as_float(pack_h2(u[32 * cc + 2 * e], u[32 * cc + 2 * e + 1]));
                        tmem_st16(trow + TMC_OU + s * 128 + 64 + 16 * cc, hv);
                    }
                    tmem_wait_st();
                }
                tc_fence_before();
                const bool fail = lead1 && !ctl.wait(CB_DEC, static_cast<uint32_t>(c) & 1u);
                if (named_bar_any(kBarU, 128, fail)) {
                    stop = true;
                    continue;
                }
                if (lead1) {
                    // S^T += Ut^T Kd ; O^T += Ut^T P^T
                    const uint32_t uh = tmem + TMC_OU + s * 128 + 64;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16_ts(tmem + TMC_S, uh + kk * 8, sdesc_sw128(stg_a + kRKD * 128 + kk * 32, 16, 1024), ID_ST,
                                   1u);
                    mma_commit(&bars[CB_SDONE]);   // the next chunk's state copy need not wait for O
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16_ts(tmem + TMC_OU + s * 128, uh + kk * 8, sdesc_sw128(stg_a + kRP * 128 + kk * 32, 16, 1024),
                                   ID_O, 1u);
                    mma_commit(&bars[CB_ODONE + st]);
                    issued_o = c;
                }
            }
        }
        // UMMAs complete in issue order: each issuing thread waits for its last commit
        if (lead && issued_a >= 0) ctl.drain(CB_ADONE, static_cast<uint32_t>(issued_a) & 1u);
        if (lead1 && issued_o >= 0) ctl.drain(CB_ODONE + issued_o % kVCStages, (issued_o / kVCStages) & 1);
        // ---- the final state (both halves)
        const int cp = nch - 1;
        {
            // the final state once the last update is done, unless the group stopped
            bool fail = stop;
            if (lead && !fail && nch > 0) fail = !ctl.wait(CB_SDONE, static_cast<uint32_t>(cp) & 1u);
            if (!named_bar_any(kBarS, 256, fail || !s_final || nch == 0)) {
                tc_fence_after();
                float *dst = s_final + static_cast<size_t>(bh) * kD * kD + static_cast<size_t>(64 * half) * kD + v;
#pragma unroll 1
                for (int cc = 0; cc < 4; ++cc) {
                    float t[16];
                    tmem_ld16(trow + TMC_S + 64 * half + cc * 16, t);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        probe_finite(nf, t[e]);
                        if (in_bounds((static_cast<long long>(bh) * kD + 64 * half + cc * 16 + e) * kD + v, n_state, err_word))
                            dst[static_cast<size_t>(cc * 16 + e) * kD] = t[e];
                    }
                }
            }
        }
        report_nonfinite(ctl.aborted() ? 0.f : nf, err_word);
    } else if (warp >= 10) {
        // ================================================================ output warps (10-13)
        // thread v: TMEM lane v. Each chunk's output tile, once complete, is read, handed back
        // (OFREE) and stored; the last tile holds the sequence's ragged tail.
        const int v = (warp & 3) * 32 + lane;
        const bool olead = v == 0;
        const int head = bh % H;
        float *xn = reinterpret_cast<float *>(smem + VC_XN);
        const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        float nf = 0.f;
#pragma unroll 1
        for (int c = 0; c < nch; ++c) {
            if (!ctl.group_wait(CB_ODONE + c % kVCStages, (c / kVCStages) & 1, kBarO, olead, 128)) break;
            tc_fence_after();
            float ov[64];
            ld_cols<64>(trow + TMC_OU + (c & 1) * 128, ov);
            tc_fence_before();
            named_bar(kBarO, 128);
            if (olead) mbar_arrive(&bars[CB_OFREE + (c & 1)]);
            const bool last = c == nch - 1;
            const int n = last ? min(kC, Lrem - c * kC) : kC;
            const size_t elem0 = (row0 + static_cast<size_t>(c) * kC) * kD + v;
            if constexpr (OPTS) {
                store_out_rows_group(ov, out, elem0, n, head, v, kBarO, xn, xn + 256, last && seq_end, nf);
            } else {
                float *ocol = static_cast<float *>(out.o) + elem0;
#pragma unroll
                for (int r = 0; r < 64; ++r)
                    if (r < n && in_bounds(static_cast<long long>(elem0) + static_cast<long long>(r) * kD, n_out, err_word))
                        ocol[static_cast<size_t>(r) * kD] = ov[r];
                if (last && seq_end) probe_tile(nf, ov, n);
            }
        }
        report_nonfinite(ctl.aborted() ? 0.f : nf, err_word);
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

namespace {

// One stream-ordered memory pool per device for the per-chunk records; it keeps what it
// has reserved (release threshold: never), so repeated calls of one size allocate once.
cudaMemPool_t record_pool(int dev) {
    static std::mutex mu;
    static cudaMemPool_t pools[64] = {};
    if (dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!pools[dev]) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t p = nullptr;
        if (cudaMemPoolCreate(&p, &props) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        cuuint64_t keep = ~0ull;
        cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &keep);
        pools[dev] = p;
    }
    return pools[dev];
}

template <bool DELTA, bool SCALAR>
bool launch_prep(const CUtensorMap &mv, const void *q, const void *k, const void *v, const float *beta,
                 const float *g, uint8_t *recs, float *egl, int BH, int L, int cbase, int nseg, float scale,
                 cudaStream_t stream) {
    auto kp = vg_prep_kernel<DELTA, SCALAR>;
    if (!ensure_smem_limit(reinterpret_cast<const void *>(kp), kVPAlloc)) return false;
    unsigned *err = device_error_word();
    if (!err) return false;
    kp<<<static_cast<unsigned>(static_cast<long long>(BH) * nseg), kVPThreads, kVPAlloc, stream>>>(
        mv, static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k), beta, g, recs, egl, L,
        cbase, nseg, scale, wait_limit_cycles(), err);
    return cudaGetLastError() == cudaSuccess;
}

template <bool DELTA, bool OPTS>
bool launch_chain(const uint8_t *recs, const float *egl, const OutArgs &out, const float *s0, float *s_final, int BH,
                  int H, int L, int cbase, int nseg, cudaStream_t stream) {
    auto kc = vg_chain_kernel<DELTA, OPTS>;
    if (!ensure_smem_limit(reinterpret_cast<const void *>(kc), kVCAlloc)) return false;
    unsigned *err = device_error_word();
    if (!err) return false;
    kc<<<BH, kVCThreads, kVCAlloc, stream>>>(recs, egl, out, s0, s_final, H, L, cbase, nseg, wait_limit_cycles(),
                                             err);
    return cudaGetLastError() == cudaSuccess;
}

bool prep_any(bool delta, bool scalar, const CUtensorMap &mv, const void *q, const void *k, const void *v,
              const float *beta, const float *g, uint8_t *recs, float *egl, int BH, int L, int cbase, int nseg,
              float scale, cudaStream_t stream) {
    if (delta)
        return scalar ? launch_prep<true, true>(mv, q, k, v, beta, g, recs, egl, BH, L, cbase, nseg, scale, stream)
                      : launch_prep<true, false>(mv, q, k, v, beta, g, recs, egl, BH, L, cbase, nseg, scale, stream);
    return scalar ? launch_prep<false, true>(mv, q, k, v, beta, g, recs, egl, BH, L, cbase, nseg, scale, stream)
                  : launch_prep<false, false>(mv, q, k, v, beta, g, recs, egl, BH, L, cbase, nseg, scale, stream);
}

bool chain_any(bool delta, bool opts, const uint8_t *recs, const float *egl, const OutArgs &out, const float *s0,
               float *s_final, int BH, int H, int L, int cbase, int nseg, cudaStream_t stream) {
    if (delta)
        return opts ? launch_chain<true, true>(recs, egl, out, s0, s_final, BH, H, L, cbase, nseg, stream)
                    : launch_chain<true, false>(recs, egl, out, s0, s_final, BH, H, L, cbase, nseg, stream);
    return opts ? launch_chain<false, true>(recs, egl, out, s0, s_final, BH, H, L, cbase, nseg, stream)
                : launch_chain<false, false>(recs, egl, out, s0, s_final, BH, H, L, cbase, nseg, stream);
}

// Two streams per device (created once) for a long sequence cut into segments: the prep
// kernels on one with the lowest priority, the chain kernels on one with the highest, so that
// as the prep CTAs of segment i + 1 retire, the SMs they free go to the chain of segment i.
struct SegStreams {
    cudaStream_t prep = nullptr, chain = nullptr;
};
SegStreams seg_streams(int dev) {
    static std::mutex mu;
    static SegStreams streams[64];
    if (dev < 0 || dev >= 64) return SegStreams{};
    std::lock_guard<std::mutex> lock(mu);
    SegStreams &s = streams[dev];
    if (!s.prep || !s.chain) {
        int least = 0, greatest = 0;
        if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess ||
            (!s.prep && cudaStreamCreateWithPriority(&s.prep, cudaStreamNonBlocking, least) != cudaSuccess) ||
            (!s.chain && cudaStreamCreateWithPriority(&s.chain, cudaStreamNonBlocking, greatest) != cudaSuccess)) {
            cudaGetLastError();
            return SegStreams{};
        }
    }
    return s;
}

constexpr int kSegChunks = 64;   // chunks of each head per segment when a call is split

// Few heads with long sequences: the chain kernel runs on as many SMs as there are heads,
// so the sequence is cut into segments and the prep of segment i + 1 runs on the other SMs
// while the chain takes segment i.
bool split_in_segments(int BH, int nch) {
    const int sms = sm_count();
    return sms > 0 && 3LL * BH <= sms && nch >= 2 * kSegChunks;
}

}  // namespace

size_t tc_vg_workspace_bytes(int B, int H, int L) {
    const long long nch = (static_cast<long long>(L) + kC - 1) / kC;
    const long long BH = static_cast<long long>(B) * H;
    const size_t per_chunk = kRecBytes + kD * sizeof(float);
    if (split_in_segments(static_cast<int>(BH), static_cast<int>(nch)))
        return 2 * static_cast<size_t>(BH) * kSegChunks * per_chunk + static_cast<size_t>(BH) * kD * kD * sizeof(float);
    return static_cast<size_t>(BH) * nch * per_chunk;
}

bool tc_vg_takes_scalar(int B, int H, int L) {
    return split_in_segments(B * H, (L + kC - 1) / kC);
}

gdn_status_t launch_tc_vg(bool delta, bool per_key, const void *q, const void *k, const void *v, const float *beta,
                          const float *g, void *o, const float *s0, float *s_final, int B, int H, int L, float scale,
                          FwdOpts oo, cudaStream_t stream, bool *fallback) {
    *fallback = false;
    const int BH = B * H;
    const int nch = (L + kC - 1) / kC;
    const bool split = split_in_segments(BH, nch);
    const int seg = split ? kSegChunks : nch;
    const long long nrec = static_cast<long long>(BH) * seg;   // records of one segment
    if (nrec > 2147483647LL || (per_key && reinterpret_cast<uintptr_t>(g) % 8 != 0)) {
        // one prep CTA per record; the vector-gate prep reads g two floats at a time
        *fallback = true;
        return GDN_ERR_UNSUPPORTED;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_CUDA;
    cudaMemPool_t pool = record_pool(dev);
    const SegStreams ss = split ? seg_streams(dev) : SegStreams{};
    void *ws = nullptr;
    if (!pool || (split && (!ss.prep || !ss.chain)) ||
        cudaMallocFromPoolAsync(&ws, tc_vg_workspace_bytes(B, H, L), pool, stream) != cudaSuccess) {
        cudaGetLastError();
        *fallback = true;   // the caller takes the kernel that needs no workspace
        return GDN_ERR_CUDA;
    }
    const size_t slot_bytes = static_cast<size_t>(nrec) * (kRecBytes + kD * sizeof(float));
    auto recs_of = [&](int slot) { return static_cast<uint8_t *>(ws) + slot * slot_bytes; };
    auto egl_of = [&](int slot) { return reinterpret_cast<float *>(recs_of(slot) + static_cast<size_t>(nrec) * kRecBytes); };
    CUtensorMap mv;
    const OutArgs out = make_out_args(o, v, oo);
    const bool opts = oo.bf16 || oo.dskip != nullptr || oo.xnorm != kXNormNone;
    const bool scalar = !per_key;
    bool ok = make_qkv_map(&mv, v, L, BH);
    if (ok && !split) {
        ok = prep_any(delta, scalar, mv, q, k, v, beta, g, recs_of(0), egl_of(0), BH, L, 0, nch, scale, stream) &&
             chain_any(delta, opts, recs_of(0), egl_of(0), out, s0, s_final, BH, H, L, 0, nch, stream);
    } else if (ok) {
        // segments of kSegChunks chunks; records in two slots; the state between segments in a
        // (BH, dk, dv) buffer after the slots
        float *state = reinterpret_cast<float *>(recs_of(2));
        const int nsegs = (nch + seg - 1) / seg;
        std::vector<cudaEvent_t> evs;
        auto event = [&]() -> cudaEvent_t {
            cudaEvent_t e = nullptr;
            if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return nullptr;
            evs.push_back(e);
            return e;
        };
        cudaEvent_t start = event();
        ok = start && cudaEventRecord(start, stream) == cudaSuccess && cudaStreamWaitEvent(ss.prep, start, 0) == cudaSuccess &&
             cudaStreamWaitEvent(ss.chain, start, 0) == cudaSuccess;
        std::vector<cudaEvent_t> chain_done(nsegs, nullptr);
        for (int i = 0; ok && i < nsegs; ++i) {
            const int cb = i * seg, n = std::min(seg, nch - cb), sl = i & 1;
            if (i >= 2) ok = cudaStreamWaitEvent(ss.prep, chain_done[i - 2], 0) == cudaSuccess;   // slot reuse
            cudaEvent_t prepped = ok ? event() : nullptr;
            ok = ok && prepped &&
                 prep_any(delta, scalar, mv, q, k, v, beta, g, recs_of(sl), egl_of(sl), BH, L, cb, n, scale, ss.prep) &&
                 cudaEventRecord(prepped, ss.prep) == cudaSuccess && cudaStreamWaitEvent(ss.chain, prepped, 0) == cudaSuccess;
            chain_done[i] = ok ? event() : nullptr;
            ok = ok && chain_done[i] &&
                 chain_any(delta, opts, recs_of(sl), egl_of(sl), out, i == 0 ? s0 : state,
                           i == nsegs - 1 ? s_final : state, BH, H, L, cb, n, ss.chain) &&
                 cudaEventRecord(chain_done[i], ss.chain) == cudaSuccess;
        }
        // the caller's stream continues once the last chain kernel is done (it follows every
        // kernel of the call)
        ok = ok && cudaStreamWaitEvent(stream, chain_done[nsegs - 1], 0) == cudaSuccess;
        if (!ok) {
            // leave nothing of this call running behind the caller's back
            cudaStreamSynchronize(ss.prep);
            cudaStreamSynchronize(ss.chain);
        }
        for (cudaEvent_t e : evs) cudaEventDestroy(e);   // released once their work is done
    }
    // stream-ordered: the workspace is released once every kernel of the call has run (the side
    // stream's work all precedes events the caller's stream waited for)
    const bool freed = cudaFreeAsync(ws, stream) == cudaSuccess;
    return ok && freed ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace gdn
