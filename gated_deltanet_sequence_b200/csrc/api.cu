// C-ABI entry points of libgdn.so: argument validation and kernel dispatch.
// Every launch goes on the caller's stream. Only the vector-gate tensor-core form (tc_vg.cu) takes
// memory: a stream-ordered workspace from a pool the library owns.
#include <math.h>

#include "common.cuh"
#include "tc_kernels.cuh"

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool opt_aligned16(const void *p) { return p == nullptr || aligned16(p); }
bool opt_aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool head_dim_ok(int d) { return d == 64 || d == 128; }
// token rows of a call (the padded copies index them with an int)
bool rows_fit_int(const int *cu, int B, int H, int L) { return (double)(cu ? 1 : B) * H * L < 1073741824.0; }
constexpr gdn::FwdOpts kDefaultOut{false, nullptr, false, gdn::kXNormNone, nullptr, 0.f};   // fp32 o, no options

// The output-normalisation fields of the options: a known kind, a positive finite eps
// when one is set, a 4-byte aligned weight.
bool set_xnorm(const gdn_fwd_opts_t &opts, gdn::FwdOpts *oo) {
    if (opts.xnorm != GDN_XNORM_NONE && opts.xnorm != GDN_XNORM_RMS && opts.xnorm != GDN_XNORM_LAYER) return false;
    if (opts.xnorm != GDN_XNORM_NONE && !(isfinite(opts.xnorm_eps) && opts.xnorm_eps > 0.f)) return false;
    if (!opt_aligned4(opts.xnorm_weight)) return false;
    oo->xnorm = opts.xnorm == GDN_XNORM_RMS ? gdn::kXNormRms : opts.xnorm == GDN_XNORM_LAYER ? gdn::kXNormLayer
                                                                                          : gdn::kXNormNone;
    oo->xw = opts.xnorm_weight;
    oo->xeps = opts.xnorm_eps;
    return true;
}

gdn_status_t check_prefill(const void *q, const void *k, const void *v, const float *g, float *o,
                           const float *s0, float *s_final, int B, int H, int L, int dk, int dv,
                           int chunk, float scale, gdn_dtype_t in_dtype) {
    if (B < 1 || H < 1 || L < 0 || !isfinite(scale)) return GDN_ERR_INVALID_ARG;
    if (in_dtype != GDN_F32 && in_dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (L > 0 && (!q || !k || !v || !o)) return GDN_ERR_INVALID_ARG;
    if (!opt_aligned16(q) || !opt_aligned16(k) || !opt_aligned16(v) || !opt_aligned16(o) ||
        !opt_aligned4(g) || !opt_aligned16(s0) || !opt_aligned16(s_final))
        return GDN_ERR_INVALID_ARG;
    if (chunk < 1) return GDN_ERR_INVALID_ARG;
    if (!head_dim_ok(dk) || !head_dim_ok(dv) || chunk > 64) return GDN_ERR_UNSUPPORTED;
    // every element offset must fit the kernels' 64-bit index arithmetic and the
    // per-head length must fit a 32-bit token index
    const double elems = (double)B * H * (double)L * (dk > dv ? dk : dv);
    if (elems > 9.0e18 || (double)B * H > 2147483647.0) return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

}  // namespace

namespace gdn {
// The per-chunk prep kernel and the per-head chain kernel (tc_vg.cu), dense bf16 batches at
// dk = dv = 128, C = 64, with a stream-ordered workspace: vector-valued gates (per_key), and
// scalar gates for few heads with long sequences (tc_vg_takes_scalar), whose sequences are then
// cut into segments whose prep overlaps the chain of the segment before. *fallback is set when
// the call cannot run there (no workspace, or too many chunks); nothing has been launched then.
gdn_status_t launch_tc_vg(bool delta, bool per_key, const void *q, const void *k, const void *v, const float *beta,
                          const float *g, void *o, const float *s0, float *s_final, int B, int H, int L, float scale,
                          FwdOpts oo, cudaStream_t stream, bool *fallback);
bool tc_vg_takes_scalar(int B, int H, int L);
// Zero-padded copies for head sizes of 64 (pad.cu): dst[o][r][c] from src with zero fill (or a
// crop when the source is the larger), rows given in bytes; and the copies' workspace.
bool pad_copy(void *dst, const void *src, long long n_outer, int rows_dst, int cols_dst_bytes, int rows_src,
              int cols_src_bytes, cudaStream_t stream);
bool pad_alloc(void **p, size_t bytes, cudaStream_t stream);
// Head sizes of 64 on the one-CTA Gated DeltaNet kernel without copies (tc_gdn.cu): whether the
// kernel takes nctas (sequence, head) pairs, and the launch (plain fp32 output, scalar gate).
bool tc_gdn_takes_narrow(int nctas);
gdn_status_t launch_tc_gdn_narrow(const void *q, const void *k, const void *v, const float *beta, const float *g,
                                  float *o, const float *s0, float *s_final, const int *cu, int B, int H, int L,
                                  int dk, int dv, float scale, cudaStream_t stream);
// The same for linear attention on its kernel (tc_la.cu), which takes every batch.
gdn_status_t launch_tc_la_narrow(const void *q, const void *k, const void *v, const float *g, float *o,
                                 const float *s0, float *s_final, const int *cu, int B, int H, int L, int dk, int dv,
                                 float scale, cudaStream_t stream);
}  // namespace gdn

extern "C" {

static gdn_status_t prefill_ex(bool delta, const void *q, const void *k, const void *v, const float *beta,
                               const float *g, void *o, const float *s0, float *s_final, const int *cu_seqlens,
                               int B, int H, int L, int dk, int dv, int chunk, float scale, gdn_dtype_t in_dtype,
                               const gdn_fwd_opts_t *opts, void *cuda_stream);

// bf16 calls at chunk 64 with dk or dv = 64 run on the tensor-core kernels through copies padded
// to 128 (pad.cu); not with the output normalisation, which reduces over the value width
static bool pad_applies(gdn_dtype_t in_dtype, int dk, int dv, int chunk, int L) {
    return in_dtype == GDN_BF16 && chunk == 64 && L > 0 && (dk != 128 || dv != 128);
}

// The padded call: q, k (dk -> 128), v (dv -> 128), a vector gate (dk -> 128, log-decay 0), the
// skip weights (dv -> 128) and S0 (dk x dv -> 128 x 128) are copied with zero fill into a
// stream-ordered workspace, the call runs at 128 x 128, and o and S_final are cropped back.
// Rows of the padded state and output beyond dk / dv stay zero (zero keys and values), so the
// first dk x dv entries are the results of the unpadded call. *fallback: no workspace.
static gdn_status_t padded_prefill(bool delta, const void *q, const void *k, const void *v, const float *beta,
                                   const float *g, void *o, const float *s0, float *s_final, const int *cu_seqlens,
                                   int B, int H, int L, int dk, int dv, float scale, const gdn::FwdOpts &oo,
                                   cudaStream_t stream, bool *fallback) {
    *fallback = false;
    const long long rows = static_cast<long long>(cu_seqlens ? 1 : B) * H * L;   // token rows
    const long long nstate = static_cast<long long>(B) * H;
    const int ob = oo.bf16 ? 2 : 4;
    const bool vec = oo.gate_per_key;
    auto up = [](long long x) { return static_cast<size_t>((x + 255) / 256 * 256); };
    size_t off = 0;
    const size_t o_q = off; off += up(rows * 256);
    const size_t o_k = off; off += up(rows * 256);
    const size_t o_v = off; off += up(rows * 256);
    const size_t o_o = off; off += up(rows * 128 * ob);
    const size_t o_g = off; if (vec) off += up(rows * 512);
    const size_t o_s0 = off; if (s0) off += up(nstate * 65536);
    const size_t o_sf = off; if (s_final) off += up(nstate * 65536);
    const size_t o_d = off; if (oo.dskip) off += up(static_cast<long long>(H) * 512);
    void *ws = nullptr;
    if (!gdn::pad_alloc(&ws, off, stream)) {
        *fallback = true;
        return GDN_ERR_CUDA;
    }
    uint8_t *w = static_cast<uint8_t *>(ws);
    bool ok = gdn::pad_copy(w + o_q, q, 1, static_cast<int>(rows), 256, static_cast<int>(rows), dk * 2, stream) &&
              gdn::pad_copy(w + o_k, k, 1, static_cast<int>(rows), 256, static_cast<int>(rows), dk * 2, stream) &&
              gdn::pad_copy(w + o_v, v, 1, static_cast<int>(rows), 256, static_cast<int>(rows), dv * 2, stream);
    if (vec) ok = ok && gdn::pad_copy(w + o_g, g, 1, static_cast<int>(rows), 512, static_cast<int>(rows), dk * 4, stream);
    if (s0) ok = ok && gdn::pad_copy(w + o_s0, s0, nstate, 128, 512, dk, dv * 4, stream);
    if (oo.dskip) ok = ok && gdn::pad_copy(w + o_d, oo.dskip, 1, H, 512, H, dv * 4, stream);
    gdn_status_t st = GDN_ERR_CUDA;
    if (ok) {
        gdn_fwd_opts_t po = {};
        po.out_dtype = oo.bf16 ? GDN_BF16 : GDN_F32;
        po.d_skip = oo.dskip ? reinterpret_cast<const float *>(w + o_d) : nullptr;
        po.g_per_key = vec ? 1 : 0;
        po.xnorm = GDN_XNORM_NONE;
        st = prefill_ex(delta, w + o_q, w + o_k, w + o_v, beta, vec ? reinterpret_cast<const float *>(w + o_g) : g,
                        w + o_o, s0 ? reinterpret_cast<const float *>(w + o_s0) : nullptr,
                        s_final ? reinterpret_cast<float *>(w + o_sf) : nullptr, cu_seqlens, B, H, L, 128, 128, 64,
                        scale, GDN_BF16, &po, stream);
        if (st == GDN_OK) {
            ok = gdn::pad_copy(o, w + o_o, 1, static_cast<int>(rows), dv * ob, static_cast<int>(rows), 128 * ob, stream);
            if (s_final) ok = ok && gdn::pad_copy(s_final, w + o_sf, nstate, dk, dv * 4, 128, 512, stream);
            if (!ok) st = GDN_ERR_CUDA;
        }
    }
    if (cudaFreeAsync(ws, stream) != cudaSuccess && st == GDN_OK) st = GDN_ERR_CUDA;
    return st;
}

const char *gdn_status_str(gdn_status_t s) {
    switch (s) {
        case GDN_OK: return "GDN_OK";
        case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
        case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
        case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
        case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
        case GDN_ERR_NONFINITE: return "GDN_ERR_NONFINITE";
        case GDN_ERR_BOUNDS: return "GDN_ERR_BOUNDS";
    }
    return "GDN_ERR_UNKNOWN";
}

int gdn_version(void) { return 102; }

gdn_status_t lin_attn_chunk_fwd(const void *q, const void *k, const void *v, const float *g,
                                float *o, const float *s0, float *s_final, int B, int H, int L,
                                int dk, int dv, int chunk, float scale, gdn_dtype_t in_dtype,
                                void *cuda_stream) {
    gdn_status_t st = check_prefill(q, k, v, g, o, s0, s_final, B, H, L, dk, dv, chunk, scale, in_dtype);
    if (st != GDN_OK) return st;
    if (pad_applies(in_dtype, dk, dv, chunk, L))
        return prefill_ex(false, q, k, v, nullptr, g, o, s0, s_final, nullptr, B, H, L, dk, dv, chunk, scale, in_dtype,
                          nullptr, cuda_stream);
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    if (gdn::tc_supported(in_dtype, dk, dv, chunk) && L > 0)
        return gdn::launch_tc_la(q, k, v, g, o, s0, s_final, nullptr, B, H, L, scale, kDefaultOut, stream);
    return gdn::launch_simt_fwd(q, k, v, nullptr, g, o, s0, s_final, nullptr, B, H, L, dk, dv, chunk,
                                scale, in_dtype, kDefaultOut, stream);
}

gdn_status_t gdn_chunk_fwd(const void *q, const void *k, const void *v, const float *beta,
                           const float *g, float *o, const float *s0, float *s_final, int B, int H,
                           int L, int dk, int dv, int chunk, float scale, gdn_dtype_t in_dtype,
                           void *cuda_stream) {
    gdn_status_t st = check_prefill(q, k, v, g, o, s0, s_final, B, H, L, dk, dv, chunk, scale, in_dtype);
    if (st != GDN_OK) return st;
    if (L > 0 && !beta) return GDN_ERR_INVALID_ARG;
    if (!opt_aligned4(beta)) return GDN_ERR_INVALID_ARG;
    if (pad_applies(in_dtype, dk, dv, chunk, L))
        return prefill_ex(true, q, k, v, beta, g, o, s0, s_final, nullptr, B, H, L, dk, dv, chunk, scale, in_dtype,
                          nullptr, cuda_stream);
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    if (gdn::tc_supported(in_dtype, dk, dv, chunk) && L > 0 && gdn::tc_vg_takes_scalar(B, H, L)) {
        // few heads, long sequences: prep on every SM, overlapped with the per-head chain
        bool fallback = false;
        const gdn_status_t vs = gdn::launch_tc_vg(true, false, q, k, v, beta, g, o, s0, s_final, B, H, L, scale,
                                                  kDefaultOut, stream, &fallback);
        if (!fallback) return vs;
    }
    if (gdn::tc_supported(in_dtype, dk, dv, chunk) && L > 0)
        return gdn::launch_tc_gdn(q, k, v, beta, g, o, s0, s_final, nullptr, B, H, L, scale, kDefaultOut, stream);
    // with L == 0 beta may be NULL: the kernel then only writes s0 (or zeros) to s_final
    return gdn::launch_simt_fwd(q, k, v, beta, g, o, s0, s_final, nullptr, B, H, L, dk, dv, chunk,
                                scale, in_dtype, kDefaultOut, stream);
}

gdn_status_t lin_attn_chunk_fwd_varlen(const void *q, const void *k, const void *v, const float *g,
                                       float *o, const float *s0, float *s_final,
                                       const int *cu_seqlens, int N, int H, int T, int dk, int dv,
                                       int chunk, float scale, gdn_dtype_t in_dtype,
                                       void *cuda_stream) {
    if (N < 1 || !cu_seqlens || !opt_aligned4(cu_seqlens)) return GDN_ERR_INVALID_ARG;
    gdn_status_t st = check_prefill(q, k, v, g, o, s0, s_final, 1, H, T, dk, dv, chunk, scale, in_dtype);
    if (st != GDN_OK) return st;
    if ((double)N * H > 2147483647.0) return GDN_ERR_INVALID_ARG;
    if (pad_applies(in_dtype, dk, dv, chunk, T))
        return prefill_ex(false, q, k, v, nullptr, g, o, s0, s_final, cu_seqlens, N, H, T, dk, dv, chunk, scale,
                          in_dtype, nullptr, cuda_stream);
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    if (gdn::tc_supported(in_dtype, dk, dv, chunk) && T > 0)
        return gdn::launch_tc_la(q, k, v, g, o, s0, s_final, cu_seqlens, N, H, T, scale, kDefaultOut, stream);
    return gdn::launch_simt_fwd(q, k, v, nullptr, g, o, s0, s_final, cu_seqlens, N, H, T, dk, dv, chunk,
                                scale, in_dtype, kDefaultOut, stream);
}

gdn_status_t gdn_chunk_fwd_varlen(const void *q, const void *k, const void *v, const float *beta,
                                  const float *g, float *o, const float *s0, float *s_final,
                                  const int *cu_seqlens, int N, int H, int T, int dk, int dv, int chunk,
                                  float scale, gdn_dtype_t in_dtype, void *cuda_stream) {
    if (N < 1 || !cu_seqlens || !opt_aligned4(cu_seqlens)) return GDN_ERR_INVALID_ARG;
    gdn_status_t st = check_prefill(q, k, v, g, o, s0, s_final, 1, H, T, dk, dv, chunk, scale, in_dtype);
    if (st != GDN_OK) return st;
    if ((double)N * H > 2147483647.0) return GDN_ERR_INVALID_ARG;
    if (T > 0 && !beta) return GDN_ERR_INVALID_ARG;
    if (!opt_aligned4(beta)) return GDN_ERR_INVALID_ARG;
    if (pad_applies(in_dtype, dk, dv, chunk, T))
        return prefill_ex(true, q, k, v, beta, g, o, s0, s_final, cu_seqlens, N, H, T, dk, dv, chunk, scale,
                          in_dtype, nullptr, cuda_stream);
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    if (gdn::tc_supported(in_dtype, dk, dv, chunk) && T > 0)
        return gdn::launch_tc_gdn(q, k, v, beta, g, o, s0, s_final, cu_seqlens, N, H, T, scale, kDefaultOut, stream);
    return gdn::launch_simt_fwd(q, k, v, beta, g, o, s0, s_final, cu_seqlens, N, H, T, dk, dv, chunk,
                                scale, in_dtype, kDefaultOut, stream);
}

// The general prefill call: dense (cu_seqlens == NULL) or packed batches, with the output
// options. Validation as for the dense / packed calls, plus the options.
static gdn_status_t prefill_ex(bool delta, const void *q, const void *k, const void *v, const float *beta,
                               const float *g, void *o, const float *s0, float *s_final, const int *cu_seqlens,
                               int B, int H, int L, int dk, int dv, int chunk, float scale, gdn_dtype_t in_dtype,
                               const gdn_fwd_opts_t *opts, void *cuda_stream) {
    gdn::FwdOpts oo = kDefaultOut;
    if (opts) {
        if (opts->out_dtype != GDN_F32 && opts->out_dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
        if (!opt_aligned4(opts->d_skip)) return GDN_ERR_INVALID_ARG;
        if (opts->g_per_key != 0 && opts->g_per_key != 1) return GDN_ERR_INVALID_ARG;
        if (!set_xnorm(*opts, &oo)) return GDN_ERR_INVALID_ARG;
        oo.bf16 = opts->out_dtype == GDN_BF16;
        oo.dskip = opts->d_skip;
        oo.gate_per_key = opts->g_per_key == 1 && g != nullptr;
    }
    if (B < 1 || !opt_aligned4(cu_seqlens)) return GDN_ERR_INVALID_ARG;
    const int grid_b = cu_seqlens ? 1 : B;   // batch extent of the token grid
    gdn_status_t st = check_prefill(q, k, v, g, static_cast<float *>(o), s0, s_final, grid_b, H, L, dk, dv, chunk,
                                    scale, in_dtype);
    if (st != GDN_OK) return st;
    if ((double)B * H > 2147483647.0) return GDN_ERR_INVALID_ARG;
    if (delta && L > 0 && !beta) return GDN_ERR_INVALID_ARG;
    if (!opt_aligned4(beta)) return GDN_ERR_INVALID_ARG;
    if ((double)B * H * (double)L * dk > 9.0e18) return GDN_ERR_INVALID_ARG;   // g of (rows, dk)
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    // Head size 64 with the plain fp32 output and a scalar gate, for linear attention and for
    // Gated DeltaNet on batches its one-CTA tensor-core kernel takes: the kernel reads the
    // 64-wide tiles directly (their halves past dk or dv load as zeros) and writes only dk x dv
    // states and dv output columns, which gives the results of the zero-padded call below
    // without its copies
    const bool narrow = pad_applies(in_dtype, dk, dv, chunk, L) && (dk == 64 || dk == 128) &&
                        (dv == 64 || dv == 128) && !oo.bf16 && !oo.dskip && oo.xnorm == gdn::kXNormNone &&
                        !oo.gate_per_key && aligned16(q) && aligned16(k) && aligned16(v);
    if (narrow && !delta)
        return gdn::launch_tc_la_narrow(q, k, v, g, static_cast<float *>(o), s0, s_final, cu_seqlens, B, H, L, dk, dv,
                                        scale, stream);
    if (narrow && gdn::tc_gdn_takes_narrow(B * H) && (cu_seqlens || !gdn::tc_vg_takes_scalar(B, H, L)))
        return gdn::launch_tc_gdn_narrow(q, k, v, beta, g, static_cast<float *>(o), s0, s_final, cu_seqlens, B, H, L,
                                         dk, dv, scale, stream);
    if (pad_applies(in_dtype, dk, dv, chunk, L) && oo.xnorm == gdn::kXNormNone && rows_fit_int(cu_seqlens, B, H, L)) {
        bool fallback = false;
        const gdn_status_t ps = padded_prefill(delta, q, k, v, beta, g, o, s0, s_final, cu_seqlens, B, H, L, dk, dv,
                                               scale, oo, stream, &fallback);
        if (!fallback) return ps;
    }
    // vector-valued gates: the two tensor-core kernels for dense bf16 batches at dk = dv = 128,
    // C = 64; the fp32 chunk kernel for every other input dtype, size and layout
    if (gdn::tc_supported(in_dtype, dk, dv, chunk) && L > 0 && oo.gate_per_key && !cu_seqlens) {
        bool fallback = false;
        const gdn_status_t vs = gdn::launch_tc_vg(delta, true, q, k, v, beta, g, o, s0, s_final, B, H, L, scale, oo,
                                                  stream, &fallback);
        if (!fallback) return vs;
    }
    if (delta && gdn::tc_supported(in_dtype, dk, dv, chunk) && L > 0 && !cu_seqlens && gdn::tc_vg_takes_scalar(B, H, L)) {
        bool fallback = false;
        const gdn_status_t vs = gdn::launch_tc_vg(true, false, q, k, v, beta, g, o, s0, s_final, B, H, L, scale, oo,
                                                  stream, &fallback);
        if (!fallback) return vs;
    }
    if (gdn::tc_supported(in_dtype, dk, dv, chunk) && L > 0 && !oo.gate_per_key)
        return delta ? gdn::launch_tc_gdn(q, k, v, beta, g, o, s0, s_final, cu_seqlens, B, H, L, scale, oo, stream)
                     : gdn::launch_tc_la(q, k, v, g, o, s0, s_final, cu_seqlens, B, H, L, scale, oo, stream);
    return gdn::launch_simt_fwd(q, k, v, delta ? beta : nullptr, g, o, s0, s_final, cu_seqlens, B, H, L, dk, dv,
                                chunk, scale, in_dtype, oo, stream);
}

gdn_status_t lin_attn_chunk_fwd_ex(const void *q, const void *k, const void *v, const float *g, void *o,
                                   const float *s0, float *s_final, const int *cu_seqlens, int B, int H, int L,
                                   int dk, int dv, int chunk, float scale, gdn_dtype_t in_dtype,
                                   const gdn_fwd_opts_t *opts, void *cuda_stream) {
    return prefill_ex(false, q, k, v, nullptr, g, o, s0, s_final, cu_seqlens, B, H, L, dk, dv, chunk, scale,
                      in_dtype, opts, cuda_stream);
}

gdn_status_t gdn_chunk_fwd_ex(const void *q, const void *k, const void *v, const float *beta, const float *g,
                              void *o, const float *s0, float *s_final, const int *cu_seqlens, int B, int H, int L,
                              int dk, int dv, int chunk, float scale, gdn_dtype_t in_dtype,
                              const gdn_fwd_opts_t *opts, void *cuda_stream) {
    return prefill_ex(true, q, k, v, beta, g, o, s0, s_final, cu_seqlens, B, H, L, dk, dv, chunk, scale, in_dtype,
                      opts, cuda_stream);
}

static gdn_status_t decode_impl(const void *q, const void *k, const void *v, const float *beta,
                                const float *g, float *state, void *o, int N, int H, int dk, int dv,
                                float scale, gdn_dtype_t in_dtype, const gdn_fwd_opts_t *opts,
                                void *cuda_stream) {
    if (N < 1 || H < 1 || !isfinite(scale)) return GDN_ERR_INVALID_ARG;
    if (in_dtype != GDN_F32 && in_dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (!q || !k || !v || !state || !o) return GDN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(state) || !aligned16(o) ||
        !opt_aligned4(beta) || !opt_aligned4(g))
        return GDN_ERR_INVALID_ARG;
    gdn::FwdOpts oo = kDefaultOut;
    if (opts) {
        if (opts->out_dtype != GDN_F32 && opts->out_dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
        if (opts->g_per_key != 0 && opts->g_per_key != 1) return GDN_ERR_INVALID_ARG;
        if (!opt_aligned4(opts->d_skip)) return GDN_ERR_INVALID_ARG;
        if (!set_xnorm(*opts, &oo)) return GDN_ERR_INVALID_ARG;
        oo.bf16 = opts->out_dtype == GDN_BF16;
        oo.dskip = opts->d_skip;
        oo.gate_per_key = opts->g_per_key == 1 && g != nullptr;
    }
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return GDN_ERR_UNSUPPORTED;
    if ((double)N * H > 2147483647.0) return GDN_ERR_INVALID_ARG;
    return gdn::launch_decode(q, k, v, beta, g, state, o, N, H, dk, dv, scale, in_dtype, oo,
                              static_cast<cudaStream_t>(cuda_stream));
}

gdn_status_t gdn_decode_step(const void *q, const void *k, const void *v, const float *beta,
                             const float *g, float *state, float *o, int N, int H, int dk, int dv,
                             float scale, gdn_dtype_t in_dtype, void *cuda_stream) {
    return decode_impl(q, k, v, beta, g, state, o, N, H, dk, dv, scale, in_dtype, nullptr, cuda_stream);
}

gdn_status_t gdn_decode_step_ex(const void *q, const void *k, const void *v, const float *beta,
                                const float *g, float *state, void *o, int N, int H, int dk, int dv,
                                float scale, gdn_dtype_t in_dtype, const gdn_fwd_opts_t *opts,
                                void *cuda_stream) {
    return decode_impl(q, k, v, beta, g, state, o, N, H, dk, dv, scale, in_dtype, opts, cuda_stream);
}

size_t gdn_chunk_bwd_workspace_bytes(int B, int H, int L, int dk, int dv, int chunk) {
    if (B < 1 || H < 1 || L < 0 || chunk < 1 || chunk > 128 || !head_dim_ok(dk) || !head_dim_ok(dv)) return 0;
    return gdn::bwd_workspace_floats(static_cast<long>(B) * H, L, dk, dv, chunk) * sizeof(float);
}

gdn_status_t gdn_chunk_bwd(const void *q, const void *k, const void *v, const float *beta, const float *g,
                           const float *s0, const float *d_o, const float *ds_final, float *dq, float *dk, float *dv,
                           float *dbeta, float *dg, float *ds0, void *workspace, size_t workspace_bytes, int B, int H,
                           int L, int dk_, int dv_, int chunk, float scale, gdn_dtype_t in_dtype, void *cuda_stream) {
    if (B < 1 || H < 1 || L < 0 || !isfinite(scale) || chunk < 1) return GDN_ERR_INVALID_ARG;
    if (in_dtype != GDN_F32 && in_dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (!head_dim_ok(dk_) || !head_dim_ok(dv_) || chunk > 128) return GDN_ERR_UNSUPPORTED;
    if ((double)B * H > 2147483647.0 || (double)B * H * (double)L * 128.0 > 9.0e18) return GDN_ERR_INVALID_ARG;
    if (L > 0 && (!q || !k || !v || !d_o || !dq || !dk || !dv)) return GDN_ERR_INVALID_ARG;
    if (L > 0 && ((beta && !dbeta) || (g && !dg))) return GDN_ERR_INVALID_ARG;
    if (!opt_aligned16(q) || !opt_aligned16(k) || !opt_aligned16(v) || !opt_aligned16(d_o) || !opt_aligned16(dq) ||
        !opt_aligned16(dk) || !opt_aligned16(dv) || !opt_aligned16(s0) || !opt_aligned16(ds_final) ||
        !opt_aligned16(ds0) || !opt_aligned16(workspace) || !opt_aligned4(beta) || !opt_aligned4(g) ||
        !opt_aligned4(dbeta) || !opt_aligned4(dg))
        return GDN_ERR_INVALID_ARG;
    const size_t need = gdn_chunk_bwd_workspace_bytes(B, H, L, dk_, dv_, chunk);
    if (!workspace || workspace_bytes < need) return GDN_ERR_INVALID_ARG;
    return gdn::launch_bwd(q, k, v, beta, g, s0, d_o, ds_final, dq, dk, dv, beta ? dbeta : nullptr,
                           g ? dg : nullptr, ds0, static_cast<float *>(workspace), B, H, L, dk_, dv_, chunk, scale,
                           in_dtype, static_cast<cudaStream_t>(cuda_stream));
}

gdn_status_t gdn_state_compose(const float *mn, const float *n, const float *s_in, float *s_out, float lambda,
                               int count, int d, void *cuda_stream) {
    if (count < 0 || !isfinite(lambda) || lambda == 0.f || !isfinite(1.f / lambda)) return GDN_ERR_INVALID_ARG;
    if (!head_dim_ok(d)) return GDN_ERR_UNSUPPORTED;
    if (count == 0) return GDN_OK;
    if (!mn || !n || !s_out || !aligned16(mn) || !aligned16(n) || !aligned16(s_out) || !opt_aligned16(s_in))
        return GDN_ERR_INVALID_ARG;
    if ((double)count * d * d > 9.0e18 || count > 2147483647 / 4) return GDN_ERR_INVALID_ARG;
    // s_out is written while mn, n and s_in are still being read by other CTAs
    const size_t bytes = static_cast<size_t>(count) * d * d * sizeof(float);
    auto overlaps = [&](const float *a) {
        const char *x = reinterpret_cast<const char *>(a), *y = reinterpret_cast<const char *>(s_out);
        return a && x < y + bytes && y < x + bytes;
    };
    if (overlaps(mn) || overlaps(n) || overlaps(s_in)) return GDN_ERR_INVALID_ARG;
    return gdn::launch_state_compose(mn, n, s_in, s_out, lambda, count, d, static_cast<cudaStream_t>(cuda_stream));
}

gdn_status_t gdn_state_identity(float *s, float value, int count, int d, void *cuda_stream) {
    if (count < 0 || !isfinite(value)) return GDN_ERR_INVALID_ARG;
    if (!head_dim_ok(d)) return GDN_ERR_UNSUPPORTED;
    if (count == 0) return GDN_OK;
    if (!s || !aligned16(s)) return GDN_ERR_INVALID_ARG;
    return gdn::launch_state_identity(s, value, count, d, static_cast<cudaStream_t>(cuda_stream));
}

}  // extern "C"
