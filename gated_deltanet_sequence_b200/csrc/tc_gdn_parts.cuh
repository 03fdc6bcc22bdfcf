// Device helpers shared by the Gated DeltaNet tensor-core kernels (one-CTA and
// cluster forms): TMEM row loads, fp16 operand stores in the 128-byte swizzled
// layout, the output and W epilogues, and the warp-level tf32 block products of the UT
// solve. The bounded waits and the abort protocol are in tc_ctl.cuh.
#pragma once
#include "tc_ctl.cuh"

namespace gdn {
namespace tcgdn {
using namespace ptx;
using gdn::Ctl;

constexpr int kC = 64;           // chunk rows
constexpr int kD = 128;          // dk = dv

template <int N>
__device__ __forceinline__ void ld_cols(uint32_t taddr, float (&v)[N]) {
    static_assert(N % 16 == 0, "16-column pieces");
#pragma unroll
    for (int cc = 0; cc < N / 16; ++cc) {
        float t[16];
        tmem_ld16(taddr + cc * 16, t);
#pragma unroll
        for (int e = 0; e < 16; ++e) v[cc * 16 + e] = t[e];
    }
    tmem_wait_ld();
}

// 16 fp32 values -> two swizzled 16-byte chunks (ch, ch+1) of row `row` in a 128-byte-row tile
__device__ __forceinline__ void st_row16_h(uint32_t tile, uint32_t row, int ch, const float *x) {
    st_shared_v4(tile + sw128(row, ch), pack_h2(x[0], x[1]), pack_h2(x[2], x[3]), pack_h2(x[4], x[5]),
                 pack_h2(x[6], x[7]));
    st_shared_v4(tile + sw128(row, ch + 1), pack_h2(x[8], x[9]), pack_h2(x[10], x[11]), pack_h2(x[12], x[13]),
                 pack_h2(x[14], x[15]));
}

// 64 output rows of one value column from TMEM to HBM (rows >= n are padding), with the
// output options (fp32 / bf16, D-skip term, output normalisation) when OPTS, plain fp32
// otherwise. With OPTS the whole 128-thread group (thread gt = value column) calls it
// and meets on bar_id; xn: 384 floats of shared scratch; head indexes the (H, dv) weights.
// With `probe` the stored values go through the non-finite probe nf.
template <bool OPTS>
__device__ __forceinline__ void store_out_col(uint32_t taddr, const OutArgs &out, size_t elem0, int n, int head,
                                              int gt, int bar_id, float *xn, bool probe, float &nf) {
    float ov[64];
    ld_cols<64>(taddr, ov);
    if constexpr (OPTS) {
        store_out_rows_group(ov, out, elem0, n, head, gt, bar_id, xn, xn + 256, probe, nf);
    } else {
        float *ocol = static_cast<float *>(out.o) + elem0;
#pragma unroll
        for (int r = 0; r < 64; ++r)
            if (r < n) ocol[static_cast<size_t>(r) * kD] = ov[r];
        if (probe) probe_tile(nf, ov, n);
    }
}

// W^T row j (TMEM) -> fp16 MN-major W operand in a stage's V slot
__device__ __forceinline__ void store_w_row(uint32_t trow_x, uint32_t wtile, int j) {
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
        float w[16];
        tmem_ld16(trow_x + cc * 16, w);
        tmem_wait_ld();
        st_row16_h(wtile, j, 2 * cc, w);
    }
}

// warp-level tensor-core product for the small blocks of the UT solve (tf32 inputs,
// fp32 accumulation): d += a (16 x 8, row-major) * b (8 x 8)
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t u;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(u) : "f"(x));
    return u;
}
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// acc (16 x 16, two 16 x 8 tiles) += X (16 x 8KS) * Z (8KS x 16), both read from shared
// memory through the accessors; lane layout of the m16n8k8 fragments (g = lane / 4,
// t = lane % 4): A (g|g+8, t|t+4), B (t|t+4, g), D (g|g+8, 2t|2t+1)
template <int KS, typename XF, typename ZF>
__device__ __forceinline__ void block_mm(float (&acc)[2][4], XF xget, ZF zget, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll 1
    for (int ks = 0; ks < KS; ++ks) {
        const uint32_t a[4] = {to_tf32(xget(g, 8 * ks + t)), to_tf32(xget(g + 8, 8 * ks + t)),
                               to_tf32(xget(g, 8 * ks + t + 4)), to_tf32(xget(g + 8, 8 * ks + t + 4))};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const uint32_t b[2] = {to_tf32(zget(8 * ks + t, 8 * nt + g)), to_tf32(zget(8 * ks + t + 4, 8 * nt + g))};
            mma_tf32_16x8x8(acc[nt], a, b);
        }
    }
}
// write a block_mm result (optionally negated) through an accessor
template <typename WF>
__device__ __forceinline__ void block_store(const float (&acc)[2][4], WF wput, int lane, float sgn) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        wput(g, 8 * nt + 2 * t, sgn * acc[nt][0]);
        wput(g, 8 * nt + 2 * t + 1, sgn * acc[nt][1]);
        wput(g + 8, 8 * nt + 2 * t, sgn * acc[nt][2]);
        wput(g + 8, 8 * nt + 2 * t + 1, sgn * acc[nt][3]);
    }
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

}  // namespace tcgdn
}  // namespace gdn
