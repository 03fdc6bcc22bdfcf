// State composition for the sequence-split (context-parallel) prefill.
//
// Over one segment of a sequence the token recurrence is affine in the state that enters
// the segment (page "混合注意力学习(1)", section "Gated DeltaNet": each token maps the state,
// in the key-row layout, by S -> alpha (I - beta k k^T) S + beta k v^T; plain and gated
// linear attention drop the erase term): S_out = M S_in + N, with M (d x d) the ordered
// product of the segment's token maps and N (d x d) the segment's state from a zero start.
// With dk = dv = d, a prefill run of the segment from S0 = lambda I ends in lambda M + N and a
// run from S0 = 0 ends in N, so the prefill kernels produce both; the two kernels here write
// the scaled identity states and apply S_out = ((lambda M + N) - N) / lambda S_in + N in fp32
// (lambda a power of two keeps the division exact; a large lambda keeps the rounding of N,
// which the subtraction cancels, small next to M). Segments (or ranks) apply this in order to
// find the state entering each segment, and a last prefill run of each segment from that
// state gives its outputs.
#include "common.cuh"

namespace gdn {

namespace {

constexpr int kTile = 32;   // output rows per CTA and the k step

// One CTA: rows r0 .. r0+31 of s_out for one state. Warp w owns rows r0 + 4w .. r0 + 4w + 3,
// lane l columns l, l + 32, ...; M tiles (32 x 32, padded) and S_in tiles (32 x D) pass
// through shared memory. Sums run over k in increasing order.
template <int D>
__global__ void __launch_bounds__(256) compose_kernel(const float *__restrict__ mn, const float *__restrict__ n,
                                                      const float *__restrict__ s_in, float *__restrict__ s_out,
                                                      float inv_lambda) {
    constexpr int NC = D / 32;
    __shared__ float sm[kTile][kTile + 1];
    __shared__ float ss[kTile][D];
    const size_t base = static_cast<size_t>(blockIdx.x) * D * D;
    const int r0 = blockIdx.y * kTile;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float acc[4][NC];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < NC; ++j) acc[i][j] = 0.f;
    if (s_in) {
#pragma unroll 1
        for (int k0 = 0; k0 < D; k0 += kTile) {
#pragma unroll
            for (int e = tid; e < kTile * kTile; e += 256) {
                const int i = e >> 5, j = e & 31;
                const size_t at = base + static_cast<size_t>(r0 + i) * D + k0 + j;
                sm[i][j] = (mn[at] - n[at]) * inv_lambda;
            }
#pragma unroll
            for (int e = tid; e < kTile * D; e += 256) {
                const int i = e / D, j = e % D;
                ss[i][j] = s_in[base + static_cast<size_t>(k0 + i) * D + j];
            }
            __syncthreads();
#pragma unroll 8
            for (int kk = 0; kk < kTile; ++kk) {
                float m[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) m[i] = sm[4 * warp + i][kk];
#pragma unroll
                for (int j = 0; j < NC; ++j) {
                    const float s = ss[kk][lane + 32 * j];
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[i][j] = fmaf(m[i], s, acc[i][j]);
                }
            }
            __syncthreads();
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const size_t row = base + static_cast<size_t>(r0 + 4 * warp + i) * D;
#pragma unroll
        for (int j = 0; j < NC; ++j) s_out[row + lane + 32 * j] = acc[i][j] + n[row + lane + 32 * j];
    }
}

__global__ void identity_kernel(float *__restrict__ s, float value, long long total, int d) {
    for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
         e += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long within = e % (static_cast<long long>(d) * d);
        s[e] = (within / d == within % d) ? value : 0.f;
    }
}

}  // namespace

gdn_status_t launch_state_compose(const float *mn, const float *n, const float *s_in, float *s_out, float lambda,
                                  int count, int d, cudaStream_t stream) {
    const dim3 grid(count, d / kTile);
    if (d == 128)
        compose_kernel<128><<<grid, 256, 0, stream>>>(mn, n, s_in, s_out, 1.f / lambda);
    else
        compose_kernel<64><<<grid, 256, 0, stream>>>(mn, n, s_in, s_out, 1.f / lambda);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status_t launch_state_identity(float *s, float value, int count, int d, cudaStream_t stream) {
    const long long total = static_cast<long long>(count) * d * d;
    const long long want = (total + 255) / 256;
    const int blocks = static_cast<int>(want < 4096 ? want : 4096);
    identity_kernel<<<blocks, 256, 0, stream>>>(s, value, total, d);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace gdn
