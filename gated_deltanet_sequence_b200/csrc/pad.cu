// Head sizes of 64 on the tensor cores: copies of the operands zero-padded to 128.
//
// With dk = 64 the key coordinates 64..127 of the padded q and k are zero: every product over
// the key dimension (q.k, k.k, and the reads S^T k, S^T q) is unchanged, and rows 64..127 of
// the state only ever receive k_t[j] u_t^T = 0 (and decay from zero), so they stay zero. With
// dv = 64 the value columns 64..127 of v are zero and the state's columns 64..127 and the
// output's stay zero, independent of the others. So a call at dk or dv = 64 gives, on the first
// dk x dv entries, the results of the padded call at 128 x 128, which runs on the tensor-core
// kernels; the padded output and state are then cropped. A vector-valued gate is padded with
// zero log-decays, the skip weights with zeros.
#include <algorithm>
#include <mutex>

#include "tc_kernels.cuh"

namespace gdn {

namespace {

// dst[o][r][c] = (r < rows_src && c < cols_src) ? src[o][r][c] : 0 in 16-byte units; rows are
// cols_* bytes long (multiples of 16). With rows_src >= rows_dst and cols_src >= cols_dst this
// crops instead.
__global__ void pad_copy_kernel(uint4 *__restrict__ dst, const uint4 *__restrict__ src, long long n_outer,
                                int rows_dst, int cw_dst, int rows_src, int cw_src) {
    const long long total = n_outer * rows_dst * cw_dst;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int c = static_cast<int>(i % cw_dst);
        const long long orow = i / cw_dst;
        const int r = static_cast<int>(orow % rows_dst);
        const long long o = orow / rows_dst;
        uint4 x = make_uint4(0u, 0u, 0u, 0u);
        if (r < rows_src && c < cw_src) x = src[(o * rows_src + r) * cw_src + c];
        dst[i] = x;
    }
}

cudaMemPool_t pad_pool(int dev) {
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
        unsigned long long keep = ~0ull;
        cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &keep);
        pools[dev] = p;
    }
    return pools[dev];
}

}  // namespace

bool pad_copy(void *dst, const void *src, long long n_outer, int rows_dst, int cols_dst_bytes, int rows_src,
              int cols_src_bytes, cudaStream_t stream) {
    const long long total = n_outer * rows_dst * (cols_dst_bytes / 16);
    if (total <= 0) return true;
    const int sms = sm_count();
    const long long blocks = std::min<long long>((total + 255) / 256, static_cast<long long>(sms > 0 ? sms : 148) * 8);
    pad_copy_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<uint4 *>(dst), static_cast<const uint4 *>(src), n_outer, rows_dst, cols_dst_bytes / 16, rows_src,
        cols_src_bytes / 16);
    return cudaGetLastError() == cudaSuccess;
}

bool pad_alloc(void **p, size_t bytes, cudaStream_t stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    cudaMemPool_t pool = pad_pool(dev);
    if (!pool || cudaMallocFromPoolAsync(p, bytes, pool, stream) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return true;
}

}  // namespace gdn
