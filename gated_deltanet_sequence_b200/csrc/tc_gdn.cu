// Tensor-core chunkwise prefill kernels (tcgen05 + TMA, sm_100a).
#include "tc_kernels.cuh"

namespace gdn {

// Device-side error word (static storage in the library image, one per device).
__device__ unsigned g_device_error = 0u;

bool read_and_clear_device_error(unsigned *err) {
    const unsigned zero = 0u;
    if (cudaMemcpyFromSymbol(err, g_device_error, sizeof(unsigned)) != cudaSuccess) return false;
    if (*err != 0u && cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess)
        return false;
    return true;
}

bool tc_supported(gdn_dtype_t, int, int, int) { return false; }

gdn_status_t launch_tc_gdn(const void *, const void *, const void *, const float *, const float *,
                           float *, const float *, float *, int, int, int, float, cudaStream_t) {
    return GDN_ERR_UNSUPPORTED;
}
gdn_status_t launch_tc_la(const void *, const void *, const void *, const float *, float *,
                          const float *, float *, int, int, int, float, cudaStream_t) {
    return GDN_ERR_UNSUPPORTED;
}

}  // namespace gdn
