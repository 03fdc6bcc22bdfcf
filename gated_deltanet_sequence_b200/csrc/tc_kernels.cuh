// Tensor-core (tcgen05 + TMA) prefill kernels for sm_100a: host-side interface.
#pragma once
#include "common.cuh"

namespace gdn {
// True when the tcgen05 kernels handle this configuration.
bool tc_supported(gdn_dtype_t in_dtype, int dk, int dv, int chunk);
gdn_status_t launch_tc_gdn(const void *q, const void *k, const void *v, const float *beta,
                           const float *g, float *o, const float *s0, float *s_final, int B, int H,
                           int L, float scale, cudaStream_t stream);
gdn_status_t launch_tc_la(const void *q, const void *k, const void *v, const float *g, float *o,
                          const float *s0, float *s_final, int B, int H, int L, float scale,
                          cudaStream_t stream);
// Reads and clears the device-side error word of the current device.
bool read_and_clear_device_error(unsigned *err);
}  // namespace gdn
