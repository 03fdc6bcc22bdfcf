// Tensor-core (tcgen05 + TMA) prefill kernels for sm_100a: host-side interface.
#pragma once
#include "common.cuh"

namespace gdn {
// True when the tcgen05 kernels handle this configuration.
bool tc_supported(gdn_dtype_t in_dtype, int dk, int dv, int chunk);
// cu (device, nullable): sequence offsets of a packed batch; B is then the number of
// sequences and L the packed length T of each head row (tokens of head h at rows h*T ..).
// o is fp32 or bf16 as oo.bf16 says; oo.dskip adds the D-skip term (v is then read again
// from global memory by the output epilogue).
gdn_status_t launch_tc_gdn(const void *q, const void *k, const void *v, const float *beta,
                           const float *g, void *o, const float *s0, float *s_final, const int *cu,
                           int B, int H, int L, float scale, FwdOpts oo, cudaStream_t stream);
// Cluster form (one chain CTA + two prep CTAs per (sequence, head)); same arguments and
// the same bits as launch_tc_gdn. tc_gdn_cluster_fits: every cluster fits on the device
// at once (3 x B*H <= SM count), i.e. the one-CTA form would leave most SMs idle.
gdn_status_t launch_tc_gdn_cluster(const void *q, const void *k, const void *v, const float *beta,
                                   const float *g, void *o, const float *s0, float *s_final,
                                   const int *cu, int B, int H, int L, float scale, FwdOpts oo,
                                   cudaStream_t stream);
bool tc_gdn_cluster_fits(int nctas);
gdn_status_t launch_tc_la(const void *q, const void *k, const void *v, const float *g, void *o,
                          const float *s0, float *s_final, const int *cu, int B, int H, int L,
                          float scale, FwdOpts oo, cudaStream_t stream);
// Reads and clears the device-side error word of the current device.
bool read_and_clear_device_error(unsigned *err);
// Device address of that word on the current device (looked up once per device),
// handed to kernels that may record a bounded-wait timeout; nullptr on failure.
unsigned *device_error_word();
// Bounded-wait limit handed to the tensor-core kernels (clock cycles, ~2 s at 2 GHz).
constexpr long long kWaitLimitCycles = 4000000000LL;
}  // namespace gdn

#include <cuda.h>
namespace gdn {
// 3-D TMA map over a (BH, L, 128) bf16 tensor: 64 x 64 boxes, 128-byte swizzle,
// zero fill outside the tensor (rows past L read as zeros).
bool make_qkv_map(CUtensorMap *m, const void *ptr, int L, int BH);
}  // namespace gdn
