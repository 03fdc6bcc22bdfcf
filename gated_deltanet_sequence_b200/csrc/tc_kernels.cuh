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
// Number of SMs of the current device (cached per device); 0 on error.
int sm_count();
gdn_status_t launch_tc_la(const void *q, const void *k, const void *v, const float *g, void *o,
                          const float *s0, float *s_final, const int *cu, int B, int H, int L,
                          float scale, FwdOpts oo, cudaStream_t stream);
// Takes one condition out of the device-side error word of the current device, on
// `stream` (a one-thread kernel clears only the bit it reports, atomically, so a bit
// that another kernel sets meanwhile is kept for the next call): *err receives
// kErrBadSeqlens if that bit was set, else kErrWaitTimeout if that one was, else
// kErrNonFinite if that one was, else 0.
bool take_device_error(cudaStream_t stream, unsigned *err);
// Device address of that word on the current device (looked up once per device),
// handed to kernels that may record a bounded-wait timeout; nullptr on failure.
unsigned *device_error_word();
// Bounded-wait limit of the tensor-core kernels (clock cycles, ~2 s at 2 GHz), and the
// limit of their final drains of copies and UMMAs already issued (always this value).
constexpr long long kWaitLimitCycles = 4000000000LL;
constexpr long long kDrainLimitCycles = 4000000000LL;
// The wait limit handed to the next launches: kWaitLimitCycles unless a test lowered it
// through gdn_set_wait_limit_for_testing.
long long wait_limit_cycles();
// Raises the dynamic shared-memory limit of kernel `fn` to `bytes` on the current device
// (once per device and kernel). False on a CUDA error.
bool ensure_smem_limit(const void *fn, unsigned bytes);
}  // namespace gdn

#include <cuda.h>
namespace gdn {
// 3-D TMA map over a (BH, L, 128) bf16 tensor: 64 x 64 boxes, 128-byte swizzle,
// zero fill outside the tensor (rows past L read as zeros).
bool make_qkv_map(CUtensorMap *m, const void *ptr, int L, int BH);
}  // namespace gdn
