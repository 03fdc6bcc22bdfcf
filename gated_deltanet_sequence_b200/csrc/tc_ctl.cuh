// Bounded waits and the abort protocol shared by the tensor-core kernels.
//
// Every mbarrier wait gives up after `limit` clock cycles. The first wait that gives up
// records kErrWaitTimeout in the device-side error word and sets a CTA-wide abort flag;
// from then on every wait fails at once, and each role stops issuing (no further
// arrivals, copies or UMMAs) and leaves its loop. Warp groups decide together: the
// group leader polls, and the group meets on a reduction barrier (bar.red.or) whose
// result — "did any member see a failure" — every member receives from the barrier
// itself, so no member can read a verdict that another member changes afterwards.
// The TMA thread and the UMMA issuers then drain what they issued, with a fixed long
// limit that does not depend on `limit` (copies and UMMAs in flight always complete),
// before the CTA frees its tensor memory and exits.
#pragma once
#include "tc_kernels.cuh"
#include "tc_ptx.cuh"

namespace gdn {
namespace ptx {

// Named barrier over `nthreads` threads (a multiple of 32) that also ORs `pred` over
// them: every participant gets true when any participant passed true.
__device__ __forceinline__ bool named_bar_any(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

}  // namespace ptx

struct Ctl {
    uint64_t *bar;
    int *abort_flag;     // CTA-wide: set by the first wait that gives up
    unsigned *err;
    long long limit;     // cycles a wait may take before it gives up

    __device__ __forceinline__ bool aborted() const { return *reinterpret_cast<volatile int *>(abort_flag) != 0; }
    __device__ __forceinline__ bool give_up() const {
        atomicOr(err, kErrWaitTimeout);
        *reinterpret_cast<volatile int *>(abort_flag) = 1;
        return false;
    }
    __device__ __forceinline__ bool wait(int b, uint32_t parity) const {
        if (aborted()) return false;
        return ptx::mbar_wait(&bar[b], parity, limit) ? true : give_up();
    }
    // Cluster-scope acquire, for phases completed by arrivals of another CTA of the
    // cluster (its shared-memory writes become visible here).
    __device__ __forceinline__ bool wait_cluster(int b, uint32_t parity) const {
        if (aborted()) return false;
        return ptx::mbar_wait_cluster(&bar[b], parity, limit) ? true : give_up();
    }
    // Sleeps between polls, for roles off the critical path (their polling would
    // otherwise take issue slots from the warps they share a scheduler with).
    __device__ __forceinline__ bool wait_lazy(int b, uint32_t parity) const {
        if (aborted()) return false;
        const uint32_t a = ptx::smem_u32(&bar[b]);
        if (ptx::mbar_try_wait(a, parity)) return true;
        const long long t0 = clock64();
        do {
            __nanosleep(100);
            if (ptx::mbar_try_wait(a, parity)) return true;
        } while (clock64() - t0 <= limit);
        return give_up();
    }
    // Wait for operations this thread issued (TMA copies, UMMA commits); ignores the
    // abort flag and uses the fixed drain limit.
    __device__ __forceinline__ void drain(int b, uint32_t parity) const {
        ptx::mbar_wait(&bar[b], parity, kDrainLimitCycles);
    }
    // Group-uniform wait: the leader polls; the group meets on `bar_id` and every thread
    // gets the same verdict.
    __device__ __forceinline__ bool group_wait(int b, uint32_t parity, int bar_id, bool leader,
                                               int nthreads = 128) const {
        const bool fail = leader && !wait(b, parity);
        return !ptx::named_bar_any(bar_id, nthreads, fail);
    }
    __device__ __forceinline__ bool group_wait_cluster(int b, uint32_t parity, int bar_id, bool leader,
                                                       int nthreads = 128) const {
        const bool fail = leader && !wait_cluster(b, parity);
        return !ptx::named_bar_any(bar_id, nthreads, fail);
    }
    // Several phases, one barrier: the leader polls each in turn (entries with b < 0 are
    // skipped; bit i of cluster_mask selects the cluster-scope acquire for entry i).
    template <int N>
    __device__ __forceinline__ bool group_wait_all(const int (&b)[N], const uint32_t (&parity)[N], int bar_id,
                                                   bool leader, int nthreads = 128, unsigned cluster_mask = 0u) const {
        bool fail = false;
        if (leader) {
#pragma unroll
            for (int i = 0; i < N; ++i)
                if (!fail && b[i] >= 0)
                    fail = !(((cluster_mask >> i) & 1u) ? wait_cluster(b[i], parity[i]) : wait(b[i], parity[i]));
        }
        return !ptx::named_bar_any(bar_id, nthreads, fail);
    }
};

}  // namespace gdn
