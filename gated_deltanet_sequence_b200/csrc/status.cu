// Library-wide host state of libgdn.so: the device-side error word that kernels report
// into, the bounded-wait limit handed to the tensor-core kernels, and the per-device
// shared-memory attribute of the kernels that need more than the default 48 KB.
#include <atomic>
#include <mutex>
#include <set>
#include <utility>

#include "tc_kernels.cuh"

namespace gdn {

// Device-side error word: one per device (static storage in the library image), shared
// by every kernel of this library on that device, whatever stream or caller launched it.
__device__ unsigned g_device_error = 0u;
// Where the one-thread kernel below leaves the condition it took out of the word.
__device__ unsigned g_error_taken = 0u;

namespace {

std::atomic<long long> g_wait_limit{kWaitLimitCycles};

// Reports one condition and clears only that bit, atomically: a malformed sequence-offset
// list first, then a bounded wait that gave up, then (debug builds) an access out of its
// extent, then a non-finite stored result. Bits set meanwhile by kernels on other streams
// stay in the word.
__global__ void take_error_kernel(unsigned *word, unsigned *taken) {
    const unsigned now = atomicOr(word, 0u);
    const unsigned bit = (now & kErrBadSeqlens)    ? kErrBadSeqlens
                         : (now & kErrWaitTimeout) ? kErrWaitTimeout
                         : (now & kErrBounds)      ? kErrBounds
                                                   : (now & kErrNonFinite);
    if (bit) atomicAnd(word, ~bit);
    *taken = bit;
}

}  // namespace

unsigned *device_error_word() {
    static std::mutex mu;
    static unsigned *addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        addr[dev] = static_cast<unsigned *>(p);
    }
    return addr[dev];
}

bool take_device_error(cudaStream_t stream, unsigned *err) {
    unsigned *word = device_error_word();
    void *taken = nullptr;
    if (!word || cudaGetSymbolAddress(&taken, g_error_taken) != cudaSuccess) return false;
    take_error_kernel<<<1, 1, 0, stream>>>(word, static_cast<unsigned *>(taken));
    if (cudaGetLastError() != cudaSuccess) return false;
    if (cudaMemcpyAsync(err, taken, sizeof(unsigned), cudaMemcpyDeviceToHost, stream) != cudaSuccess) return false;
    return cudaStreamSynchronize(stream) == cudaSuccess;
}

int sm_count() {
    static std::mutex mu;
    static int sms[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    std::lock_guard<std::mutex> lock(mu);
    if (sms[dev] == 0 && cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    return sms[dev];
}

long long wait_limit_cycles() { return g_wait_limit.load(std::memory_order_relaxed); }

bool ensure_smem_limit(const void *fn, unsigned bytes) {
    static std::mutex mu;
    static std::set<std::pair<int, const void *>> done;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> lock(mu);
    if (done.count({dev, fn})) return true;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) !=
        cudaSuccess)
        return false;
    done.insert({dev, fn});
    return true;
}

}  // namespace gdn

extern "C" {

void gdn_set_wait_limit_for_testing(long long cycles) {
    gdn::g_wait_limit.store(cycles > 0 ? cycles : gdn::kWaitLimitCycles, std::memory_order_relaxed);
}

gdn_status_t gdn_sync_status(void *cuda_stream) {
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    if (cudaStreamSynchronize(stream) != cudaSuccess) return GDN_ERR_CUDA;
    unsigned err = 0u;
    if (!gdn::take_device_error(stream, &err)) return GDN_ERR_CUDA;
    if (err & gdn::kErrBadSeqlens) return GDN_ERR_INVALID_ARG;
    if (err & gdn::kErrWaitTimeout) return GDN_ERR_TIMEOUT;
    if (err & gdn::kErrBounds) return GDN_ERR_BOUNDS;
    return err ? GDN_ERR_NONFINITE : GDN_OK;
}

}  // extern "C"
