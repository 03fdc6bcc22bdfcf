// Prefill from pinned host buffers: the batch crosses PCIe in groups of sequences while
// earlier groups are computed, on three CUDA streams with two device staging slots.
//
// The (sequence, head) recurrences are independent (each head of each sequence carries its
// own state), so a batch can be split between sequences without changing any result: every
// group is one call of the dense prefill, which gives each (sequence, head) the same bits
// whatever the batch around it. While group i is computed, group i + 1 is uploaded and group
// i - 1 downloaded; the host-to-device and device-to-host copies overlap each other (PCIe is
// full duplex) and the compute, so a step costs about the larger transfer. Each tensor of a
// group is one cudaMemcpyAsync (the group's rows are contiguous in the (B, H, L, d) layout).
#include <math.h>

#include <vector>

#include "common.cuh"

namespace {

constexpr size_t kAlign = 256;
size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Byte layout of one staging slot for `G` sequences.
struct SlotLayout {
    size_t q, k, v, beta, g, s0, o, sf, bytes;
};
SlotLayout slot_layout(int G, int H, int L, int dk, int dv, size_t in_bytes, bool has_g, bool has_s0,
                       bool has_sf) {
    SlotLayout s{};
    const size_t rows = static_cast<size_t>(G) * H * L;
    size_t at = 0;
    s.q = at; at += up(rows * dk * in_bytes);
    s.k = at; at += up(rows * dk * in_bytes);
    s.v = at; at += up(rows * dv * in_bytes);
    s.beta = at; at += up(rows * sizeof(float));
    s.g = at; if (has_g) at += up(rows * sizeof(float));
    s.s0 = at; if (has_s0) at += up(static_cast<size_t>(G) * H * dk * dv * sizeof(float));
    s.o = at; at += up(rows * dv * sizeof(float));
    s.sf = at; if (has_sf) at += up(static_cast<size_t>(G) * H * dk * dv * sizeof(float));
    s.bytes = at;
    return s;
}

bool pinned_host(const void *p) {
    if (!p) return true;
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();   // clear the (non-sticky) error of the query
        return false;
    }
    return a.type == cudaMemoryTypeHost;
}

// Owns the pipeline's streams and events; releasing them never waits (the runtime frees
// them once their work is done).
struct Pipeline {
    cudaStream_t up = nullptr, comp = nullptr, down = nullptr;
    std::vector<cudaEvent_t> events;
    ~Pipeline() {
        for (cudaEvent_t e : events) cudaEventDestroy(e);
        if (up) cudaStreamDestroy(up);
        if (comp) cudaStreamDestroy(comp);
        if (down) cudaStreamDestroy(down);
    }
    cudaEvent_t event() {
        cudaEvent_t e = nullptr;
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return nullptr;
        events.push_back(e);
        return e;
    }
};

}  // namespace

extern "C" {

size_t gdn_chunk_fwd_host_staging_bytes(int B, int H, int L, int dk, int dv, int group, gdn_dtype_t in_dtype,
                                        int has_g, int has_s0, int has_s_final) {
    if (B < 1 || H < 1 || L < 0 || dk < 1 || dv < 1 || group < 1) return 0;
    const int G = group < B ? group : B;
    const size_t in_bytes = in_dtype == GDN_BF16 ? 2 : 4;
    return 2 * slot_layout(G, H, L, dk, dv, in_bytes, has_g != 0, has_s0 != 0, has_s_final != 0).bytes;
}

gdn_status_t gdn_chunk_fwd_host(const void *q, const void *k, const void *v, const float *beta, const float *g,
                                float *o, const float *s0, float *s_final, void *staging, size_t staging_bytes,
                                int B, int H, int L, int dk, int dv, int chunk, float scale, gdn_dtype_t in_dtype,
                                int group, void *cuda_stream) {
    if (B < 1 || H < 1 || L < 1 || group < 1 || !isfinite(scale)) return GDN_ERR_INVALID_ARG;
    if (in_dtype != GDN_F32 && in_dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (!q || !k || !v || !beta || !o || !staging) return GDN_ERR_INVALID_ARG;
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128) || chunk < 1 || chunk > 64) return GDN_ERR_UNSUPPORTED;
    for (const void *p : {q, k, v, static_cast<const void *>(beta), static_cast<const void *>(g),
                          static_cast<const void *>(o), static_cast<const void *>(s0),
                          static_cast<const void *>(s_final)})
        if (!pinned_host(p)) return GDN_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(staging) % kAlign != 0) return GDN_ERR_INVALID_ARG;
    const size_t need = gdn_chunk_fwd_host_staging_bytes(B, H, L, dk, dv, group, in_dtype, g != nullptr,
                                                         s0 != nullptr, s_final != nullptr);
    if (need == 0 || staging_bytes < need) return GDN_ERR_INVALID_ARG;

    const int G = group < B ? group : B;
    const size_t in_bytes = in_dtype == GDN_BF16 ? 2 : 4;
    const SlotLayout lay = slot_layout(G, H, L, dk, dv, in_bytes, g != nullptr, s0 != nullptr, s_final != nullptr);
    const size_t seq_rows = static_cast<size_t>(H) * L;            // token rows of one sequence
    const size_t seq_state = static_cast<size_t>(H) * dk * dv;      // state floats of one sequence
    cudaStream_t caller = static_cast<cudaStream_t>(cuda_stream);

    Pipeline pl;
    if (cudaStreamCreateWithFlags(&pl.up, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&pl.comp, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&pl.down, cudaStreamNonBlocking) != cudaSuccess)
        return GDN_ERR_CUDA;
    cudaEvent_t start = pl.event();
    if (!start || cudaEventRecord(start, caller) != cudaSuccess) return GDN_ERR_CUDA;
    cudaEvent_t free_in[2] = {start, start}, free_out[2] = {start, start}, last = start;
    auto ok = [](cudaError_t e) { return e == cudaSuccess; };
    bool good = true;
    for (int i = 0, b0 = 0; good && b0 < B; ++i, b0 += G) {
        const int n = (B - b0) < G ? (B - b0) : G;
        char *slot = static_cast<char *>(staging) + static_cast<size_t>(i & 1) * lay.bytes;
        const size_t r0 = static_cast<size_t>(b0) * seq_rows, nr = static_cast<size_t>(n) * seq_rows;
        const size_t st0 = static_cast<size_t>(b0) * seq_state, nst = static_cast<size_t>(n) * seq_state;
        // upload (once the slot's previous group has been computed)
        good = ok(cudaStreamWaitEvent(pl.up, free_in[i & 1], 0)) &&
               ok(cudaMemcpyAsync(slot + lay.q, static_cast<const char *>(q) + r0 * dk * in_bytes, nr * dk * in_bytes,
                                  cudaMemcpyHostToDevice, pl.up)) &&
               ok(cudaMemcpyAsync(slot + lay.k, static_cast<const char *>(k) + r0 * dk * in_bytes, nr * dk * in_bytes,
                                  cudaMemcpyHostToDevice, pl.up)) &&
               ok(cudaMemcpyAsync(slot + lay.v, static_cast<const char *>(v) + r0 * dv * in_bytes, nr * dv * in_bytes,
                                  cudaMemcpyHostToDevice, pl.up)) &&
               ok(cudaMemcpyAsync(slot + lay.beta, beta + r0, nr * sizeof(float), cudaMemcpyHostToDevice, pl.up)) &&
               (!g || ok(cudaMemcpyAsync(slot + lay.g, g + r0, nr * sizeof(float), cudaMemcpyHostToDevice, pl.up))) &&
               (!s0 || ok(cudaMemcpyAsync(slot + lay.s0, s0 + st0, nst * sizeof(float), cudaMemcpyHostToDevice, pl.up)));
        cudaEvent_t loaded = good ? pl.event() : nullptr;
        good = good && loaded && ok(cudaEventRecord(loaded, pl.up));
        // compute (once uploaded and the slot's previous outputs are downloaded)
        good = good && ok(cudaStreamWaitEvent(pl.comp, loaded, 0)) && ok(cudaStreamWaitEvent(pl.comp, free_out[i & 1], 0));
        if (good)
            good = gdn_chunk_fwd(slot + lay.q, slot + lay.k, slot + lay.v, reinterpret_cast<const float *>(slot + lay.beta),
                                 g ? reinterpret_cast<const float *>(slot + lay.g) : nullptr,
                                 reinterpret_cast<float *>(slot + lay.o),
                                 s0 ? reinterpret_cast<const float *>(slot + lay.s0) : nullptr,
                                 s_final ? reinterpret_cast<float *>(slot + lay.sf) : nullptr, n, H, L, dk, dv, chunk,
                                 scale, in_dtype, pl.comp) == GDN_OK;
        cudaEvent_t done = good ? pl.event() : nullptr;
        good = good && done && ok(cudaEventRecord(done, pl.comp));
        if (good) free_in[i & 1] = done;
        // download
        good = good && ok(cudaStreamWaitEvent(pl.down, done, 0)) &&
               ok(cudaMemcpyAsync(o + r0 * dv, slot + lay.o, nr * dv * sizeof(float), cudaMemcpyDeviceToHost, pl.down)) &&
               (!s_final || ok(cudaMemcpyAsync(s_final + st0, slot + lay.sf, nst * sizeof(float),
                                               cudaMemcpyDeviceToHost, pl.down)));
        cudaEvent_t out = good ? pl.event() : nullptr;
        good = good && out && ok(cudaEventRecord(out, pl.down));
        if (good) free_out[i & 1] = last = out;
    }
    if (!good) {
        // leave nothing of this call in flight behind the caller's back
        cudaStreamSynchronize(pl.up);
        cudaStreamSynchronize(pl.comp);
        cudaStreamSynchronize(pl.down);
        return GDN_ERR_CUDA;
    }
    // the caller's stream continues once the last download is done (it follows every copy
    // and computation of the call)
    return cudaStreamWaitEvent(caller, last, 0) == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // extern "C"
