// kpa_noalloc.cu -- kpa_decode for callers that cannot allocate device memory.
//
// kpa_decode needs a scratch workspace for its per-split partial results.  Some
// callers can neither call cudaMalloc nor carve a workspace out of memory they
// own: code that runs while a stream is being captured in a mode that forbids
// allocation, plugins whose host framework owns every device allocation, or
// serving loops that must not allocate on the decode path.  For them this file
// keeps one fixed scratch array in the library's own device memory.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds it until the process exits.  Host code cannot use the array's
// name as a device address: the first call on each device looks the address up
// with cudaGetSymbolAddress (with that device current) and caches it; later
// calls reuse it.  All calls on a device share the array and it keeps the
// previous call's contents; the only part that must start at zero, the
// per-sequence completion counters, is cleared on the stream before every call.
// Calls whose work overlaps on the GPU
// (other streams, other threads) race on the array and must be serialised by
// the caller.
#include <mutex>

#include "kpa_internal.cuh"

static __device__ __align__(256) unsigned char g_noalloc_scratch[KPA_DECODE_NOALLOC_MAX_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch[kMaxDevices];

// Device address of the scratch array on the current device (looked up once).
kpa_status scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        kpa::record_cuda_error(e);
        return KPA_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return KPA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) {
            kpa::record_cuda_error(e);
            return KPA_ERR_CUDA;
        }
        g_scratch[dev] = p;
    }
    *out = g_scratch[dev];
    return KPA_OK;
}

}  // namespace

extern "C" kpa_status kpa_decode_noalloc(const kpa_config *cfg, int32_t batch, const void *q,
                                         const int32_t *q_pos, const void *kcache,
                                         const void *vcache, int32_t capacity,
                                         const int32_t *seq_len, int32_t max_len, float sm_scale,
                                         float *out, kpa_stream stream) {
    if (batch < 0 || max_len < 0) return KPA_ERR_INVALID_ARG;
    // the workspace of this (dense-query) decode, and where its counters sit in it
    size_t need = 0, off = 0, count_bytes = 0;
    kpa_status s = kpa::decode_dense_plan(cfg, batch, max_len, &need, &off, &count_bytes);
    if (s != KPA_OK) return s;
    if (need > (size_t)KPA_DECODE_NOALLOC_MAX_BYTES) return KPA_ERR_WORKSPACE;
    void *scratch = nullptr;
    s = scratch_address(&scratch);
    if (s != KPA_OK) return s;
    // the decode's per-sequence counters must start at zero; an earlier call that
    // stopped on a device error may have left them set
    if (batch > 0 && count_bytes > 0) {
        cudaError_t e = cudaMemsetAsync(static_cast<char *>(scratch) + off, 0, count_bytes,
                                        (cudaStream_t)stream);
        if (e != cudaSuccess) {
            kpa::record_cuda_error(e);
            return KPA_ERR_CUDA;
        }
    }
    return kpa_decode_split(cfg, batch, q, q_pos, kcache, vcache, capacity, seq_len, max_len,
                            sm_scale, 0, out, scratch, (size_t)KPA_DECODE_NOALLOC_MAX_BYTES, stream);
}
