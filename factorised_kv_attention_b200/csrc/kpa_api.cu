// kpa_api.cu -- the extern "C" entry points of libkpa: argument checks, split
// planning, workspace layout and launches.  Every check that the host can make
// happens here, before anything is enqueued.
#include <math.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "kpa_decode_factored.cuh"
#include "kpa_internal.cuh"
#include "kpa_mma_decode.cuh"
#include "kpa_prefill_mma.cuh"

namespace kpa {

// Per-device error word (kpa_read_device_error).
__device__ int g_device_error;

namespace {

thread_local int t_last_cuda = 0;

kpa_status cuda_fail(cudaError_t e) {
    t_last_cuda = (int)e;
    return KPA_ERR_CUDA;
}

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int *g_err_ptr[kMaxDevices];
int g_sms[kMaxDevices];

kpa_status device_state(int **err, int *sms) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return KPA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_err_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_device_error);
        if (e != cudaSuccess) return cuda_fail(e);
        int n = 0;
        e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e);
        g_sms[dev] = n;
        g_err_ptr[dev] = static_cast<int *>(p);
    }
    if (err) *err = g_err_ptr[dev];
    if (sms) *sms = g_sms[dev];
    return KPA_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Shape checks shared by every call.  need_q: the query rank is used.
kpa_status check_cfg(const kpa_config *c, bool need_q, bool need_model) {
    if (!c) return KPA_ERR_INVALID_ARG;
    if (c->h1 <= 0 || c->h2 <= 0 || c->d1 <= 0 || c->d2 <= 0) return KPA_ERR_INVALID_ARG;
    if (c->r_k <= 0 || c->r_v <= 0 || c->r_q < 0) return KPA_ERR_INVALID_ARG;
    if (need_q && c->r_q <= 0) return KPA_ERR_INVALID_ARG;
    if (need_model && c->d_model <= 0) return KPA_ERR_INVALID_ARG;
    if (c->dtype != KPA_F32 && c->dtype != KPA_BF16) return KPA_ERR_INVALID_ARG;
    if (!(c->rope_base > 0.0) || !isfinite(c->rope_base)) return KPA_ERR_INVALID_ARG;
    if (c->order != 0 && c->order != 2 && c->order != 3) return KPA_ERR_INVALID_ARG;
    if (c->order == 3) {
        // third-order TPA: heads in a, RoPE pairs on b (d1 = d_b), no shared B
        if (c->h2 != 1 || c->d1 % 2 != 0 || c->shared_b != 0) return KPA_ERR_INVALID_ARG;
        if (c->d1 > 2 * kMaxHalfD2) return KPA_ERR_UNSUPPORTED;
    } else if (c->d2 % 2 != 0) {
        return KPA_ERR_INVALID_ARG;                           // RoPE pairs
    }
    if (c->shared_b != 0 && c->shared_b != 1) return KPA_ERR_INVALID_ARG;
    if (c->shared_b && c->r_k != c->r_v) return KPA_ERR_INVALID_ARG;   // B^K_r = B^V_r
    const int64_t h = (int64_t)c->h1 * c->h2, dh = (int64_t)c->d1 * c->d2;
    if (h > 4096 || dh > 4096) return KPA_ERR_UNSUPPORTED;
    if (c->d2 > 2 * kMaxHalfD2) return KPA_ERR_UNSUPPORTED;
    if (c->r_k > 64 || c->r_v > 64 || c->r_q > 64) return KPA_ERR_UNSUPPORTED;
    return KPA_OK;
}

Dims dims_of(const kpa_config *c) {
    Dims d;
    d.h1 = c->h1; d.h2 = c->h2; d.d1 = c->d1; d.d2 = c->d2;
    d.rk = c->r_k; d.rv = c->r_v;
    d.h = c->h1 * c->h2;
    d.dh = c->d1 * c->d2;
    d.ek = c->r_k * (c->h1 * c->d1 + c->h2 * c->d2);
    d.shared = c->shared_b ? 1 : 0;
    d.ev = d.shared ? c->r_v * c->h1 * c->d1 : c->r_v * (c->h1 * c->d1 + c->h2 * c->d2);
    d.order = c->order == 3 ? 3 : 2;
    if (d.order == 3) {                                       // record [a | b | c]
        d.ek = c->r_k * (c->h1 + c->d1 + c->d2);
        d.ev = c->r_v * (c->h1 + c->d1 + c->d2);
    }
    return d;
}

RopeTable rope_table(const kpa_config *c) {
    RopeTable t;
    const int n = c->order == 3 ? c->d1 : c->d2;              // the rotated factor's length
    for (int m = 0; m < kMaxHalfD2; ++m)
        t.theta[m] = m < n / 2 ? pow(c->rope_base, -2.0 * (double)m / (double)n) : 0.0;
    return t;
}

size_t dtype_size(kpa_dtype t) { return t == KPA_BF16 ? 2 : 4; }

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

constexpr size_t kSmemLimit = 200 * 1024;

// Test and measurement switches, scoped to the host thread that sets them (a caller
// that flips them changes only its own later calls, never another thread's).
// The bounded waits give up after 1 s unless a test shortens them.
thread_local DecodeTestHooks t_hooks = {-1, -1, 1000000000ull};

// 0: the default kernels; 1: the tcgen05 TPA decode where it applies; 2: the factored
// score for decodes from query factors on TPA shapes (testing and measurement: both are
// slower than the defaults on the shapes measured so far).
thread_local int t_decode_engine = 0;
thread_local int t_prefill_engine = 0;

DecodeTestHooks current_hooks() { return t_hooks; }

constexpr int kMaxClusterSplits = 16;

// How many clusters of `size` CTAs of a tensor-core variant can be resident at once
// on this device (cached per device).
int cluster_capacity(int variant, int size) {
    constexpr int kMaxVariants = 24;
    static std::atomic<int> known[kMaxDevices][kMaxVariants][kMaxClusterSplits + 1];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices || variant < 0 ||
        variant >= kMaxVariants || size < 1 || size > kMaxClusterSplits)
        return 0;
    int k = known[dev][variant][size].load();
    if (k == 0) {
        k = mma_decode_max_clusters(variant, size);
        known[dev][variant][size].store(k > 0 ? k : -1);
    }
    return k > 0 ? k : 0;
}

// Split plan.  Auto splits aim at one wave of CTAs: ceil(sms * ctas_per_sm / batch)
// pieces per sequence, each a multiple of 16 slots.
// factored_rq > 0: the plan of the factored-score decode from query factors of that rank
// no_fuse: the splits always end in the combine kernel (the call wants its log-sum-exp).
kpa_status plan_decode(const Dims &d, kpa_dtype dt, int batch, int max_len, int tps_req, int sms,
                       DecodePlan *p, int factored_rq = 0, bool no_fuse = false) {
    if (tps_req < 0 || (tps_req > 0 && tps_req % 64 != 0)) return KPA_ERR_INVALID_ARG;
    p->variant = dt == KPA_BF16 && factored_rq == 0 ? mma_decode_variant(d) : -1;
    if (d.shared && p->variant < 0) return KPA_ERR_UNSUPPORTED;   // shared B: tensor-core variants only
    int ctas_per_sm = 2;
    if (factored_rq > 0) {
        if (!factored_decode_supported(d, factored_rq)) return KPA_ERR_UNSUPPORTED;
        p->tile = 32;
        // latency-bound CUDA-core kernel: every CTA slot the occupancy query allows (up to 4)
        ctas_per_sm = std::min(4, factored_ctas_per_sm(d, factored_rq));
    } else if (p->variant >= 0) {
        p->tile = mma_decode_tile(p->variant);
        const size_t smem = mma_decode_smem(p->variant);
        ctas_per_sm = smem > 0 ? (int)((227 * 1024) / smem) : 1;
        // resident CTAs as the occupancy calculator counts them (registers included)
        const int resident = cluster_capacity(p->variant, 1);
        if (resident > 0 && sms > 0 && resident / sms < ctas_per_sm) ctas_per_sm = resident / sms;
        if (ctas_per_sm < 1) ctas_per_sm = 1;
    } else if (d.order == 3) {
        if (!order3_decode_supported(d, dt)) return KPA_ERR_UNSUPPORTED;
        p->tile = kOrder3Tile;
        // latency-bound CUDA-core kernel: fill every CTA slot the occupancy query allows
        // (up to 4 per SM; more splits only add partials to merge)
        ctas_per_sm = std::min(4, order3_ctas_per_sm(d, dt));
    } else {
        int tile = 32;
        while (tile > 8 && decode_fma_smem_bytes(d, dt, tile) > kSmemLimit) tile /= 2;
        if (decode_fma_smem_bytes(d, dt, tile) > kSmemLimit) return KPA_ERR_UNSUPPORTED;
        if ((d.h * d.dh + 255) / 256 > 32) return KPA_ERR_UNSUPPORTED;
        p->tile = tile;
    }
    const int target = ctas_per_sm * (sms > 0 ? sms : 148);
    const int per_seq = batch > 0 ? (target > batch ? target / batch : 1) : 1;
    // A sequence's splits merge inside one thread-block cluster (over DSMEM) when all
    // the clusters are resident at once and still cover most of the SMs; a cluster of
    // one CTA needs no merge at all.  Otherwise the splits of a sequence are merged
    // through global memory.
    int c = p->variant >= 0 ? (per_seq < kMaxClusterSplits ? per_seq : kMaxClusterSplits) : 0;
    while (c > 1 && cluster_capacity(p->variant, c) < batch) --c;
    // Several sequences may have different lengths (the host does not see them): up to
    // 4 waves of shorter splits let the CTA scheduler balance the long ones, as long as
    // every split still streams at least 1 MiB of cache.  That takes precedence over a
    // one-wave cluster plan.
    int over_split = 0;
    if (batch > 1 && tps_req == 0) {
        const int64_t bytes_tok = (int64_t)(d.ek + d.ev) * (dt == KPA_BF16 ? 2 : 4);
        const int64_t tps_min = ((int64_t)1 << 20) / bytes_tok;
        for (int k = 4; k > 1 && !over_split; --k) {
            const int64_t cand = ((int64_t)max_len + (int64_t)k * per_seq - 1) / ((int64_t)k * per_seq);
            if (cand >= tps_min) over_split = k * per_seq;
        }
    }
    const bool cluster_auto =
        !over_split && (c == 1 || (c > 1 && (int64_t)batch * c * 5 >= (int64_t)target * 4));
    int tps = tps_req;
    if (tps == 0) {
        const int want_split = over_split ? over_split : cluster_auto ? c : per_seq;
        const int64_t want = ((int64_t)max_len + want_split - 1) / want_split;
        tps = (int)(((want + 15) / 16) * 16);
        // the generic CUDA-core kernel walks its split tile by tile through latency
        // chains, so a short sequence goes faster over more SMs: splits down to 16 slots
        const int tps_floor = p->variant < 0 && d.order != 3 && factored_rq == 0 ? 16 : 64;
        if (tps < tps_floor) tps = tps_floor;
        // whole tiles per split (no ragged last tile) when that keeps most of the splits
        if (p->variant >= 0 && p->tile > 0) {
            const int whole = (tps + p->tile - 1) / p->tile * p->tile;
            const int64_t n0 = ((int64_t)max_len + tps - 1) / tps;
            const int64_t n1 = ((int64_t)max_len + whole - 1) / whole;
            if (n1 * 20 >= n0 * 17) tps = whole;
        }
    }
    p->tokens_per_split = tps;
    p->n_split = max_len > 0 ? (int)(((int64_t)max_len + tps - 1) / tps) : 1;
    // the last split runs to the end of its sequence: a remainder of at most a quarter of a
    // split joins the split before it instead of becoming a split (and a partial) of its own
    if (p->n_split > 1 && (int64_t)max_len - (int64_t)(p->n_split - 1) * tps <= tps / 4) --p->n_split;
    // the tcgen05 kernel, on request, for TPA at h = 16, d_h = 64, R = 2 (its splits merge
    // through global memory)
    p->engine = p->variant >= 0 && p->tile == 128 && tc_decode_supported(d) && t_decode_engine == 1;
    p->cluster = !p->engine && p->variant >= 0 && p->n_split <= kMaxClusterSplits &&
                 (p->n_split == 1 || cluster_capacity(p->variant, p->n_split) >= batch);
    // otherwise the last CTA of a sequence merges its splits when that read is small
    // In a grid of one wave the first tile's latency is on every CTA's critical path, so
    // the kernel requests it before reading the length (a split past a sequence's end then
    // copies one tile for nothing).  In several waves the later CTAs' latency overlaps the
    // running ones, and the copies of empty splits would only add DRAM traffic.
    p->spec = (int64_t)batch * p->n_split <= (int64_t)target;
    if (no_fuse) p->cluster = 0;
    p->fused = !no_fuse && (p->cluster ||
                            (p->variant >= 0 && (size_t)p->n_split * d.h * d.dh * sizeof(float) <= 256 * 1024));
    const size_t o_bytes = (size_t)batch * p->n_split * d.h * d.dh * sizeof(float);
    const size_t ml_bytes = (size_t)batch * p->n_split * d.h * 2 * sizeof(float);
    p->part_o_off = 0;
    p->part_ml_off = align256(o_bytes);
    p->counters_off = p->part_ml_off + align256(ml_bytes);
    p->bytes = p->counters_off + align256((size_t)batch * sizeof(int));
    return KPA_OK;
}

}  // namespace

void record_cuda_error(cudaError_t e) { t_last_cuda = (int)e; }

kpa_status decode_dense_plan(const kpa_config *cfg, int batch, int max_len, size_t *total, size_t *offset,
                             size_t *bytes) {
    kpa_status s = check_cfg(cfg, false, false);
    if (s != KPA_OK) return s;
    int sms = 0;
    s = device_state(nullptr, &sms);
    if (s != KPA_OK) return s;
    DecodePlan p;
    s = plan_decode(dims_of(cfg), cfg->dtype, batch, max_len, 0, sms, &p);
    if (s != KPA_OK) return s;
    *total = batch == 0 ? 0 : p.bytes;
    *offset = p.counters_off;
    *bytes = (size_t)batch * sizeof(int);
    return KPA_OK;
}

}  // namespace kpa

using namespace kpa;

extern "C" {

const char *kpa_status_string(kpa_status s) {
    switch (s) {
        case KPA_OK: return "KPA_OK";
        case KPA_ERR_INVALID_ARG: return "KPA_ERR_INVALID_ARG: invalid argument";
        case KPA_ERR_UNSUPPORTED: return "KPA_ERR_UNSUPPORTED: shape or dtype not covered";
        case KPA_ERR_WORKSPACE: return "KPA_ERR_WORKSPACE: workspace missing or too small";
        case KPA_ERR_CUDA: return "KPA_ERR_CUDA: a CUDA call failed";
        case KPA_ERR_TIMEOUT: return "KPA_ERR_TIMEOUT: a bounded device wait ran out";
        case KPA_ERR_DEVICE_CHECK: return "KPA_ERR_DEVICE_CHECK: a device-side index check failed";
    }
    return "unknown kpa_status";
}

int kpa_last_cuda_error(void) { return t_last_cuda; }

kpa_status kpa_cache_bytes_per_token(const kpa_config *cfg, size_t *k_bytes, size_t *v_bytes) {
    kpa_status s = check_cfg(cfg, false, false);
    if (s != KPA_OK) return s;
    const Dims d = dims_of(cfg);
    if (k_bytes) *k_bytes = (size_t)d.ek * dtype_size(cfg->dtype);
    if (v_bytes) *v_bytes = (size_t)d.ev * dtype_size(cfg->dtype);
    return KPA_OK;
}

}  // extern "C"

namespace kpa {
namespace {

kpa_status append_factors_impl(const kpa_config *cfg, int32_t batch, int32_t n_tok, const void *k_factors,
                               const void *v_factors, const int32_t *start_pos, const int32_t *pos_offset,
                               int32_t capacity, void *kcache, void *vcache, kpa_stream stream) {
    kpa_status s = check_cfg(cfg, false, false);
    if (s != KPA_OK) return s;
    if (batch < 0 || n_tok < 0) return KPA_ERR_INVALID_ARG;
    if (capacity <= 0 || capacity % KPA_TOKEN_GROUP != 0) return KPA_ERR_INVALID_ARG;
    // a shared B is rotated in the decode at the slot's own position
    if (pos_offset && cfg->shared_b) return KPA_ERR_UNSUPPORTED;
    if (batch == 0 || n_tok == 0) return KPA_OK;
    if (!k_factors || !v_factors || !start_pos || !kcache || !vcache) return KPA_ERR_INVALID_ARG;
    if (!aligned16(kcache) || !aligned16(vcache) || !aligned16(k_factors) || !aligned16(v_factors) ||
        (reinterpret_cast<uintptr_t>(start_pos) & 3) || (reinterpret_cast<uintptr_t>(pos_offset) & 3))
        return KPA_ERR_INVALID_ARG;
    if ((int64_t)n_tok / KPA_TOKEN_GROUP + 2 > INT32_MAX || batch > 65535) return KPA_ERR_UNSUPPORTED;
    int *err = nullptr;
    s = device_state(&err, nullptr);
    if (s != KPA_OK) return s;
    const Dims d = dims_of(cfg);
    cudaError_t e = launch_append_factors(d, cfg->dtype, batch, n_tok, k_factors, v_factors, start_pos, pos_offset,
                                          capacity, kcache, vcache, rope_table(cfg), err, (cudaStream_t)stream);
    return e == cudaSuccess ? KPA_OK : cuda_fail(e);
}

}  // namespace
}  // namespace kpa

extern "C" {

kpa_status kpa_append_factors(const kpa_config *cfg, int32_t batch, int32_t n_tok,
                              const void *k_factors, const void *v_factors,
                              const int32_t *start_pos, int32_t capacity, void *kcache,
                              void *vcache, kpa_stream stream) {
    return append_factors_impl(cfg, batch, n_tok, k_factors, v_factors, start_pos, nullptr, capacity, kcache,
                               vcache, stream);
}

kpa_status kpa_append_factors_pos(const kpa_config *cfg, int32_t batch, int32_t n_tok, const void *k_factors,
                                  const void *v_factors, const int32_t *start_pos, const int32_t *pos_offset,
                                  int32_t capacity, void *kcache, void *vcache, kpa_stream stream) {
    if (!pos_offset && batch > 0 && n_tok > 0) return KPA_ERR_INVALID_ARG;
    return append_factors_impl(cfg, batch, n_tok, k_factors, v_factors, start_pos, pos_offset, capacity, kcache,
                               vcache, stream);
}

kpa_status kpa_decode_workspace_size(const kpa_config *cfg, int32_t batch, int32_t max_len,
                                     int32_t tokens_per_split, size_t *bytes) {
    kpa_status s = check_cfg(cfg, false, false);
    if (s != KPA_OK) return s;
    if (!bytes || batch < 0 || max_len < 0) return KPA_ERR_INVALID_ARG;
    int sms = 0;
    s = device_state(nullptr, &sms);
    if (s != KPA_OK) return s;
    DecodePlan p;
    s = plan_decode(dims_of(cfg), cfg->dtype, batch, max_len, tokens_per_split, sms, &p);
    if (s != KPA_OK) return s;
    size_t need = p.bytes;
    // with the factored-score engine selected, room for its plan too
    if (t_decode_engine == 2 && cfg->dtype == KPA_BF16 && factored_decode_supported(dims_of(cfg), cfg->r_q)) {
        DecodePlan pf;
        if (plan_decode(dims_of(cfg), cfg->dtype, batch, max_len, tokens_per_split, sms, &pf, cfg->r_q) == KPA_OK)
            need = std::max(need, pf.bytes);
    }
    *bytes = batch == 0 ? 0 : need;
    return KPA_OK;
}

kpa_status kpa_decode_plan(const kpa_config *cfg, int32_t batch, int32_t max_len,
                           int32_t tokens_per_split, int32_t *n_split, int32_t *tokens_per_split_out,
                           int32_t *launches) {
    kpa_status s = check_cfg(cfg, false, false);
    if (s != KPA_OK) return s;
    if (batch < 0 || max_len < 0) return KPA_ERR_INVALID_ARG;
    int sms = 0;
    s = device_state(nullptr, &sms);
    if (s != KPA_OK) return s;
    DecodePlan p;
    s = plan_decode(dims_of(cfg), cfg->dtype, batch, max_len, tokens_per_split, sms, &p);
    if (s != KPA_OK) return s;
    if (n_split) *n_split = p.n_split;
    if (tokens_per_split_out) *tokens_per_split_out = p.tokens_per_split;
    if (launches) *launches = batch == 0 ? 0 : (max_len > 0 && !p.fused ? 2 : 1);
    return KPA_OK;
}

kpa_status kpa_decode_kernel_kind(const kpa_config *cfg, int32_t batch, int32_t max_len,
                                  int32_t tokens_per_split, int32_t *kind) {
    if (!kind) return KPA_ERR_INVALID_ARG;
    kpa_status s = check_cfg(cfg, false, false);
    if (s != KPA_OK) return s;
    if (batch < 0 || max_len < 0) return KPA_ERR_INVALID_ARG;
    int sms = 0;
    s = device_state(nullptr, &sms);
    if (s != KPA_OK) return s;
    DecodePlan p;
    s = plan_decode(dims_of(cfg), cfg->dtype, batch, max_len, tokens_per_split, sms, &p);
    if (s != KPA_OK) return s;
    *kind = p.variant < 0 ? KPA_DECODE_KERNEL_CUDA_CORES
                          : (p.engine ? KPA_DECODE_KERNEL_TCGEN05 : KPA_DECODE_KERNEL_MMA_SYNC);
    return KPA_OK;
}

}  // extern "C"

namespace kpa {
namespace {

// Shared body of the decode entry points: the query is either dense (q) or given as
// factors (qf with strides; only the tensor-core variants take it).
kpa_status decode_impl(const kpa_config *cfg, int32_t batch, const void *q, const float *qf, int32_t qf_stride,
                       int32_t qf_seq_stride, const int32_t *q_pos, const void *kcache, const void *vcache,
                       int32_t capacity, const int32_t *seq_len, int32_t max_len, float sm_scale,
                       int32_t tokens_per_split, float *out, void *workspace, size_t ws_bytes, kpa_stream stream,
                       float *lse = nullptr) {
    kpa_status s = check_cfg(cfg, false, false);
    if (s != KPA_OK) return s;
    if (batch < 0 || max_len < 0) return KPA_ERR_INVALID_ARG;
    if (capacity <= 0 || capacity % KPA_TOKEN_GROUP != 0 || max_len > capacity)
        return KPA_ERR_INVALID_ARG;
    if (!isfinite(sm_scale)) return KPA_ERR_INVALID_ARG;
    if (qf && (cfg->r_q <= 0 || qf_stride <= 0 || qf_seq_stride < 0)) return KPA_ERR_INVALID_ARG;
    if (batch == 0) return KPA_OK;
    if (batch > 65535) return KPA_ERR_UNSUPPORTED;
    if ((!q && !qf) || !kcache || !vcache || !seq_len || !out) return KPA_ERR_INVALID_ARG;
    if ((q && !aligned16(q)) || (qf && (reinterpret_cast<uintptr_t>(qf) & 3)) || !aligned16(kcache) ||
        !aligned16(vcache) || !aligned16(out) || (reinterpret_cast<uintptr_t>(seq_len) & 3) ||
        (reinterpret_cast<uintptr_t>(q_pos) & 3) || (reinterpret_cast<uintptr_t>(lse) & 3))
        return KPA_ERR_INVALID_ARG;
    int *err = nullptr, sms = 0;
    s = device_state(&err, &sms);
    if (s != KPA_OK) return s;
    const Dims d = dims_of(cfg);
    if (lse && d.shared) return KPA_ERR_UNSUPPORTED;              // (its keys rotate at the slot)
    DecodePlan p;
    s = plan_decode(d, cfg->dtype, batch, max_len, tokens_per_split, sms, &p, 0, lse != nullptr);
    if (s != KPA_OK) return s;
    // query factors: the factored score on request (TPA shapes), else the tensor-core
    // kernel, which assembles the query (never a third-order cache)
    const bool factored = qf && t_decode_engine == 2 && cfg->dtype == KPA_BF16 &&
                          factored_decode_supported(d, cfg->r_q);
    if (qf && (d.order == 3 || (!factored && p.variant < 0))) return KPA_ERR_UNSUPPORTED;
    if (qf && !factored && (int64_t)cfg->r_q * (d.h1 * d.d1 + d.h2 * d.d2) > mma_decode_qf_max(p.variant))
        return KPA_ERR_UNSUPPORTED;                               // staged in the kernel's query rows
    if (!workspace || ws_bytes < p.bytes) return KPA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return KPA_ERR_INVALID_ARG;
    if (p.n_split > 65535 * 16) return KPA_ERR_UNSUPPORTED;

    float *part_o = reinterpret_cast<float *>(static_cast<char *>(workspace) + p.part_o_off);
    float *part_ml = reinterpret_cast<float *>(static_cast<char *>(workspace) + p.part_ml_off);
    const float qscale = (float)((double)sm_scale / (double)d.rk * 1.4426950408889634);
    cudaStream_t st = (cudaStream_t)stream;
    int *counters = reinterpret_cast<int *>(static_cast<char *>(workspace) + p.counters_off);
    const float out_scale = (float)(1.0 / (double)d.rv);
    cudaError_t e = cudaSuccess;
    if (max_len > 0 && factored) {
        DecodePlan pf;
        s = plan_decode(d, cfg->dtype, batch, max_len, tokens_per_split, sms, &pf, cfg->r_q);
        if (s != KPA_OK) return s;
        if (ws_bytes < pf.bytes) return KPA_ERR_WORKSPACE;
        float *fo = reinterpret_cast<float *>(static_cast<char *>(workspace) + pf.part_o_off);
        float *fml = reinterpret_cast<float *>(static_cast<char *>(workspace) + pf.part_ml_off);
        const float fscale = (float)((double)sm_scale / ((double)cfg->r_q * d.rk) * 1.4426950408889634);
        e = launch_decode_factored(d, cfg->r_q, batch, qf, qf_stride, qf_seq_stride, q_pos, kcache, vcache, capacity,
                                   seq_len, max_len, fscale, pf, fo, fml, rope_table(cfg), err, st);
        if (e != cudaSuccess) return cuda_fail(e);
        e = launch_decode_combine(d, batch, seq_len, max_len, pf, fo, fml, out_scale, out, st);
        return e == cudaSuccess ? KPA_OK : cuda_fail(e);
    }
    if (max_len > 0 && p.variant >= 0) {
        DecodeArgs args;
        args.q = static_cast<const __nv_bfloat16 *>(q);
        args.q_pos = q_pos;
        args.kc = static_cast<const __nv_bfloat16 *>(kcache);
        args.vc = static_cast<const __nv_bfloat16 *>(vcache);
        args.cap = capacity;
        args.seq_len = seq_len;
        args.max_len = max_len;
        args.qscale = qscale;
        args.tps = p.tokens_per_split;
        args.n_split = p.n_split;
        args.part_o = part_o;
        args.part_ml = part_ml;
        args.counters = counters;
        args.out = out;
        args.out_scale = out_scale;
        args.fused = p.fused;
        args.cluster = p.cluster;
        args.spec = p.spec;
        args.err = err;
        args.qf = qf;
        args.qf_stride = qf_stride;
        args.qf_seq_stride = qf_seq_stride;
        args.rq = cfg->r_q;
        if (p.engine && !qf)
            e = launch_decode_tc(args, batch, p, rope_table(cfg), current_hooks(), st);
        else
            e = launch_decode_mma(p.variant, args, batch, p, rope_table(cfg), current_hooks(), st);
    } else if (max_len > 0 && d.order == 3) {
        e = launch_decode_order3(d, cfg->dtype, batch, q, q_pos, kcache, vcache, capacity, seq_len, max_len,
                                 qscale, p, part_o, part_ml, rope_table(cfg), err, st);
    } else if (max_len > 0) {
        e = launch_decode_fma(d, cfg->dtype, batch, q, q_pos, kcache, vcache, capacity, seq_len,
                              max_len, qscale, p, part_o, part_ml, rope_table(cfg), err, st, sms);
    }
    if (e != cudaSuccess) return cuda_fail(e);
    if (max_len > 0 && p.fused) return KPA_OK;
    // the partials' statistics are base 2 (the score scale carries log2 e): ln = log2 * ln 2
    e = launch_decode_combine(d, batch, seq_len, max_len, p, part_o, part_ml, out_scale, out, st, lse,
                              0.6931471805599453f);
    return e == cudaSuccess ? KPA_OK : cuda_fail(e);
}

}  // namespace
}  // namespace kpa

extern "C" {

kpa_status kpa_decode_split(const kpa_config *cfg, int32_t batch, const void *q,
                            const int32_t *q_pos, const void *kcache, const void *vcache,
                            int32_t capacity, const int32_t *seq_len, int32_t max_len,
                            float sm_scale, int32_t tokens_per_split, float *out,
                            void *workspace, size_t ws_bytes, kpa_stream stream) {
    return decode_impl(cfg, batch, q, nullptr, 0, 0, q_pos, kcache, vcache, capacity, seq_len, max_len, sm_scale,
                       tokens_per_split, out, workspace, ws_bytes, stream);
}

kpa_status kpa_decode_qf(const kpa_config *cfg, int32_t batch, const float *q_factors, int32_t qf_stride,
                         int32_t qf_seq_stride, const int32_t *q_pos, const void *kcache, const void *vcache,
                         int32_t capacity, const int32_t *seq_len, int32_t max_len, float sm_scale, float *out,
                         void *workspace, size_t ws_bytes, kpa_stream stream) {
    return decode_impl(cfg, batch, nullptr, q_factors, qf_stride, qf_seq_stride, q_pos, kcache, vcache, capacity,
                       seq_len, max_len, sm_scale, 0, out, workspace, ws_bytes, stream);
}

kpa_status kpa_decode(const kpa_config *cfg, int32_t batch, const void *q, const int32_t *q_pos,
                      const void *kcache, const void *vcache, int32_t capacity,
                      const int32_t *seq_len, int32_t max_len, float sm_scale, float *out,
                      void *workspace, size_t ws_bytes, kpa_stream stream) {
    return kpa_decode_split(cfg, batch, q, q_pos, kcache, vcache, capacity, seq_len, max_len,
                            sm_scale, 0, out, workspace, ws_bytes, stream);
}

kpa_status kpa_decode_lse(const kpa_config *cfg, int32_t batch, const void *q, const int32_t *q_pos,
                          const void *kcache, const void *vcache, int32_t capacity, const int32_t *seq_len,
                          int32_t max_len, float sm_scale, float *out, float *lse, void *workspace, size_t ws_bytes,
                          kpa_stream stream) {
    if (!lse && batch > 0 && cfg) return KPA_ERR_INVALID_ARG;
    return decode_impl(cfg, batch, q, nullptr, 0, 0, q_pos, kcache, vcache, capacity, seq_len, max_len, sm_scale, 0,
                       out, workspace, ws_bytes, stream, lse);
}

kpa_status kpa_merge_lse(int32_t batch, int32_t heads, int32_t d_h, int32_t n_parts, const float *outs,
                         const float *lses, float *out, float *lse, kpa_stream stream) {
    if (batch < 0 || heads < 0 || d_h < 0 || n_parts < 0) return KPA_ERR_INVALID_ARG;
    if ((int64_t)batch * heads == 0 || d_h == 0) return KPA_OK;
    if (n_parts == 0 || !outs || !lses || !out) return KPA_ERR_INVALID_ARG;
    if (d_h > 1024 || heads > 65535 || batch > 65535 || n_parts > 4096) return KPA_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(outs) & 3) || (reinterpret_cast<uintptr_t>(lses) & 3) ||
        (reinterpret_cast<uintptr_t>(out) & 3) || (reinterpret_cast<uintptr_t>(lse) & 3))
        return KPA_ERR_INVALID_ARG;
    cudaError_t e = launch_merge_lse(batch, heads, d_h, n_parts, outs, lses, out, lse, (cudaStream_t)stream);
    return e == cudaSuccess ? KPA_OK : cuda_fail(e);
}

kpa_status kpa_prefill_workspace_size(const kpa_config *cfg, int32_t batch, int32_t n_tok,
                                      size_t *bytes) {
    kpa_status s = check_cfg(cfg, false, false);
    if (s != KPA_OK) return s;
    if (!bytes || batch < 0 || n_tok < 0) return KPA_ERR_INVALID_ARG;
    *bytes = 0;                                  // K/V tiles live on chip only
    return KPA_OK;
}

// Which prefill kernel takes these dims on the calling thread: the tcgen05 kernel
// where it is instantiated (unless the thread chose the mma.sync kernel), else the
// mma.sync kernel where it fits, else -1.
static int prefill_kind(const Dims &d) {
    if (d.order == 3) return -1;
    if (prefill_supported(d) && t_prefill_engine == 0) return KPA_PREFILL_KERNEL_TCGEN05;
    return prefill_mma_supported(d) ? KPA_PREFILL_KERNEL_MMA_SYNC : -1;
}

kpa_status kpa_prefill_kernel_kind(const kpa_config *cfg, int32_t *kind) {
    kpa_status s = check_cfg(cfg, false, false);
    if (s != KPA_OK) return s;
    if (!kind) return KPA_ERR_INVALID_ARG;
    if (cfg->dtype != KPA_BF16) return KPA_ERR_UNSUPPORTED;
    const int k = prefill_kind(dims_of(cfg));
    if (k < 0) return KPA_ERR_UNSUPPORTED;
    *kind = k;
    return KPA_OK;
}

// The prefill with a dense bf16 query (q) or with query factors (qf.ptr).
static kpa_status prefill_impl(const kpa_config *cfg, int32_t batch, int32_t n_tok, const void *q,
                               const PrefillQf &qf, const int32_t *start_pos, const void *kcache,
                               const void *vcache, int32_t capacity, float sm_scale, float *out,
                               kpa_stream stream) {
    kpa_status s = check_cfg(cfg, qf.ptr != nullptr, false);
    if (s != KPA_OK) return s;
    if (batch < 0 || n_tok < 0) return KPA_ERR_INVALID_ARG;
    if (capacity <= 0 || capacity % KPA_TOKEN_GROUP != 0) return KPA_ERR_INVALID_ARG;
    if (!isfinite(sm_scale)) return KPA_ERR_INVALID_ARG;
    if (qf.ptr && (qf.stride <= 0 || qf.seq_stride < 0 || qf.tok_stride < 0)) return KPA_ERR_INVALID_ARG;
    if (cfg->dtype != KPA_BF16 || cfg->order == 3) return KPA_ERR_UNSUPPORTED;
    const Dims d = dims_of(cfg);
    const int kind = prefill_kind(d);
    if (kind < 0) return KPA_ERR_UNSUPPORTED;
    if (qf.ptr && cfg->r_q > kPrefillQfMaxRq) return KPA_ERR_UNSUPPORTED;
    if (batch == 0 || n_tok == 0) return KPA_OK;
    if (batch > 65535 || d.h > 65535 || (int64_t)batch * n_tok > INT32_MAX / 2) return KPA_ERR_UNSUPPORTED;
    if ((!q && !qf.ptr) || !start_pos || !kcache || !vcache || !out) return KPA_ERR_INVALID_ARG;
    if ((q && !aligned16(q)) || (qf.ptr && (reinterpret_cast<uintptr_t>(qf.ptr) & 3)) || !aligned16(kcache) ||
        !aligned16(vcache) || !aligned16(out) || (reinterpret_cast<uintptr_t>(start_pos) & 3))
        return KPA_ERR_INVALID_ARG;
    int *err = nullptr;
    s = device_state(&err, nullptr);
    if (s != KPA_OK) return s;
    const float qscale = (float)((double)sm_scale / (double)d.rk * 1.4426950408889634);
    const float out_scale = (float)(1.0 / (double)d.rv);
    cudaError_t e = kind == KPA_PREFILL_KERNEL_TCGEN05
                        ? launch_prefill(d, batch, n_tok, q, qf, start_pos, kcache, vcache, capacity, qscale,
                                         out_scale, out, rope_table(cfg), err, current_hooks().wait_limit_ns,
                                         (cudaStream_t)stream)
                        : launch_prefill_mma(d, batch, n_tok, q, qf, start_pos, kcache, vcache, capacity, qscale,
                                             out_scale, out, rope_table(cfg), err, (cudaStream_t)stream);
    return e == cudaSuccess ? KPA_OK : cuda_fail(e);
}

kpa_status kpa_prefill(const kpa_config *cfg, int32_t batch, int32_t n_tok, const void *q,
                       const int32_t *start_pos, const void *kcache, const void *vcache,
                       int32_t capacity, float sm_scale, float *out, void *workspace,
                       size_t ws_bytes, kpa_stream stream) {
    (void)workspace;
    (void)ws_bytes;
    const PrefillQf none = {nullptr, 0, 0, 0, 0};
    if (!q && batch > 0 && n_tok > 0 && check_cfg(cfg, false, false) == KPA_OK) return KPA_ERR_INVALID_ARG;
    return prefill_impl(cfg, batch, n_tok, q, none, start_pos, kcache, vcache, capacity, sm_scale, out, stream);
}

kpa_status kpa_prefill_qf(const kpa_config *cfg, int32_t batch, int32_t n_tok, const float *q_factors,
                          int64_t qf_stride, int64_t qf_seq_stride, int64_t qf_tok_stride,
                          const int32_t *start_pos, const void *kcache, const void *vcache,
                          int32_t capacity, float sm_scale, float *out, void *workspace, size_t ws_bytes,
                          kpa_stream stream) {
    (void)workspace;
    (void)ws_bytes;
    if (!cfg) return KPA_ERR_INVALID_ARG;
    if (!q_factors && batch > 0 && n_tok > 0) return KPA_ERR_INVALID_ARG;
    const PrefillQf qf = {q_factors, qf_stride, qf_seq_stride, qf_tok_stride, cfg->r_q};
    return prefill_impl(cfg, batch, n_tok, nullptr, qf, start_pos, kcache, vcache, capacity, sm_scale, out,
                        stream);
}

kpa_status kpa_append_workspace_size(const kpa_config *cfg, int32_t batch, int32_t n_tok,
                                     size_t *bytes) {
    kpa_status s = check_cfg(cfg, true, true);
    if (s != KPA_OK) return s;
    if (cfg->order == 3) return KPA_ERR_UNSUPPORTED;             // the merged projection: Kronecker form
    if (!bytes || batch < 0 || n_tok < 0) return KPA_ERR_INVALID_ARG;
    const int64_t eq = (int64_t)cfg->r_q * (cfg->h1 * cfg->d1 + cfg->h2 * cfg->d2);
    *bytes = align256((size_t)eq * batch * n_tok * sizeof(float));
    return KPA_OK;
}

kpa_status kpa_append(const kpa_config *cfg, int32_t batch, int32_t n_tok, const void *x,
                      const void *w, const int32_t *start_pos, int32_t capacity, void *kcache,
                      void *vcache, void *q_out, void *workspace, size_t ws_bytes,
                      kpa_stream stream) {
    kpa_status s = check_cfg(cfg, true, true);
    if (s != KPA_OK) return s;
    if (batch < 0 || n_tok < 0) return KPA_ERR_INVALID_ARG;
    if (capacity <= 0 || capacity % KPA_TOKEN_GROUP != 0) return KPA_ERR_INVALID_ARG;
    if (cfg->dtype != KPA_BF16 || cfg->order == 3) return KPA_ERR_UNSUPPORTED;
    // TMA rows of x and W are d_model bf16 values: a multiple of 16 bytes
    if (cfg->d_model % 8 != 0) return KPA_ERR_UNSUPPORTED;
    // factor pairs (2m, 2m+1) of B must start on even columns of the projection
    if ((cfg->h1 * cfg->d1) % 2 != 0 && (cfg->r_q % 2 != 0 || cfg->r_k % 2 != 0 || cfg->r_v % 2 != 0))
        return KPA_ERR_UNSUPPORTED;
    if (batch == 0 || n_tok == 0) return KPA_OK;
    if ((int64_t)batch * n_tok > INT32_MAX / 2) return KPA_ERR_UNSUPPORTED;
    if (!x || !w || !start_pos || !kcache || !vcache) return KPA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w) || !aligned16(kcache) || !aligned16(vcache) ||
        !aligned16(q_out) || (reinterpret_cast<uintptr_t>(start_pos) & 3))
        return KPA_ERR_INVALID_ARG;
    const Dims d = dims_of(cfg);
    const size_t smem = append_smem_bytes(append_tile_n(cfg->r_q * (d.h1 * d.d1 + d.h2 * d.d2) + d.ek + d.ev),
                                          2, d.d2);
    if (smem > 227 * 1024) return KPA_ERR_UNSUPPORTED;
    size_t need = 0;
    s = kpa_append_workspace_size(cfg, batch, n_tok, &need);
    if (s != KPA_OK) return s;
    if ((q_out || workspace) && (!workspace || ws_bytes < need)) return KPA_ERR_WORKSPACE;
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255)) return KPA_ERR_INVALID_ARG;
    int *err = nullptr;
    s = device_state(&err, nullptr);
    if (s != KPA_OK) return s;
    cudaError_t e = launch_append(d, cfg->r_q, cfg->d_model, batch, n_tok, x, w, start_pos, capacity,
                                  kcache, vcache, q_out, static_cast<float *>(workspace), rope_table(cfg),
                                  err, current_hooks().wait_limit_ns, (cudaStream_t)stream);
    return e == cudaSuccess ? KPA_OK : cuda_fail(e);
}

kpa_status kpa_test_set_decode_hooks(int32_t skip_tile, int32_t skip_split,
                                     uint64_t wait_limit_ns) {
    if (wait_limit_ns == 0) return KPA_ERR_INVALID_ARG;
    t_hooks.skip_tile = skip_tile;
    t_hooks.skip_split = skip_split;
    t_hooks.wait_limit_ns = wait_limit_ns;
    return KPA_OK;
}

kpa_status kpa_test_set_prefill_engine(int32_t engine) {
    if (engine < 0 || engine > 1) return KPA_ERR_INVALID_ARG;
    t_prefill_engine = engine;
    return KPA_OK;
}

kpa_status kpa_test_set_decode_engine(int32_t engine) {
    if (engine < 0 || engine > 2) return KPA_ERR_INVALID_ARG;
    t_decode_engine = engine;
    return KPA_OK;
}

kpa_status kpa_read_device_error(kpa_stream stream, int32_t *code) {
    if (!code) return KPA_ERR_INVALID_ARG;
    int *err = nullptr;
    kpa_status s = device_state(&err, nullptr);
    if (s != KPA_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    int host = 0;
    cudaError_t e = cudaMemcpyAsync(&host, err, sizeof(int), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(err, 0, sizeof(int), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e);
    *code = host;
    return KPA_OK;
}

}  // extern "C"
