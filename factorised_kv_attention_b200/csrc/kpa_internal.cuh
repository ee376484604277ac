// kpa_internal.cuh -- types and helpers shared by libkpa's kernels and host code.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/kpa.h"

namespace kpa {

// Device-side error codes share the numbering of kpa_status.
constexpr int kErrTimeout = KPA_ERR_TIMEOUT;
constexpr int kErrDeviceCheck = KPA_ERR_DEVICE_CHECK;

constexpr int kGroup = KPA_TOKEN_GROUP;   // tokens per interleaved cache group
constexpr int kMaxHalfD2 = 128;           // RoPE table length (d2 <= 256)

// Shape of one attention layer, with the derived sizes the kernels index by.
struct Dims {
    int h1, h2, d1, d2;
    int rk, rv;
    int h, dh;      // h1*h2, d1*d2
    int ek, ev;     // elements per key / value record
    int shared;     // one B for keys and values: key record [A^K | B] (B unrotated), value record [A^V]
    int order;      // 2: Kronecker form; 3: third-order TPA, record [a | b | c] (h2 = 1, d1 = d_b, d2 = d_c)
};

// theta_m = base^(-2m/n), m < n/2, formed on the host in float64 and passed by
// value (Definition 2.3; the pairing and sign are documented in kpa.h).  n is d2,
// or d_b = d1 for a third-order cache (RoPE on the b factors).
struct RopeTable {
    double theta[kMaxHalfD2];
};

// Records the first device-side error; later ones are dropped.
__device__ __forceinline__ void raise_error(int *err, int code) {
    if (err) atomicCAS(err, 0, code);
}

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
    return __bfloat162float(v);
}
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// Element offset of (slot s, element e) inside one sequence's plane of the
// interleaved cache: group s/8 holds its records element-major, token-minor.
__host__ __device__ __forceinline__ int64_t cache_offset(int64_t s, int e, int E) {
    return ((s / kGroup) * E + e) * kGroup + (s % kGroup);
}

// cos/sin of the angle pos * theta.  The angle is formed and reduced to [-pi, pi]
// in float64 (Cody-Waite reduction: 2 pi split into a double and its remainder, so
// the reduced angle keeps float64 accuracy for any position below 2^31); the float
// sine and cosine of the remainder follow.
__device__ __forceinline__ void rope_cs(double pos, double theta, float &c, float &s) {
    constexpr double kInvTwoPi = 0.15915494309189535;       // 1 / (2 pi)
    constexpr double kTwoPiHi = 6.283185307179586;          // 2 pi rounded to double
    constexpr double kTwoPiLo = 2.4492935982947064e-16;     // 2 pi - kTwoPiHi
    const double phi = pos * theta;
    const double k = rint(phi * kInvTwoPi);
    const double r = fma(-k, kTwoPiLo, fma(-k, kTwoPiHi, phi));
    sincosf((float)r, &s, &c);
}

// The same angle with the hardware sine/cosine approximations on the reduced argument
// r in [-pi, pi] (absolute error a few 1e-7 there): for the decode query, whose
// rotation feeds a bf16-level dot product, at a fraction of the latency.
__device__ __forceinline__ void rope_cs_fast(double pos, double theta, float &c, float &s) {
    constexpr double kInvTwoPi = 0.15915494309189535;
    constexpr double kTwoPiHi = 6.283185307179586;
    constexpr double kTwoPiLo = 2.4492935982947064e-16;
    const double phi = pos * theta;
    const double k = rint(phi * kInvTwoPi);
    const double r = fma(-k, kTwoPiLo, fma(-k, kTwoPiHi, phi));
    __sincosf((float)r, &s, &c);
}

// Raise a kernel's dynamic shared-memory limit once per device and kernel (so
// later calls, including ones made while a stream is being captured, launch
// directly).  The kernel is a template argument: one cache per kernel.
template <auto Kernel>
inline cudaError_t ensure_dynamic_smem(size_t bytes) {
    static std::atomic<int> granted[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (bytes <= 48 * 1024 || (size_t)granted[dev].load() >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) granted[dev].store((int)bytes);
    return e;
}

// Remember a CUDA error for kpa_last_cuda_error (calling thread).
void record_cuda_error(cudaError_t e);

// ---- host-side launchers (one per kernel file) ------------------------------
// pos_offset (nullable, device [batch]): the keys of slot s are rotated at position
// s + pos_offset[b] instead of s
cudaError_t launch_append_factors(const Dims &d, kpa_dtype dt, int batch, int n_tok,
                                  const void *kf, const void *vf, const int32_t *start_pos,
                                  const int32_t *pos_offset, int cap, void *kc, void *vc, const RopeTable &rope,
                                  int *err, cudaStream_t st);

struct DecodePlan {
    int variant;         // tensor-core kernel variant, or -1 for the CUDA-core kernel
    int tokens_per_split;
    int n_split;         // splits per sequence (grid x)
    int tile;            // tokens per shared-memory tile
    int fused;           // the decode kernel merges the splits itself (no combine launch)
    int cluster;         // ... through a thread-block cluster per sequence (DSMEM)
    int engine;          // 1: the tcgen05 kernel (TPA h = 16, d_h = 64, R = 2), 0: mma.sync
    int spec;            // every CTA is resident at once (one wave): the decode copies its first
                         // tiles before it has read the sequence length
    size_t part_o_off, part_ml_off, counters_off, bytes;
};

// Workspace of a decode with a dense query and the automatic split: its size (total)
// and the byte range of its per-sequence counters (they must be zero before a call and
// are zero again after every call that completes).
kpa_status decode_dense_plan(const kpa_config *cfg, int batch, int max_len, size_t *total, size_t *offset,
                             size_t *bytes);

cudaError_t launch_decode_fma(const Dims &d, kpa_dtype dt, int batch, const void *q,
                              const int32_t *q_pos, const void *kc, const void *vc, int cap,
                              const int32_t *seq_len, int max_len, float qscale,
                              const DecodePlan &plan, float *part_o, float *part_ml,
                              const RopeTable &rope, int *err, cudaStream_t st, int sms);

// lse (nullable, [batch][h]): also the natural-log log-sum-exp of each head's scores,
// (M + log2 L) * lse_scale with the partials' base-2 statistics (lse_scale = ln 2)
cudaError_t launch_decode_combine(const Dims &d, int batch, const int32_t *seq_len,
                                  int max_len, const DecodePlan &plan, const float *part_o,
                                  const float *part_ml, float out_scale, float *out,
                                  cudaStream_t st, float *lse = nullptr, float lse_scale = 0.f);

// out[b][h] = sum_p exp(lse_p - LSE) out_p[b][h] over n_parts normalised partial outputs,
// LSE = ln sum_p exp(lse_p); lse_out (nullable) receives LSE
cudaError_t launch_merge_lse(int batch, int heads, int d_h, int n_parts, const float *outs, const float *lses,
                             float *out, float *lse_out, cudaStream_t st);

size_t decode_fma_smem_bytes(const Dims &d, kpa_dtype dt, int tile);

// Third-order TPA decode (CUDA cores): whether it covers these dims, and its launcher
// (unnormalised split partials for launch_decode_combine).
constexpr int kOrder3Tile = 32;
bool order3_decode_supported(const Dims &d, kpa_dtype dt);
int order3_ctas_per_sm(const Dims &d, kpa_dtype dt);
cudaError_t launch_decode_order3(const Dims &d, kpa_dtype dt, int batch, const void *q, const int32_t *q_pos,
                                 const void *kc, const void *vc, int cap, const int32_t *seq_len, int max_len,
                                 float qscale, const DecodePlan &p, float *part_o, float *part_ml,
                                 const RopeTable &rope, int *err, cudaStream_t st);

bool prefill_supported(const Dims &d);
// Query factors for a prefill (ptr null: a dense bf16 query instead).
struct PrefillQf {
    const float *ptr;
    long long stride, seq_stride, tok_stride;   // element, sequence and token strides (floats)
    int rq;
};
constexpr int kPrefillQfMaxRq = 6;
cudaError_t launch_prefill(const Dims &d, int batch, int n_tok, const void *q, const PrefillQf &qf,
                           const int32_t *start_pos, const void *kc, const void *vc, int cap, float qscale,
                           float out_scale, float *out, const RopeTable &rope, int *err,
                           unsigned long long wait_limit_ns, cudaStream_t st);

size_t append_smem_bytes(int BN, int stages, int d2);
int append_tile_n(int N);
cudaError_t launch_append(const Dims &d, int rq, int d_model, int batch, int n_tok, const void *x,
                          const void *w, const int32_t *start_pos, int cap, void *kc, void *vc,
                          void *q_out, float *qf, const RopeTable &rope, int *err,
                          unsigned long long wait_limit_ns, cudaStream_t st);

}  // namespace kpa
