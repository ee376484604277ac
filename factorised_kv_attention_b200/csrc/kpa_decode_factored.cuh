// kpa_decode_factored.cuh -- the factored-score TPA decode from query factors (CUDA cores).
#pragma once

#include "kpa_internal.cuh"

namespace kpa {

// Whether the factored-score decode covers a TPA shape (h2 = 1, d1 = 1, d_h = 64,
// h <= 32, R_Q R_K <= 32, R_K and R_V <= 4) with query rank rq.
bool factored_decode_supported(const Dims &d, int rq);

// CTAs of the kernel that one SM holds at once (occupancy query).
int factored_ctas_per_sm(const Dims &d, int rq);

// Unnormalised split partials (o, m, l) for launch_decode_combine.  qscale is
// sm_scale / (R_Q R_K) * log2(e).
cudaError_t launch_decode_factored(const Dims &d, int rq, int batch, const float *qf, long long qf_stride,
                                   long long qf_seq_stride, const int32_t *q_pos, const void *kc, const void *vc,
                                   int cap, const int32_t *seq_len, int max_len, float qscale, const DecodePlan &p,
                                   float *part_o, float *part_ml, const RopeTable &rope, int *err, cudaStream_t st);

}  // namespace kpa
