// kpa_prefill_mma.cuh -- the causal prefill for Kronecker splits that the tcgen05
// prefill is not instantiated for: its shape check and its launcher.
#pragma once

#include "kpa_internal.cuh"

namespace kpa {

// Dynamic shared memory of the mma.sync prefill for these dims (0: not covered,
// i.e. third order or d_h > 128).
size_t prefill_mma_smem_bytes(const Dims &d);
bool prefill_mma_supported(const Dims &d);

// Arguments as launch_prefill (qscale = sm_scale / R_K log2 e, out_scale = 1 / R_V);
// the kernel has no waits, so it takes no wait limit.
cudaError_t launch_prefill_mma(const Dims &d, int batch, int n_tok, const void *q, const PrefillQf &qf,
                               const int32_t *start_pos, const void *kc, const void *vc, int cap,
                               float qscale, float out_scale, float *out, const RopeTable &rope, int *err,
                               cudaStream_t st);

}  // namespace kpa
