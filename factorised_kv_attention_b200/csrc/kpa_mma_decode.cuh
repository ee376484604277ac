// kpa_mma_decode.cuh -- compile-time shapes of the tensor-core decode kernel.
#pragma once

#include "kpa_internal.cuh"

namespace kpa {

// Hooks for the failure-detection tests: the producer of CTA (skip_split, batch 0)
// never issues tile `skip_tile` (a copy that nothing will complete), and every
// bounded wait gives up after wait_limit_ns.  skip_tile < 0 disables the hook.
struct DecodeTestHooks {
    int skip_tile;
    int skip_split;
    unsigned long long wait_limit_ns;
};

// One instantiation per (split, ranks) family.
//   MA = h1*d1 (rows of the per-i2 GEMMs), D1, D2, RK, RV, H2 = h2,
//   SLICES  token slices per CTA (warps = H2 * SLICES),
//   CHUNKS  16-token chunks per warp per stage, STAGES ring depth.
template <int MA_, int D1_, int D2_, int RK_, int RV_, int H2_, int SLICES_, int CHUNKS_, int STAGES_>
struct MmaDecodeCfg {
    static constexpr int MA = MA_, D1 = D1_, D2 = D2_, RK = RK_, RV = RV_, H2 = H2_;
    static constexpr int SLICES = SLICES_, CHUNKS = CHUNKS_, STAGES = STAGES_;
    static constexpr int H1 = MA / D1, H = H1 * H2, DH = D1 * D2;
    static constexpr int EK = RK * (MA + H2 * D2), EV = RV * (MA + H2 * D2);
    static constexpr int WARPS = H2 * SLICES;
    static constexpr int TT = 16 * CHUNKS * SLICES;             // tokens per stage
    static constexpr int STAGE_BYTES = TT * (EK + EV) * 2;
    static constexpr size_t smem_bytes() {
        return (size_t)STAGES * STAGE_BYTES + 16 * STAGES + (size_t)H * DH * 4 + 16;
    }
    static_assert(MA % 16 == 0, "h1*d1 must be a multiple of 16");
    static_assert(D2 % 16 == 0, "d2 must be a multiple of 16");
    static_assert(D1 == 1 || D1 == 2 || D1 == 4 || D1 == 8 || D1 == 16, "d1 must be 1..16, a power of 2");
    static_assert((size_t)SLICES * H * DH * 4 + (size_t)SLICES * H * 8 <= (size_t)STAGES * STAGE_BYTES,
                  "slice merge must fit in the ring");
    static_assert(WARPS <= 31, "too many consumer warps");
    static_assert(smem_bytes() <= 227 * 1024, "shared memory");
};

// TPA, h = 16, d_h = 64, R_K = R_V = 2 (the degenerate split h1 = h, d1 = 1, h2 = 1).
using MmaTpaH16D64R2 = MmaDecodeCfg<16, 1, 64, 2, 2, 1, 8, 1, 2>;
// KPA h = 4x8, d_h = 8x16, R_K = R_V = 4.
using MmaKpaH4x8D8x16R4 = MmaDecodeCfg<32, 8, 16, 4, 4, 8, 1, 2, 2>;
// KPA h = 4x8, d_h = 8x16, R_K = R_V = 2.
using MmaKpaH4x8D8x16R2 = MmaDecodeCfg<32, 8, 16, 2, 2, 8, 1, 4, 2>;
// KPA h = 4x4, d_h = 8x16, R_K = R_V = 2.
using MmaKpaH4x4D8x16R2 = MmaDecodeCfg<32, 8, 16, 2, 2, 4, 2, 2, 2>;

#define KPA_MMA_VARIANTS(X)        \
    X(0, MmaTpaH16D64R2)           \
    X(1, MmaKpaH4x8D8x16R4)        \
    X(2, MmaKpaH4x8D8x16R2)        \
    X(3, MmaKpaH4x4D8x16R2)

// Index of the variant that covers these dims, or -1.
inline int mma_decode_variant(const Dims &d) {
#define KPA_MMA_MATCH(IDX, CFG)                                                            \
    if (d.h1 * d.d1 == CFG::MA && d.d1 == CFG::D1 && d.d2 == CFG::D2 && d.rk == CFG::RK && \
        d.rv == CFG::RV && d.h2 == CFG::H2)                                                \
        return IDX;
    KPA_MMA_VARIANTS(KPA_MMA_MATCH)
#undef KPA_MMA_MATCH
    return -1;
}

inline int mma_decode_tile(int variant) {
#define KPA_MMA_TILE(IDX, CFG) \
    if (variant == IDX) return CFG::TT;
    KPA_MMA_VARIANTS(KPA_MMA_TILE)
#undef KPA_MMA_TILE
    return 0;
}

cudaError_t launch_decode_mma(int variant, int batch, const void *q, const int32_t *q_pos,
                              const void *kc, const void *vc, int cap, const int32_t *seq_len,
                              int max_len, float qscale, const DecodePlan &plan, float *part_o,
                              float *part_ml, const RopeTable &rope, int *err,
                              const DecodeTestHooks &hooks, cudaStream_t st);

}  // namespace kpa
