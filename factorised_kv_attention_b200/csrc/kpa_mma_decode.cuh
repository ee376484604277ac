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

// Arguments of one decode launch (device pointers into the caller's buffers).
struct DecodeArgs {
    const __nv_bfloat16 *q;
    const int32_t *q_pos;
    const __nv_bfloat16 *kc, *vc;
    int cap;
    const int32_t *seq_len;
    int max_len;
    float qscale;       // sm_scale / R_K * log2(e)
    int tps;            // slots per split
    int n_split;        // splits per sequence (grid x)
    float *part_o, *part_ml;
    int *counters;      // [batch] finished splits, zero between calls
    float *out;
    float out_scale;    // 1 / R_V
    int fused;          // the last CTA of a sequence combines its splits
    int cluster;        // the splits of a sequence form one cluster and merge over DSMEM
    int spec;           // the grid is one wave: hint and copy the first tiles before the
                        // sequence length is read (else only slots below the length)
    int *err;
    // query factors instead of q (null: use q): element e of sequence b's record
    // [A^Q_0..A^Q_{rq-1} | B^Q_0..B^Q_{rq-1}] at qf[e * qf_stride + b * qf_seq_stride]
    const float *qf;
    int qf_stride, qf_seq_stride, rq;
};

// One instantiation per (split, ranks) family.
//   MA = h1*d1 (rows of the per-i2 GEMMs), D1, D2, RK, RV, H2 = h2,
//   SLICES  token slices per CTA (warps = H2 * SLICES),
//   CHUNKS  16-token chunks per warp per stage, STAGES ring depth,
//   SHARED  one B for keys and values: key record [A^K | B] (B unrotated, rotated in
//           the kernel for the score), value record [A^V].
//   DB      > 0: a third-order TPA cache (h = MA heads, d1 = 1, d2 = d_h = DB * DC):
//           records [a | b | c] with b in R^DB, c in R^DC, and the keys' features
//           b (x) c formed in registers as fp16 for both products.
//   HS      warps that split the CTA's 16-row head tiles between them (d1 = 1, h2 = 1):
//           warps = HS * SLICES, each with MA / 16 / HS tiles of its token slice.
//   MR      > 0: the records' A parts have MR = h1 d1 rows, padded to MA (a multiple of
//           16) in the tiles (d1 = 1, h2 = 1): the padded query rows are zero, their
//           outputs are never written, and the partials and outputs keep MR heads.
template <int MA_, int D1_, int D2_, int RK_, int RV_, int H2_, int SLICES_, int CHUNKS_, int STAGES_,
          bool SHARED_ = false, int DB_ = 0, int HS_ = 1, int MR_ = 0>
struct MmaDecodeCfg {
    static constexpr int MA = MA_, D1 = D1_, D2 = D2_, RK = RK_, RV = RV_, H2 = H2_;
    static constexpr int HS = HS_, MR = MR_ > 0 ? MR_ : MA_;
    static constexpr int SLICES = SLICES_, CHUNKS = CHUNKS_, STAGES = STAGES_;
    static constexpr bool SHARED = SHARED_;
    static constexpr bool ORDER3 = DB_ > 0;
    static constexpr int DB = ORDER3 ? DB_ : 1, DC = ORDER3 ? D2_ / DB : D2_;
    static constexpr int H1 = MA / D1, H = H1 * H2, DH = D1 * D2;
    static constexpr int HR1 = MR / D1, HR = HR1 * H2;           // the cache's heads (H: padded)
    static constexpr int EK = ORDER3 ? RK * (MA + DB + DC) : RK * (MR + H2 * D2);
    static constexpr int EV = ORDER3 ? RV * (MA + DB + DC) : SHARED ? RV * MR : RV * (MR + H2 * D2);
    // d1 = 8 (no shared B, second order): the rows of each 16-row query tile pair up
    // two j1 of one head per lane, so the sum over j1 and the softmax stay in registers,
    // and the value product runs once in fp16 (P' = p A^V and B^V rounded to fp16)
    static constexpr bool KPA8 = D1 == 8 && !SHARED && !ORDER3;
    static constexpr int WARPS = H2 * SLICES * HS;
    // A warp of its own streams the tiles, or (KPA8) the last consumer warp to release a
    // stage issues its next tile: sixteen consumer warps then keep 128 registers each
    // (a seventeenth warp would put five warps, at most 96 registers each, on one SM
    // sub-partition).
    static constexpr bool PRODUCER_WARP = !KPA8;
    static constexpr int THREADS = (WARPS + (PRODUCER_WARP ? 1 : 0)) * 32;
    static constexpr int TT = 16 * CHUNKS * SLICES;             // tokens per stage
    static constexpr int STAGE_BYTES = TT * (EK + EV) * 2;
    // per-warp scratch for the sum over j1 (d1 > 1): [16 tokens][MA + 4] partials,
    // [h1][16] weights, [h1] rescale factors
    static constexpr int RED_LD = MA + 4;
    static constexpr int PPL = D1 > 1 ? (H1 * 16) / 32 : 0;      // (head, token) pairs per lane
    static constexpr int SCR_FLOATS = D1 > 1 && !KPA8 ? ((16 * RED_LD + H1 * 16 + H1 + 3) / 4) * 4 : 0;
    static constexpr size_t OFF_BARS = (size_t)STAGES * STAGE_BYTES;
    static constexpr size_t OFF_Q = OFF_BARS + 16 * STAGES;
    static constexpr int Q_LD = D1 * D2 + 8;                    // padded row of the fp32 query
    // most query-factor values (E_Q) a decode from query factors takes: staged in the
    // query rows, eight per consumer thread
    static constexpr int QF_MAX = 8 * WARPS * 32 < H * Q_LD ? 8 * WARPS * 32 : (H * Q_LD) / (WARPS * 32) * (WARPS * 32);
    static constexpr size_t OFF_CS = OFF_Q + (size_t)H * Q_LD * 4;
    static constexpr size_t OFF_SCR = (OFF_CS + (size_t)(D2 / 2) * 8 + 15) / 16 * 16;
    static constexpr size_t OFF_FLAGS = OFF_SCR + (size_t)WARPS * SCR_FLOATS * 4;
    // shared B: theta_m (fp64), (cos, sin)(k theta_m) for the 16 token offsets k of a
    // chunk, and per warp (cos, sin)(p0 theta_m) at its chunk's first position p0
    // flags: [0] abort, [1] last CTA, [2] tiles issued, [4 + s] releases of stage s
    static constexpr size_t OFF_THETA = OFF_FLAGS + 64;
    static constexpr size_t OFF_STEP = OFF_THETA + (SHARED ? (size_t)(D2 / 2) * 8 : 0);
    static constexpr size_t OFF_BASE = OFF_STEP + (SHARED ? (size_t)16 * (D2 / 2) * 8 : 0);
    static constexpr size_t smem_bytes() { return OFF_BASE + (SHARED ? (size_t)WARPS * (D2 / 2) * 8 : 0); }
    // row stride (floats) of the slice-merge buffer: 8 floats of padding put the rows
    // of consecutive heads in different banks
    static constexpr int MO_LD = D1 * D2 + 8;
    static_assert(MA % 16 == 0, "h1*d1 (padded) must be a multiple of 16");
    static_assert(MR <= MA && MR > MA - 16, "MR pads to MA within one 16-row tile");
    static_assert((MR == MA && HS == 1) || (D1 == 1 && H2 == 1 && !SHARED && !ORDER3),
                  "padded rows and split head tiles: second-order TPA splits without a shared B");
    static_assert((MA / 16) % HS == 0, "head tiles split evenly between the warps");
    static_assert(D2 % 16 == 0 || (KPA8 && D2 == 8), "d2 must be a multiple of 16 (or 8 with d1 = 8)");
    static_assert(D1 == 1 || D1 == 2 || D1 == 4 || D1 == 8 || D1 == 16, "d1 must be 1..16, a power of 2");
    static_assert(D1 == 1 || KPA8 || (H1 >= 2 && 32 % H1 == 0), "h1 must divide 32 when 1 < d1 < 8");
    static_assert(!KPA8 || H1 % 2 == 0, "d1 = 8: h1 even (two heads per 16-row tile)");
    static_assert((size_t)SLICES * H * MO_LD * 4 + (size_t)SLICES * H * 8 + (size_t)H * DH * 4 + H * 8 <=
                      (size_t)STAGES * STAGE_BYTES,
                  "slice merge and merged partial must fit in the ring");
    static_assert(WARPS <= 31, "too many consumer warps");
    static_assert(STAGES <= 12, "stage release counters");
    static_assert(PRODUCER_WARP || WARPS <= 16, "sixteen warps at most without a producer warp");
    static_assert(smem_bytes() <= 227 * 1024, "shared memory");
    static_assert(!ORDER3 || (D1 == 1 && H2 == 1 && !SHARED && DB == 8 && DC == 8),
                  "third-order mode: TPA split, d_b = d_c = 8 (one c pair per fragment lane)");
};

// TPA, h = 16, d_h = 64, R_K = R_V = 2 (the degenerate split h1 = h, d1 = 1, h2 = 1).
using MmaTpaH16D64R2 = MmaDecodeCfg<16, 1, 64, 2, 2, 1, 8, 1, 2>;
// TPA, h = 16, d_h = 64, R = 2 with one B shared by keys and values.
using MmaTpaH16D64R2Shared = MmaDecodeCfg<16, 1, 64, 2, 2, 1, 8, 1, 2, true>;
// KPA h = 4x4, d_h = 8x16, R = 2 with one B shared by keys and values.
using MmaKpaH4x4D8x16R2Shared = MmaDecodeCfg<32, 8, 16, 2, 2, 4, 2, 2, 2, true>;
// TPA, h = 32, d_h = 64, R_K = R_V = 1 (the FlashTPA decoding benchmark's shape): the
// two head tiles split over two warps of each of four token slices (one warp holding
// both spilled).
using MmaTpaH32D64R1 = MmaDecodeCfg<32, 1, 64, 1, 1, 1, 4, 4, 2, false, 0, 2>;
// KPA h = 4x8, d_h = 8x16, R_K = R_V = 4.
using MmaKpaH4x8D8x16R4 = MmaDecodeCfg<32, 8, 16, 4, 4, 8, 2, 1, 2>;
// KPA h = 4x8, d_h = 8x16, R_K = R_V = 2.
using MmaKpaH4x8D8x16R2 = MmaDecodeCfg<32, 8, 16, 2, 2, 8, 2, 2, 2>;
// KPA h = 4x4, d_h = 8x16, R_K = R_V = 2.
using MmaKpaH4x4D8x16R2 = MmaDecodeCfg<32, 8, 16, 2, 2, 4, 4, 1, 2>;
// Third-order TPA, h = 16, d_h = 8 x 8, R_K = R_V = 2.
using MmaTpa3H16D8x8R2 = MmaDecodeCfg<16, 1, 64, 2, 2, 1, 8, 1, 2, false, 8>;
// The head splits of "Kronecker Product Attention" section 3.2 (d1 = d2 = 8, R_K = R_V = 2):
// h = 4x4, 2x8, 8x2 (the 353M models) and 4x5, 2x10, 10x2 (the 773M models).
using MmaKpaH4x4D8x8R2 = MmaDecodeCfg<32, 8, 8, 2, 2, 4, 4, 1, 2>;
using MmaKpaH2x8D8x8R2 = MmaDecodeCfg<16, 8, 8, 2, 2, 8, 2, 2, 2>;
using MmaKpaH8x2D8x8R2 = MmaDecodeCfg<64, 8, 8, 2, 2, 2, 8, 1, 2>;
using MmaKpaH4x5D8x8R2 = MmaDecodeCfg<32, 8, 8, 2, 2, 5, 3, 2, 2>;
using MmaKpaH2x10D8x8R2 = MmaDecodeCfg<16, 8, 8, 2, 2, 10, 1, 4, 2>;
using MmaKpaH10x2D8x8R2 = MmaDecodeCfg<80, 8, 8, 2, 2, 2, 8, 1, 2>;
// The append+prefill configuration's h = 16, d_h = 128 in two more splits: TPA (h1 = 16,
// d1 = 1; 1152-byte records, so 64 tokens per stage) and KPA h = 4x4, d_h = 8x16 at rank 4.
using MmaTpaH16D128R2 = MmaDecodeCfg<16, 1, 128, 2, 2, 1, 4, 1, 2>;
using MmaKpaH4x4D8x16R4 = MmaDecodeCfg<32, 8, 16, 4, 4, 4, 4, 1, 2>;
// TPA h = 61, d_h = 64, R = 2: the TPA explainer's 773M model.  61 heads pad to 4 tiles
// of 16 rows, one per warp of a token slice (HS = 4, two slices: 8 consumer warps);
// 1000-byte records, 64 tokens a stage.
using MmaTpaH61D64R2 = MmaDecodeCfg<64, 1, 64, 2, 2, 1, 2, 2, 2, false, 0, 4, 61>;

#define KPA_MMA_VARIANTS(X)        \
    X(0, MmaTpaH16D64R2)           \
    X(1, MmaKpaH4x8D8x16R4)        \
    X(2, MmaKpaH4x8D8x16R2)        \
    X(3, MmaKpaH4x4D8x16R2)        \
    X(4, MmaTpaH32D64R1)           \
    X(5, MmaTpaH16D64R2Shared)     \
    X(6, MmaKpaH4x4D8x16R2Shared)  \
    X(7, MmaTpa3H16D8x8R2)         \
    X(8, MmaKpaH4x4D8x8R2)         \
    X(9, MmaKpaH2x8D8x8R2)         \
    X(10, MmaKpaH8x2D8x8R2)        \
    X(11, MmaKpaH4x5D8x8R2)        \
    X(12, MmaKpaH2x10D8x8R2)       \
    X(13, MmaKpaH10x2D8x8R2)       \
    X(14, MmaTpaH16D128R2)         \
    X(15, MmaKpaH4x4D8x16R4)       \
    X(16, MmaTpaH61D64R2)

// Index of the variant that covers these dims, or -1.
inline int mma_decode_variant(const Dims &d) {
#define KPA_MMA_MATCH(IDX, CFG)                                                                    \
    if (d.rk == CFG::RK && d.rv == CFG::RV &&                                                      \
        (CFG::ORDER3 ? (d.order == 3 && d.h1 == CFG::MA && d.h2 == 1 && d.d1 == CFG::DB && d.d2 == CFG::DC) \
                     : (d.order != 3 && d.h1 * d.d1 == CFG::MR && d.d1 == CFG::D1 && d.d2 == CFG::D2 &&  \
                        d.h2 == CFG::H2 && (d.shared != 0) == CFG::SHARED)))                       \
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

// Most query-factor values (E_Q) a decode of this variant can take from query factors.
inline int mma_decode_qf_max(int variant) {
#define KPA_MMA_QFMAX(IDX, CFG) \
    if (variant == IDX) return CFG::QF_MAX;
    KPA_MMA_VARIANTS(KPA_MMA_QFMAX)
#undef KPA_MMA_QFMAX
    return 0;
}

inline size_t mma_decode_smem(int variant) {
#define KPA_MMA_SMEM(IDX, CFG) \
    if (variant == IDX) return CFG::smem_bytes();
    KPA_MMA_VARIANTS(KPA_MMA_SMEM)
#undef KPA_MMA_SMEM
    return 0;
}

// Number of clusters of `size` CTAs of a variant that fit on the current device at
// once (0: a cluster that large cannot run).
int mma_decode_max_clusters(int variant, int size);

// The tcgen05 decode (TPA, h = 16, d_h = 64, R_K = R_V = 2, dense query, no cluster;
// selected on request):
// whether it covers these dims, its shared memory, and its launcher.
bool tc_decode_supported(const Dims &d);
size_t tc_decode_smem();
cudaError_t launch_decode_tc(const DecodeArgs &args, int batch, const DecodePlan &plan, const RopeTable &rope,
                             const DecodeTestHooks &hooks, cudaStream_t st);

cudaError_t launch_decode_mma(int variant, const DecodeArgs &args, int batch, const DecodePlan &plan,
                              const RopeTable &rope, const DecodeTestHooks &hooks, cudaStream_t st);

}  // namespace kpa
