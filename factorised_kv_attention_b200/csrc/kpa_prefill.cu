// kpa_prefill.cu -- causal chunked attention in factor space on the tcgen05 tensor cores.
//
// Row t of sequence b is the query at position start_pos[b] + t; it attends to cache
// slots 0 .. start_pos[b] + t ("Kronecker Product Attention", eqs 3-4, with B^K
// pre-rotated in the cache per Theorem 2.4).  Keys and values exist only as factors:
// each 128-token K and V tile of one head is rebuilt on chip,
//     K[s][(j1,j2)] = sum_r A^K_r(s)[i1,j1] B~^K_r(s)[i2,j2]     (1/R_K folded into the scale)
//     V[s][(j1,j2)] = sum_r A^V_r(s)[i1,j1] B^V_r(s)[i2,j2]      (1/R_V folded into the output)
// and is never written to device memory.
//
// One CTA takes 256 query rows of one (sequence, head) as two 128-row halves that
// share every rebuilt K/V tile and take turns on the tensor pipe:
//   - a producer warp streams the head's factor slices of each key tile into shared
//     memory with TMA, two tiles ahead (and loads the Q tile once);
//   - eight rebuild warps form the K tile (token rows) and the V^T tile (feature rows)
//     in the 128-byte-swizzled K-major layouts tcgen05.mma reads, from ldmatrix.trans
//     fragments of the factors through stmatrix / stmatrix.trans; K runs one tile
//     ahead of V, K is double-buffered;
//   - one thread issues S_h = Q_h K^T (both operands in shared memory) and
//     O_h += P_h V (P_h read from tensor memory) in the order S0 S1 | PV0 S0' PV1 S1' ...,
//     so one half's softmax overlaps the other half's MMAs;
//   - eight softmax warps (one query row per thread) read S_h from tensor memory,
//     apply the causal mask on diagonal tiles and write P_h over S_h as fp16.
// Tensor memory: S0 | S1 | O0 | O1, 128 columns each (all 512).
//
// Numerics: the tensor-core operands are fp16 (an 11-bit significand: the rebuilt K
// and V are rounded once, P once, Q once after the softmax scale sm_scale/R_K*log2(e)
// is folded into it); accumulation is fp32.  The running maximum is only moved when a
// row's maximum grows by more than 2^8 (FlashAttention-4's conditional rescaling), so
// P stays in [0, 256].  A value outside the fp16 range becomes inf and makes the row's
// output non-finite; such a row is reported as KPA_ERR_DEVICE_CHECK.
#include <cudaTypedefs.h>
#include <cstring>

#include <cuda_fp16.h>

#include "kpa_f32x2.cuh"
#include "kpa_internal.cuh"
#include "kpa_sm100.cuh"

namespace kpa {

struct PrefillArgs {
    int batch, n_tok, cap;
    const int32_t *start_pos;
    float *out;
    float qscale;       // sm_scale / R_K * log2(e)
    float out_scale;    // 1 / R_V
    int h1, h2;
    int *err;
    unsigned long long wait_limit_ns;
    double theta[8];    // theta_m, m < d2/2 (shared B: the keys are rotated while K is rebuilt)
    // query factors instead of a dense query (null: q by TMA): element e of token t of
    // sequence b at qf[e * qf_stride + b * qf_seq_stride + t * qf_tok_stride], B^Q rotated
    const float *qf;
    long long qf_stride, qf_seq_stride, qf_tok_stride;
    int rq;
    float qf_scale;     // qscale / R_Q
};

constexpr int kPrefillMaxRq = 6;    // query rank a prefill from query factors takes

namespace {

using f32x2::fadd2;
using f32x2::ffma2;
using f32x2::fmul2;
using f32x2::fsub2;
using f32x2::unpack_bf16x2;
using f32x2::exp2_poly2;

using namespace sm100;

constexpr int HQ = 128;                       // query rows per half
constexpr int TK = 128;                       // keys per tile
constexpr int kSoftmaxWarps = 8, kRebuildWarps = 8;
constexpr int kRebuildWarp0 = kSoftmaxWarps;                  // warps 8..15
constexpr int kMmaWarp = kSoftmaxWarps + kRebuildWarps;       // warp 16
constexpr int kProducerWarp = kMmaWarp + 1;                   // warp 17
constexpr int kThreads = (kProducerWarp + 1) * 32;            // 576
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.f;
constexpr int kBox = 16 * 64 * 2;             // TMA box: 16 cache groups x (8 elements x 8 tokens) bf16

template <int D1_, int D2_, int RK_, int RV_>
struct PrefillCfg {
    static constexpr int D1 = D1_, D2 = D2_, RK = RK_, RV = RV_;
    static constexpr int DH = D1 * D2;
    static_assert(D1 == 8 && (D2 == 16 || D2 == 8), "the fragment mapping covers d1 = 8, d2 = 16 or 8");
    static_assert(RK == RV && (RK == 2 || (RK == 4 && D2 == 16)), "ranks: 2, or 4 with d2 = 16");
    static constexpr int HB = D2 / 8;                          // 8-element boxes of a B row
    // factor stages: two at R = 2; one at R = 4, where two stages of four ranks' slices
    // would not fit beside the Q, K and V tiles
    static constexpr int FST = RK == 2 ? 2 : 1;
    static constexpr uint32_t Q_HALF = HQ * DH * 2;
    static constexpr uint32_t KV_TILE = TK * DH * 2;
    static constexpr uint32_t K_ST = (1 + HB) * RK * kBox;   // A_r (1 box) and B_r (HB boxes) per rank
    static constexpr uint32_t V_ST = (1 + HB) * RV * kBox;
    static constexpr size_t OFF_Q = 0;                         // two halves
    static constexpr size_t OFF_K = OFF_Q + 2 * Q_HALF;        // two buffers
    static constexpr size_t OFF_V = OFF_K + 2 * KV_TILE;       // one buffer
    static constexpr size_t OFF_KST = OFF_V + KV_TILE;         // FST stages
    static constexpr size_t OFF_VST = OFF_KST + FST * K_ST;    // FST stages
    static constexpr size_t OFF_BAR = OFF_VST + FST * V_ST;
    static constexpr int NBAR = 24;
    static constexpr size_t SMEM = 1024 + OFF_BAR + NBAR * 8 + 16;
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

// mbarrier slots
enum : int {
    B_Q = 0,
    B_QREADY = 1,      // +h
    B_KST_FULL = 3,    // +stage
    B_VST_FULL = 5,
    B_KST_EMPTY = 7,
    B_VST_EMPTY = 9,
    B_K_FULL = 11,     // +buffer
    B_K_EMPTY = 13,
    B_V_FULL = 15,
    B_V_EMPTY = 16,
    B_S_FULL = 17,     // +h
    B_P_FULL = 19,     // +h
    B_O_FINAL = 21,    // +h
    B_DRAIN = 23,
};

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` in a 128-byte-swizzled block.
__device__ __forceinline__ uint32_t sw128_chunk(int row, int chunk) {
    return (uint32_t)row * 128 + ((uint32_t)(chunk ^ (row & 7)) << 4);
}

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t (&r)[2]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
                 : "=r"(r[0]), "=r"(r[1])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void stsm_x4(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(r0),
                 "r"(r1), "r"(r2), "r"(r3)
                 : "memory");
}
__device__ __forceinline__ void stsm_x4_t(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(r0),
                 "r"(r1), "r"(r2), "r"(r3)
                 : "memory");
}

// (x, y) -> fp16x2 word, x in the low half
__device__ __forceinline__ uint32_t pack_half2(float x, float y) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(y), "f"(x));
    return r;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}


// D[tmem] (+)= A[tmem] * B[smem]^T (A read from tensor memory), issued by one thread.
__device__ __forceinline__ void umma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                        bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"((uint32_t)accumulate)
        : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
          "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
          "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]),
        "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]), "f"(v[16]),
        "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]), "f"(v[24]),
        "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]), "f"(v[29]), "f"(v[30]), "f"(v[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t (&w)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]), "r"(w[8]),
        "r"(w[9]), "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15])
        : "memory");
}

// Which tiles a half works on: both halves start at tile 0; half h stops at last[h].
struct TilePlan {
    bool act[2];
    int last[2];
    int n_kt;
    __device__ bool active(int h, int t) const { return act[h] && t <= last[h]; }
    __device__ int first_half(int t) const { return active(0, t) ? 0 : 1; }
    __device__ int last_half(int t) const { return active(1, t) ? 1 : 0; }
};

template <class C, bool SHARED, bool QF>
__global__ void __launch_bounds__(kThreads, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
               const __grid_constant__ CUtensorMap tmv, PrefillArgs a) {
    constexpr int D1 = C::D1, RK = C::RK, RV = C::RV, DH = C::DH;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t bar0 = smem_u32(smem + C::OFF_BAR);
    auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_BAR + C::NBAR * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_pairs = (a.n_tok + 2 * HQ - 1) / (2 * HQ);
    const int pair = n_pairs - 1 - (int)blockIdx.x;             // longest rows first
    const int head = blockIdx.y, b = blockIdx.z;
    const int h = a.h1 * a.h2, i1 = head / a.h2, i2 = head % a.h2;
    const int q0 = pair * 2 * HQ;
    const int start = a.start_pos[b];
    const uint64_t limit = a.wait_limit_ns;

    // Tiles: half hh covers rows q0 + hh*128 .. min(+127, n_tok-1), positions start + row.
    TilePlan tp;
    bool range_ok = start >= 0;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const int r0 = q0 + hh * HQ;
        tp.act[hh] = r0 < a.n_tok;
        int last_slot = start + min(r0 + HQ, a.n_tok) - 1;
        if (last_slot >= a.cap) {
            range_ok = false;
            last_slot = a.cap - 1;
        }
        tp.last[hh] = tp.act[hh] && last_slot >= 0 ? last_slot / TK : -1;
        if (tp.last[hh] < 0) tp.act[hh] = false;
    }
    if (start < 0) tp.act[0] = tp.act[1] = false, tp.last[0] = tp.last[1] = -1;
    tp.n_kt = max(tp.last[0], tp.last[1]) + 1;
    // slots past the last row's position stay zero in the rebuilt tiles
    const int max_slot = min(start + min(q0 + 2 * HQ, a.n_tok) - 1, a.cap - 1);
    if (!range_ok && tid == 0) raise_error(a.err, kErrDeviceCheck);

    if (tid == 0) {
        for (int i = 0; i < C::NBAR; ++i) {
            uint32_t count = 1;
            if ((i >= B_QREADY && i < B_QREADY + 2) || (i >= B_P_FULL && i < B_P_FULL + 2)) count = 4;
            if ((i >= B_KST_EMPTY && i < B_KST_EMPTY + 2) || (i >= B_VST_EMPTY && i < B_VST_EMPTY + 2) ||
                (i >= B_K_FULL && i < B_K_FULL + 2) || i == B_V_FULL)
                count = kRebuildWarps;
            mbar_init(bar(i), count);
        }
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // Bounded wait shared by every role: gives up when the time runs out or another
    // thread has already given up, and records the timeout once.
    auto wait = [&](int i, uint32_t parity) -> bool {
        if (mbar_try_wait(bar(i), parity)) return true;
        const uint64_t t0 = globaltimer();
        for (uint32_t it = 1;; ++it) {
            if (mbar_try_wait(bar(i), parity)) return true;
            if ((it & 15) == 0) {
                if (*abort_flag) return false;
                if (globaltimer() - t0 > limit) {
                    *abort_flag = 1;
                    raise_error(a.err, kErrTimeout);
                    return false;
                }
            }
        }
    };

    if (warp == kProducerWarp) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0 && tp.n_kt > 0) {
            if (!QF) tma_prefetch_desc(&tmq);
            tma_prefetch_desc(&tmk);
            tma_prefetch_desc(&tmv);
            const int grp0 = (int)((int64_t)b * a.cap / kGroup);
            const int ea = RK * a.h1 * D1;     // first B element of a key record
            const int va = RV * a.h1 * D1;
            int issued[2][2] = {{-1, -1}, {-1, -1}};          // [plane][stage < FST]
            // the head's factor slices of tile t: A_r[i1] (one box) and B_r[i2] (two boxes) per rank
            auto issue_factors = [&](int t, bool is_v) -> bool {
                constexpr int FST = C::FST;
                const int s = t % FST, grp = grp0 + t * (TK / kGroup);
                if (t >= FST && !wait((is_v ? B_VST_EMPTY : B_KST_EMPTY) + s, ((t / FST) - 1) & 1)) return false;
                const uint32_t full = bar((is_v ? B_VST_FULL : B_KST_FULL) + s);
                mbar_expect_tx(full, is_v ? C::V_ST : C::K_ST);
                unsigned char *st = smem + (is_v ? C::OFF_VST + s * C::V_ST : C::OFF_KST + s * C::K_ST);
                const CUtensorMap *map = is_v ? &tmv : &tmk;
                // a shared B sits in the key record, after A^K, for the values too
                const CUtensorMap *bmap = is_v && !SHARED ? &tmv : &tmk;
                const int R = is_v ? RV : RK, b0 = is_v && !SHARED ? va : ea;
                for (int r = 0; r < R; ++r) {
                    tma_load_2d(smem_u32(st + r * kBox), map, (r * a.h1 * D1 + i1 * D1) * kGroup, grp, full);
#pragma unroll
                    for (int hb = 0; hb < C::HB; ++hb)
                        tma_load_2d(smem_u32(st + (R + C::HB * r + hb) * kBox), bmap,
                                    (b0 + (r * a.h2 + i2) * C::D2 + hb * 8) * kGroup, grp, full);
                }
                issued[is_v ? 1 : 0][s] = t;
                return true;
            };
            // the first key tile's factors go out ahead of Q: its rebuild is the first step
            bool ok = issue_factors(0, false);
            const int nh = (tp.act[0] ? 1 : 0) + (tp.act[1] ? 1 : 0);
            if (!QF) {                           // query factors: the softmax warps assemble Q
                mbar_expect_tx(bar(B_Q), (uint32_t)nh * C::Q_HALF);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
                    if (tp.act[hh])
#pragma unroll
                        for (int cb = 0; cb < DH / 64; ++cb)
                            tma_load_2d(smem_u32(smem + C::OFF_Q + hh * C::Q_HALF + cb * HQ * 128), &tmq,
                                        head * DH + cb * 64, b * a.n_tok + q0 + hh * HQ, bar(B_Q));
            }
            if (ok) ok = issue_factors(0, true);
            for (int t = 1; t < tp.n_kt && ok; ++t) {
                ok = issue_factors(t, false);
                if (ok) ok = issue_factors(t, true);
            }
            // every copy this thread started lands before the CTA can exit
            if (!QF) (void)mbar_wait(bar(B_Q), 0, limit);
#pragma unroll
            for (int pl = 0; pl < 2; ++pl)
#pragma unroll
                for (int s = 0; s < C::FST; ++s)
                    if (issued[pl][s] >= 0)
                        (void)mbar_wait(bar((pl ? B_VST_FULL : B_KST_FULL) + s), (issued[pl][s] / C::FST) & 1, limit);
        }
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------------- MMA issue
        if (lane == 0 && tp.n_kt > 0) {
            const uint32_t idesc_s = umma_idesc_f16_f32(HQ, TK), idesc_o = umma_idesc_f16_f32(HQ, DH);
            bool ok = true;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
                if (ok && tp.act[hh] && !wait(B_QREADY + hh, 0)) ok = false;
            auto issue_s = [&](int hh, int t) -> bool {
                const int kb = t & 1;
                if (!wait(B_K_FULL + kb, (t >> 1) & 1)) return false;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < DH / 16; ++k) {
                    const uint64_t qd =
                        umma_desc_k_sw128(smem_u32(smem + C::OFF_Q + hh * C::Q_HALF + (k / 4) * HQ * 128)) +
                        2 * (k % 4);
                    const uint64_t kd =
                        umma_desc_k_sw128(smem_u32(smem + C::OFF_K + kb * C::KV_TILE + (k / 4) * TK * 128)) +
                        2 * (k % 4);
                    umma_bf16(tmem + hh * 128, qd, kd, idesc_s, k > 0);
                }
                umma_commit(bar(B_S_FULL + hh));
                if (hh == tp.last_half(t)) umma_commit(bar(B_K_EMPTY + kb));
                return true;
            };
            auto issue_pv = [&](int hh, int t) -> bool {
                if (!wait(B_P_FULL + hh, t & 1)) return false;
                if (hh == tp.first_half(t) && !wait(B_V_FULL, t & 1)) return false;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < TK / 16; ++k) {
                    const uint64_t vd =
                        umma_desc_k_sw128(smem_u32(smem + C::OFF_V + (k / 4) * DH * 128)) + 2 * (k % 4);
                    umma_ts(tmem + 256 + hh * 128, tmem + hh * 128 + 8 * k, vd, idesc_o, t > 0 || k > 0);
                }
                if (hh == tp.last_half(t)) umma_commit(bar(B_V_EMPTY));
                if (t == tp.last[hh]) umma_commit(bar(B_O_FINAL + hh));
                return true;
            };
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
                if (ok && tp.active(hh, 0)) ok = issue_s(hh, 0);
            for (int t = 0; t < tp.n_kt && ok; ++t) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    if (ok && tp.active(hh, t)) ok = issue_pv(hh, t);
                    if (ok && tp.active(hh, t + 1)) ok = issue_s(hh, t + 1);
                }
            }
            // nothing issued here may still run when tensor memory is released
            umma_commit(bar(B_DRAIN));
            (void)mbar_wait(bar(B_DRAIN), 0, limit);
        }
    } else if (warp >= kRebuildWarp0) {
        // ---------------------------------------------------------------- K / V rebuild
        const int rw = warp - kRebuildWarp0;
        const int tok = lane >> 2;                 // token of the 8-token group this lane holds
        const int blk = lane >> 3, brow = lane & 7;   // ldmatrix / stmatrix row this lane addresses
        // Rebuild one plane of tile t: K (token rows, stmatrix) or V^T (feature rows, stmatrix.trans).
        auto rebuild = [&](int t, bool is_v) {
            const int fs = t % C::FST;                                    // factor stage
            const unsigned char *st = smem + (is_v ? C::OFF_VST + fs * C::V_ST : C::OFF_KST + fs * C::K_ST);
            const uint32_t dst = smem_u32(smem + (is_v ? C::OFF_V : C::OFF_K + (t & 1) * C::KV_TILE));
            const bool edge = t * TK + TK - 1 > max_slot;
#pragma unroll 1
            for (int gi = 0; gi < TK / kGroup / kRebuildWarps; ++gi) {
                const int g = rw + gi * kRebuildWarps;      // group of the tile, 0..15
                // A_r[tok][j1], r < R: one 16-byte row per j1 holds the group's 8 tokens
                constexpr int R = RK;
                float av[R][8];
#pragma unroll
                for (int r = 0; r < R; ++r)
#pragma unroll
                    for (int j1 = 0; j1 < 8; ++j1)
                        av[r][j1] = __uint_as_float(
                            (uint32_t)(*reinterpret_cast<const uint16_t *>(st + r * kBox + g * 128 + j1 * 16 + tok * 2))
                            << 16);
                // B_r[tok][hb*8 + 2c .. +1] for (r, hb) = block r * HB + hb
                constexpr int HB = C::HB, NBLK = R * HB;
                float2 bf[NBLK];
                if constexpr (HB == 2) {
#pragma unroll
                    for (int q4 = 0; q4 < NBLK / 4; ++q4) {          // four blocks (two ranks) per load
                        uint32_t bw[4];
                        ldsm_x4_t(smem_u32(st + (R + 4 * q4 + blk) * kBox + g * 128 + brow * 16), bw);
#pragma unroll
                        for (int i = 0; i < 4; ++i) bf[4 * q4 + i] = unpack_bf16x2(bw[i]);
                    }
                } else {
                    uint32_t bw[2];                          // lanes 0..15 address the two blocks
                    ldsm_x2_t(smem_u32(st + (R + (blk & 1)) * kBox + g * 128 + brow * 16), bw);
#pragma unroll
                    for (int i = 0; i < 2; ++i) bf[i] = unpack_bf16x2(bw[i]);
                }
                if (SHARED && !is_v) {
                    // shared B is cached unrotated: rotate this lane's pairs m = c (and 4 + c when
                    // d2 = 16) of its token at the token's slot ("Kronecker Product Attention", Thm 2.4)
                    const double pos = (double)(t * TK + g * kGroup + tok);
                    float c0, s0, c1 = 1.f, s1 = 0.f;
                    rope_cs_fast(pos, a.theta[lane & 3], c0, s0);
                    if constexpr (HB == 2) rope_cs_fast(pos, a.theta[4 + (lane & 3)], c1, s1);
#pragma unroll
                    for (int i = 0; i < NBLK; ++i) {
                        const float cc = (i % HB) ? c1 : c0, ss = (i % HB) ? s1 : s0;
                        bf[i] = make_float2(bf[i].x * cc - bf[i].y * ss, bf[i].x * ss + bf[i].y * cc);
                    }
                }
                uint32_t w[8][HB];
#pragma unroll
                for (int j1 = 0; j1 < 8; ++j1)
#pragma unroll
                    for (int hb = 0; hb < HB; ++hb) {
                        float2 acc = fmul2(make_float2(av[0][j1], av[0][j1]), bf[hb]);
#pragma unroll
                        for (int r = 1; r < R; ++r)
                            acc = ffma2(make_float2(av[r][j1], av[r][j1]), bf[r * HB + hb], acc);
                        w[j1][hb] = pack_half2(acc.x, acc.y);
                    }
                if (edge && t * TK + g * kGroup + tok > max_slot) {
#pragma unroll
                    for (int j1 = 0; j1 < 8; ++j1)
#pragma unroll
                        for (int hb = 0; hb < HB; ++hb) w[j1][hb] = 0u;
                }
                // this lane addresses row brow of block blk of each x4 store: d2 = 16, (j1 = 2i +
                // blk/2, hb = blk%2); d2 = 8, j1 = 4i + blk
#pragma unroll
                for (int i = 0; i < 8 / (4 / HB); ++i) {
                    const int f0 = HB == 2 ? (2 * i + (blk >> 1)) * 16 + (blk & 1) * 8 : (4 * i + blk) * 8;
                    uint32_t w0, w1, w2, w3;
                    if constexpr (HB == 2) {
                        w0 = w[2 * i][0], w1 = w[2 * i][HB - 1], w2 = w[2 * i + 1][0], w3 = w[2 * i + 1][HB - 1];
                    } else {
                        w0 = w[4 * i][0], w1 = w[4 * i + 1][0], w2 = w[4 * i + 2][0], w3 = w[4 * i + 3][0];
                    }
                    if (!is_v) {
                        const int row = g * kGroup + brow;                          // token row
                        const uint32_t ad = dst + (f0 >> 6) * (TK * 128) + sw128_chunk(row, (f0 & 63) >> 3);
                        stsm_x4(ad, w0, w1, w2, w3);
                    } else {
                        const int row = f0 + brow;                                  // feature row
                        const uint32_t ad = dst + (g >> 3) * (DH * 128) + sw128_chunk(row, g & 7);
                        stsm_x4_t(ad, w0, w1, w2, w3);
                    }
                }
            }
        };
        auto step = [&](int t, bool is_v) -> bool {
            const int s = t & 1, fs = t % C::FST;           // K buffer, factor stage
            bool ok = wait((is_v ? B_VST_FULL : B_KST_FULL) + fs, (t / C::FST) & 1);
            if (ok && !is_v && t >= 2) ok = wait(B_K_EMPTY + s, ((t >> 1) - 1) & 1);
            if (ok && is_v && t >= 1) ok = wait(B_V_EMPTY, (t - 1) & 1);
            if (!__all_sync(0xffffffffu, ok)) return false;
            rebuild(t, is_v);
            fence_async_smem();        // visible to the tensor cores
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(is_v ? B_V_FULL : B_K_FULL + s));
                mbar_arrive(bar((is_v ? B_VST_EMPTY : B_KST_EMPTY) + fs));
            }
            return true;
        };
        if (tp.n_kt > 0) {
            bool ok = step(0, false);
            for (int t = 0; t < tp.n_kt && ok; ++t) {
                if (t + 1 < tp.n_kt) ok = step(t + 1, false);
                if (ok) ok = step(t, true);
            }
        }
    } else {
        // ---------------------------------------------------------------- softmax rows
        const int hh = warp >> 2, quarter = warp & 3;
        const int row = quarter * 32 + lane;
        if (tp.act[hh]) {
            const int qrow = q0 + hh * HQ + row;
            const int pos = start + qrow;
            bool ok = true;
            if constexpr (QF) {
                // Q_h from the query factors ("Kronecker Product Attention", eq 2):
                // q[j1 d2 + j2] = (1/R_Q) sum_r A^Q_r[i1][j1] B^Q_r[i2][j2], scaled and rounded
                // once to fp16, written as 8-byte pieces into the 128-byte-swizzled K-major
                // tile the MMA reads.  Four passes over quarters of d2 keep B^Q in registers.
                const int t = q0 + hh * HQ + row;
                const bool live = t < a.n_tok;
                const float *src = a.qf + (long long)b * a.qf_seq_stride + (long long)t * a.qf_tok_stride;
                const int qa = a.rq * a.h1 * D1;                    // first B^Q element of the record
                unsigned char *qh = smem + C::OFF_Q + hh * C::Q_HALF;
                // A^Q[r][i1][0..D1) of the row: every load in flight at once, then kept
                float aq[kPrefillMaxRq][D1];
#pragma unroll
                for (int r = 0; r < kPrefillMaxRq; ++r)
#pragma unroll
                    for (int j1 = 0; j1 < D1; ++j1)
                        aq[r][j1] = live && r < a.rq
                                        ? __ldg(src + (long long)((r * a.h1 + i1) * D1 + j1) * a.qf_stride)
                                        : 0.f;
#pragma unroll 1
                for (int hb = 0; hb < C::D2 / 4; ++hb) {            // four features of d2 per pass
                    float bq[kPrefillMaxRq][4];
#pragma unroll
                    for (int r = 0; r < kPrefillMaxRq; ++r)
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            bq[r][u] = live && r < a.rq
                                           ? __ldg(src + (long long)(qa + (r * a.h2 + i2) * C::D2 + hb * 4 + u) *
                                                             a.qf_stride)
                                           : 0.f;
#pragma unroll
                    for (int j1 = 0; j1 < D1; ++j1) {
                        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int r = 0; r < kPrefillMaxRq; ++r)
#pragma unroll
                            for (int u = 0; u < 4; ++u) acc[u] += aq[r][j1] * bq[r][u];
                        uint2 pk;
                        pk.x = pack_half2(acc[0] * a.qf_scale, acc[1] * a.qf_scale);
                        pk.y = pack_half2(acc[2] * a.qf_scale, acc[3] * a.qf_scale);
                        const int f0 = j1 * C::D2 + hb * 4;          // first feature of the piece
                        *reinterpret_cast<uint2 *>(qh + (f0 >> 6) * HQ * 128 + sw128_chunk(row, (f0 & 63) >> 3) +
                                                   (f0 & 4) * 2) = pk;
                    }
                }
                fence_async_smem();
            } else {
            // Q_h: bf16 -> fp16 x qscale in place, once its copy has landed
            ok = wait(B_Q, 0);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                uint4 *q4 = reinterpret_cast<uint4 *>(smem + C::OFF_Q + hh * C::Q_HALF);
#pragma unroll 4
                for (int i = row; i < (int)(C::Q_HALF / 16); i += HQ) {
                    uint4 u = q4[i];
                    uint32_t *wv = reinterpret_cast<uint32_t *>(&u);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float2 f = unpack_bf16x2(wv[k]);
                        wv[k] = pack_half2(f.x * a.qscale, f.y * a.qscale);
                    }
                    q4[i] = u;
                }
                fence_async_smem();
            }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_QREADY + hh));

            const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
            const uint32_t s_addr = tmem + lane_off + hh * 128;
            const uint32_t o_addr = tmem + lane_off + 256 + hh * 128;
            const int row_first = start + q0 + hh * HQ;              // smallest position in the half
            float m_used = -INFINITY, l_run = 0.f;
            for (int t = 0; t <= tp.last[hh] && ok; ++t) {
                ok = __all_sync(0xffffffffu, wait(B_S_FULL + hh, t & 1));
                if (!ok) break;
                tc_fence_after();
                const bool masked = t * TK + TK - 1 > row_first;
                const int lim = pos - t * TK;                         // keys j <= lim are visible
                float mx = -INFINITY;
#pragma unroll 1
                for (int c = 0; c < TK / 32; ++c) {
                    float v[32];
                    tmem_ld32(s_addr + c * 32, v);
                    if (masked) {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (c * 32 + j > lim) v[j] = -INFINITY;
                    }
                    float ma = fmax3(mx, v[0], v[1]), mb = fmax3(v[2], v[3], v[4]);
#pragma unroll
                    for (int j = 5; j < 29; j += 4) {
                        ma = fmax3(ma, v[j], v[j + 1]);
                        mb = fmax3(mb, v[j + 2], v[j + 3]);
                    }
                    mx = fmax3(ma, mb, fmax3(v[29], v[30], v[31]));
                }
                // conditional rescale: move the reference maximum only when it grew past 2^8
                const bool grow = mx > m_used + kRescaleLog2;
                float alpha = 1.f;
                if (grow) {
                    alpha = m_used == -INFINITY ? 0.f : ex2(m_used - mx);
                    m_used = mx;
                    l_run *= alpha;
                }
                if (t > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
                    for (int c = 0; c < DH / 32; ++c) {
                        float v[32];
                        tmem_ld32(o_addr + c * 32, v);
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] *= alpha;
                        tmem_st32(o_addr + c * 32, v);
                    }
                }
                const float mref = m_used == -INFINITY ? 0.f : m_used;
                const float2 mref2 = make_float2(mref, mref);
                float2 suma = make_float2(0.f, 0.f), sumb = make_float2(0.f, 0.f);
#pragma unroll 1
                for (int c = 0; c < TK / 32; ++c) {
                    float v[32];
                    tmem_ld32(s_addr + c * 32, v);
                    uint32_t pw[16];
#pragma unroll
                    for (int jp = 0; jp < 16; ++jp) {
                        const float2 x = fsub2(make_float2(v[2 * jp], v[2 * jp + 1]), mref2);
                        // one pair in four on the FMA pipe, the rest on the transcendental unit
                        float2 p = (jp & 3) == 3 ? exp2_poly2(x) : make_float2(ex2(x.x), ex2(x.y));
                        if (masked) {
                            if (c * 32 + 2 * jp > lim) p.x = 0.f;
                            if (c * 32 + 2 * jp + 1 > lim) p.y = 0.f;
                        }
                        if (jp & 1)
                            sumb = fadd2(sumb, p);
                        else
                            suma = fadd2(suma, p);
                        pw[jp] = pack_half2(p.x, p.y);
                    }
                    tmem_st16u(s_addr + c * 16, pw);                  // P over the S columns already read
                }
                l_run += (suma.x + suma.y) + (sumb.x + sumb.y);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_P_FULL + hh));
            }
            // epilogue: O / l, one row per thread
            if (ok) ok = __all_sync(0xffffffffu, wait(B_O_FINAL + hh, 0));
            if (ok) {
                tc_fence_after();
                const bool write = qrow < a.n_tok;
                const float inv = l_run > 0.f ? a.out_scale / l_run : 0.f;
                float *dst = a.out + (((size_t)b * a.n_tok + qrow) * h + head) * DH;
                bool finite = true;
#pragma unroll 1
                for (int c = 0; c < DH / 32; ++c) {
                    float v[32];
                    tmem_ld32(o_addr + c * 32, v);
                    if (write) {
#pragma unroll
                        for (int j = 0; j < 32; j += 4) {
                            const float4 o = make_float4(v[j] * inv, v[j + 1] * inv, v[j + 2] * inv, v[j + 3] * inv);
                            finite &= fabsf(o.x) <= 3.4e38f && fabsf(o.y) <= 3.4e38f && fabsf(o.z) <= 3.4e38f &&
                                      fabsf(o.w) <= 3.4e38f;
                            *reinterpret_cast<float4 *>(dst + c * 32 + j) = o;
                        }
                    }
                }
                if (!finite) raise_error(a.err, kErrDeviceCheck);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

using PrefillKpaH4x4D8x16R2 = PrefillCfg<8, 16, 2, 2>;
using PrefillKpaD8x8R2 = PrefillCfg<8, 8, 2, 2>;
using PrefillKpaD8x16R4 = PrefillCfg<8, 16, 4, 4>;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) != cudaSuccess ||
            qr != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// q [rows][cols] bf16: boxes of 64 columns x 128 rows, 128-byte swizzle.
bool make_q_map(CUtensorMap *map, const void *q, uint64_t rows, uint64_t cols) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)HQ};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(q), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A cache plane viewed as [groups][E x 8] bf16 (one row per 8-token group): boxes of
// 8 elements x 8 tokens (64 values, 128 B) x 16 groups, no swizzle.
bool make_factor_map(CUtensorMap *map, const void *plane, uint64_t groups, uint64_t e) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {e * kGroup, groups};
    cuuint64_t strides[1] = {e * kGroup * 2};
    cuuint32_t box[2] = {64, 16};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(plane), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool prefill_supported(const Dims &d) {
    return d.d1 == 8 && d.rk == d.rv && ((d.d2 == 16 && (d.rk == 2 || d.rk == 4)) || (d.d2 == 8 && d.rk == 2));
}

namespace {

template <class C>
cudaError_t launch_prefill_cfg(const Dims &d, int batch, int n_tok, const void *q, const PrefillQf &qf,
                               const int32_t *start_pos, const void *kc, const void *vc, int cap, float qscale,
                               float out_scale, float *out, const RopeTable &rope, int *err,
                               unsigned long long wait_limit_ns, cudaStream_t st) {
    PrefillArgs a;
    a.batch = batch;
    a.n_tok = n_tok;
    a.cap = cap;
    a.start_pos = start_pos;
    a.out = out;
    a.qscale = qscale;
    a.out_scale = out_scale;
    a.h1 = d.h1;
    a.h2 = d.h2;
    a.err = err;
    a.wait_limit_ns = wait_limit_ns;
    for (int m = 0; m < 8; ++m) a.theta[m] = m < C::D2 / 2 ? rope.theta[m] : 0.0;
    a.qf = qf.ptr;
    a.qf_stride = qf.stride;
    a.qf_seq_stride = qf.seq_stride;
    a.qf_tok_stride = qf.tok_stride;
    a.rq = qf.rq;
    a.qf_scale = qf.rq > 0 ? qscale / (float)qf.rq : 0.f;
    if (a.qf && (a.rq < 1 || a.rq > kPrefillMaxRq)) return cudaErrorInvalidValue;
    CUtensorMap tmq, tmk, tmv;
    memset(&tmq, 0, sizeof(tmq));                   // unused (and never prefetched) with query factors
    const uint64_t groups = (uint64_t)batch * cap / kGroup;
    if ((!a.qf && !make_q_map(&tmq, q, (uint64_t)batch * n_tok, (uint64_t)d.h * d.dh)) ||
        !make_factor_map(&tmk, kc, groups, (uint64_t)d.ek) || !make_factor_map(&tmv, vc, groups, (uint64_t)d.ev))
        return cudaErrorInvalidValue;
    const bool use_qf = a.qf != nullptr;
    cudaError_t e = d.shared ? (use_qf ? ensure_dynamic_smem<prefill_kernel<C, true, true>>(C::SMEM)
                                       : ensure_dynamic_smem<prefill_kernel<C, true, false>>(C::SMEM))
                             : (use_qf ? ensure_dynamic_smem<prefill_kernel<C, false, true>>(C::SMEM)
                                       : ensure_dynamic_smem<prefill_kernel<C, false, false>>(C::SMEM));
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((n_tok + 2 * HQ - 1) / (2 * HQ)), (unsigned)d.h, (unsigned)batch);
    if (d.shared && use_qf)
        prefill_kernel<C, true, true><<<grid, kThreads, C::SMEM, st>>>(tmq, tmk, tmv, a);
    else if (d.shared)
        prefill_kernel<C, true, false><<<grid, kThreads, C::SMEM, st>>>(tmq, tmk, tmv, a);
    else if (use_qf)
        prefill_kernel<C, false, true><<<grid, kThreads, C::SMEM, st>>>(tmq, tmk, tmv, a);
    else
        prefill_kernel<C, false, false><<<grid, kThreads, C::SMEM, st>>>(tmq, tmk, tmv, a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const Dims &d, int batch, int n_tok, const void *q, const PrefillQf &qf,
                           const int32_t *start_pos, const void *kc, const void *vc, int cap, float qscale,
                           float out_scale, float *out, const RopeTable &rope, int *err,
                           unsigned long long wait_limit_ns, cudaStream_t st) {
    if (!prefill_supported(d)) return cudaErrorInvalidValue;
    if (d.d2 == 8)
        return launch_prefill_cfg<PrefillKpaD8x8R2>(d, batch, n_tok, q, qf, start_pos, kc, vc, cap, qscale,
                                                     out_scale, out, rope, err, wait_limit_ns, st);
    if (d.rk == 4)
        return launch_prefill_cfg<PrefillKpaD8x16R4>(d, batch, n_tok, q, qf, start_pos, kc, vc, cap, qscale,
                                                      out_scale, out, rope, err, wait_limit_ns, st);
    return launch_prefill_cfg<PrefillKpaH4x4D8x16R2>(d, batch, n_tok, q, qf, start_pos, kc, vc, cap, qscale,
                                                      out_scale, out, rope, err, wait_limit_ns, st);
}

}  // namespace kpa
