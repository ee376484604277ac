// kpa_decode_mma.cu -- factor-space decode on the tensor cores (bf16 caches).
//
// Same mathematics as the CUDA-core kernel (Proposition 2.2 with a dense
// query; Theorem 2.4 for the positions; online softmax; values from A^V and
// B^V), arranged so that both inner contractions are small dense GEMMs per
// i2-group of heads:
//
//   score step  T_r[(i1,j1), s] = sum_j2 Q_i2[(i1,j1), j2] * B~^K_r(s)[i2, j2]
//               M = h1*d1, K = d2, N = tokens           (mma.sync m16n8k16)
//   then        score[(i1,i2), s] = sum_r sum_j1 A^K_r(s)[i1,j1] * T_r[(i1,j1), s]
//               (elementwise with A^K, then a sum over j1 across lanes)
//   value step  O_i2[(i1,j1), j2] += sum_{s,r} (p[(i1,i2),s] A^V_r(s)[i1,j1]) B^V_r(s)[i2,j2]
//               M = h1*d1, K = tokens (per rank), N = d2 (mma.sync m16n8k16)
//
// Both operands stay bf16 x bf16 with fp32 accumulation.  The rotated, scaled
// query and the probability-weighted A^V are split into bf16 hi + lo parts so
// that rounding them costs no more than ~2^-16 relative.
//
// Data movement: one producer warp streams each split's cache groups through a
// STAGES-deep shared-memory ring with cp.async.bulk (plain bulk copies into this CTA) and
// mbarrier transaction counts; consumer warps read the 8-token groups, whose
// element-major/token-minor layout makes every fragment load a conflict-free
// 16-byte row (ldmatrix) or 32-bit word (two adjacent tokens).  Every wait is
// bounded; on expiry the kernel records KPA_ERR_TIMEOUT, drains its copies and
// returns.
#include <cooperative_groups.h>

#include <type_traits>

#include "kpa_decode_merge.cuh"
#include "kpa_f32x2.cuh"
#include "kpa_internal.cuh"
#include "kpa_mma_decode.cuh"
#include "kpa_sm100.cuh"

namespace cg = cooperative_groups;

namespace kpa {
namespace {

using f32x2::fadd2;
using f32x2::ffma2;
using f32x2::fmul2;
using f32x2::fsub2;
using f32x2::unpack_bf16x2;

// ---------------------------------------------------------------- PTX helpers
using sm100::bulk_g2s;
using sm100::mbar_arrive;
using sm100::mbar_expect_tx;
using sm100::mbar_init;
using sm100::mbar_wait;
using sm100::smem_u32;

// hint a global range (16-byte aligned, a multiple of 16 bytes) into L2.  No data is
// bound to the issuing thread, and L2 stays coherent with later writes to the range.
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x1_t(uint32_t addr, uint32_t &r0) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x1.trans.shared.b16 {%0}, [%1];" : "=r"(r0) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t &r0, uint32_t &r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t &r0, uint32_t &r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
                 : "=r"(r0), "=r"(r1)
                 : "r"(addr));
}

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// m16n8k8 (k = d2 = 8): A rows g, g + 8 at k 2c, 2c + 1; B k 2c, 2c + 1 at n g
__device__ __forceinline__ void mma16808(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(b0));
}

// The same product with fp16 operands (the score of a shared-B cache, whose rotated
// key factors are formed in registers and kept at fp16 precision).
__device__ __forceinline__ void mma16816h(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t mask_pair(uint32_t v, bool keep0, bool keep1) {
    return (keep0 ? (v & 0xffffu) : 0u) | (keep1 ? (v & 0xffff0000u) : 0u);
}





__device__ __forceinline__ uint32_t lds_u32(const unsigned char *p) {
    return *reinterpret_cast<const uint32_t *>(p);
}

// (x.x, x.y) -> bf16 hi + lo pairs, low half = x.x
__device__ __forceinline__ void split2(float2 x, uint32_t &hi, uint32_t &lo) {
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(hi) : "f"(x.y), "f"(x.x));
    const float2 r = fsub2(x, unpack_bf16x2(hi));
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(lo) : "f"(r.y), "f"(r.x));
}

// (x.x, x.y) -> fp16 hi + lo pairs, low half = x.x
__device__ __forceinline__ void split2h(float2 x, uint32_t &hi, uint32_t &lo) {
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(hi) : "f"(x.y), "f"(x.x));
    float2 h;
    asm("{\n\t.reg .f16 a, b;\n\tmov.b32 {a, b}, %2;\n\tcvt.f32.f16 %0, a;\n\tcvt.f32.f16 %1, b;\n\t}"
        : "=f"(h.x), "=f"(h.y)
        : "r"(hi));
    const float2 r = fsub2(x, h);
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(lo) : "f"(r.y), "f"(r.x));
}

// RoPE pair (x0, x1) of a bf16x2 key factor word rotated by (cos, sin) = w, as fp16x2:
// (x0 c - x1 s, x0 s + x1 c), low half first.
__device__ __forceinline__ uint32_t rotate_to_h2(uint32_t v, float2 w) {
    const float2 x = unpack_bf16x2(v);
    const float y0 = x.x * w.x - x.y * w.y, y1 = x.x * w.y + x.y * w.x;
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(y1), "f"(y0));
    return r;
}

// (lo, hi) floats -> fp16x2 word, lo in the low half
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// A-factor fragments of the d1 = 8 decode for MT m-tiles: words (row half 0, 1) of each
// m-tile, two m-tiles per ldmatrix.x4 (4 x d1 rows of 16 bytes apart), an odd last one
// by ldmatrix.x2 (its lanes 0..15 give the row addresses).  abase: this lane's row.
template <int MT, int D1>
__device__ __forceinline__ void a_frags(uint32_t abase, uint32_t (&w)[MT][2]) {
#pragma unroll
    for (int mp = 0; mp < MT / 2; ++mp)
        ldsm_x4(abase + mp * 4 * D1 * 16, w[2 * mp][0], w[2 * mp][1], w[2 * mp + 1][0], w[2 * mp + 1][1]);
    if constexpr (MT % 2 == 1) ldsm_x2(abase + (MT / 2) * 4 * D1 * 16, w[MT - 1][0], w[MT - 1][1]);
}

// bf16x2 word -> fp16x2 word (exact for values in fp16's normal range)
__device__ __forceinline__ uint32_t bf16x2_to_h2(uint32_t v) {
    const float2 x = unpack_bf16x2(v);
    return pack_h2(x.x, x.y);
}

// 2^x on the special-function unit (ex2.approx: relative error about 2^-22; 2^-inf = 0)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// bf16 element of one token in a group row (2-byte load), widened by a shift
__device__ __forceinline__ float lds_bf16f(const unsigned char *p) {
    return __uint_as_float((uint32_t)*reinterpret_cast<const unsigned short *>(p) << 16);
}

__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
    return make_float2(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x);
}

// ------------------------------------------------------------------- kernel
template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
decode_mma_kernel(DecodeArgs a, RopeTable rope, DecodeTestHooks hooks) {
    constexpr int MA = C::MA, D1 = C::D1, D2 = C::D2, RK = C::RK, RV = C::RV, H2 = C::H2;
    constexpr int H1 = MA / D1, H = H1 * H2, DH = D1 * D2;
    // MR record rows (the cache's h1 d1; MA pads them to whole 16-row tiles), HR the
    // cache's heads: the query, the partials and the outputs have HR heads
    constexpr int MR = C::MR, HR1 = C::HR1, HR = C::HR, HS = C::HS;
    constexpr int MT = MA / 16, MTW = MT / HS, KS = D2 / 16, NT = D2 / 8;
    constexpr int EK = C::EK, EV = C::EV;
    constexpr int WARPS = C::WARPS, SLICES = C::SLICES, CHUNKS = C::CHUNKS, STAGES = C::STAGES;
    constexpr int TT = C::TT;
    constexpr int KBYTES = TT * EK * 2, STAGE_BYTES = C::STAGE_BYTES;
    constexpr int RED_LD = C::RED_LD;               // floats per token row of the j1 scratch
    constexpr int A_K = RK * MR, A_V = RV * MR;     // start of B in a key / value record
    // third order: query pair i = (head, m, jc) -> its first feature (head, 2m, jc); the
    // records' b and c factors start at A_K (A_V) and A_K + RK DB (A_V + RV DB)
    auto o3_pair_feature = [](int i) {
        constexpr int DCN = C::ORDER3 ? C::DC : 1;     // (1 keeps other shapes' unused copy defined)
        constexpr int PH = C::ORDER3 ? (C::DB / 2) * C::DC : 1;   // pairs per head
        const int h = i / PH, rem = i % PH;
        return h * DH + (rem / DCN) * 2 * DCN + rem % DCN;
    };
    constexpr int C_K = A_K + RK * C::DB, C_V = A_V + RV * C::DB;

    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char *stage_base = smem;                                           // ring
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BARS);          // full, empty
    float *qs = reinterpret_cast<float *>(smem + C::OFF_Q);                     // [H][Q_LD]
    float2 *cs = reinterpret_cast<float2 *>(smem + C::OFF_CS);                  // [D2/2]
    float *scratch = reinterpret_cast<float *>(smem + C::OFF_SCR);              // per warp
    volatile int *flags = reinterpret_cast<volatile int *>(smem + C::OFF_FLAGS);  // abort, last

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.y, split = blockIdx.x;
    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + STAGES);
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, WARPS);
        }
        for (int i = 0; i < 16; ++i) flags[i] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // Ahead of the dependency on the previous grid: hint this CTA's first ring of tiles
    // into L2.  A prefetch binds no data and L2 stays coherent with anything the
    // previous grid still writes, so it reads no input early; the cache streams in
    // while the previous call finishes (its split merge).  Only kernel parameters are
    // used here.  Slots [p0, p1) clipped to max_len, rounded up to whole 8-slot groups,
    // stay inside the cache (capacity >= max_len, a multiple of 8).  Only in a grid of
    // one wave (a.spec): with several waves a split past its sequence's end would read
    // its slots for nothing.
    if (tid == 0 && a.spec) {
        const int p0 = split * a.tps;
        const int p1 = min(p0 + STAGES * TT, a.max_len);
        if (p1 > p0) {
            const uint32_t groups = (uint32_t)((p1 - p0 + kGroup - 1) / kGroup);
            bulk_prefetch_l2(a.kc + ((size_t)b * a.cap + p0) * EK, groups * EK * kGroup * 2);
            bulk_prefetch_l2(a.vc + ((size_t)b * a.cap + p0) * EV, groups * EV * kGroup * 2);
        }
    }
    // launched with programmatic stream serialization: wait for the previous grid in
    // the stream before reading any input, and let the next grid be scheduled now
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");

    // In a grid of one wave the first tile's copy starts before the sequence length is
    // known: slots [t0, t0 + TT) clipped to max_len are inside the cache whatever the
    // length, and tokens past the length are masked later.
    const int t0 = split * a.tps;
    const int spec_n = min(TT, a.max_len - t0);
    const bool spec = a.spec && spec_n > 0 &&
                      !(hooks.skip_tile == 0 && split == hooks.skip_split && b == 0);
    if (tid == 0 && spec) {
        const int groups = (spec_n + kGroup - 1) / kGroup;
        const uint32_t kbytes = (uint32_t)groups * EK * kGroup * 2;
        const uint32_t vbytes = (uint32_t)groups * EV * kGroup * 2;
        const uint32_t dst = smem_u32(stage_base);
        mbar_expect_tx(full0, kbytes + vbytes);
        bulk_g2s(dst, a.kc + ((size_t)b * a.cap + t0) * EK, kbytes, full0);
        bulk_g2s(dst + KBYTES, a.vc + ((size_t)b * a.cap + t0) * EV, vbytes, full0);
    }

    // every input of the prologue is requested at once (one round trip)
    const bool rotate = a.q_pos != nullptr;
    int L = a.seq_len[b];
    const double qpos = rotate ? (double)a.q_pos[b] : 0.0;
    constexpr int QPT = (HR * DH / 2 + WARPS * 32 - 1) / (WARPS * 32);  // query pairs per thread
    __nv_bfloat162 qv[QPT];
    if (warp < WARPS && !a.qf) {
        const __nv_bfloat162 *qb = reinterpret_cast<const __nv_bfloat162 *>(a.q + (size_t)b * HR * DH);
#pragma unroll
        for (int k = 0; k < QPT; ++k) {
            const int i = tid + k * WARPS * 32;
            if (i < HR * DH / 2) {
                if constexpr (C::ORDER3) {
                    // third order: the RoPE pair of (head, m, c index) is features (2m DC + jc, + DC)
                    const int e0 = o3_pair_feature(i);
                    qv[k] = __halves2bfloat162(a.q[(size_t)b * HR * DH + e0], a.q[(size_t)b * HR * DH + e0 + C::DC]);
                } else {
                    qv[k] = qb[i];
                }
            }
        }
    }
    // query factors: the sequence's E_Q values (at most QF_PT per consumer thread) are
    // requested here, in the same round trip as the other inputs
    constexpr int QF_PT = C::QF_MAX / (WARPS * 32);
    const int eq = a.qf ? a.rq * (HR1 * D1 + H2 * D2) : 0;
    float qfv[QF_PT];
    if (warp < WARPS && a.qf) {
        const float *qfb = a.qf + (size_t)b * a.qf_seq_stride;
#pragma unroll
        for (int k = 0; k < QF_PT; ++k) {
            const int e = tid + k * WARPS * 32;
            qfv[k] = e < eq ? __ldg(qfb + (size_t)e * a.qf_stride) : 0.f;
        }
    }
    if (L > a.max_len || L < 0) {
        if (split == 0 && tid == 0) raise_error(a.err, kErrDeviceCheck);
        L = L < 0 ? 0 : a.max_len;
    }
    if (t0 >= L && !a.cluster) {                           // empty split (a cluster member stays)
        if (a.fused && L == 0 && split == 0)                // an empty sequence gets zeros
            for (int i = tid; i < HR * DH; i += C::THREADS) a.out[(size_t)b * HR * DH + i] = 0.f;
        if (tid == 0 && spec && !mbar_wait(full0, 0, hooks.wait_limit_ns))
            raise_error(a.err, kErrTimeout);               // its speculative copy lands first
        return;
    }
    // the last split runs to the end of the sequence (it may hold up to 5/4 of a split)
    const int t1 = max(t0, split == a.n_split - 1 ? L : min(t0 + a.tps, L));
    const int n_tiles = (t1 - t0 + TT - 1) / TT;
    __syncthreads();                                        // barriers initialised

    const uint64_t limit = hooks.wait_limit_ns;
    const __nv_bfloat16 *kb = a.kc + ((size_t)b * a.cap + t0) * EK;   // group-aligned (t0 % 8 == 0)
    const __nv_bfloat16 *vb = a.vc + ((size_t)b * a.cap + t0) * EV;

    // tile t of this split into stage t % STAGES (the test hook may withhold one)
    auto issue_tile = [&](int t) {
        const int s = t % STAGES;
        const int n = min(TT, t1 - t0 - t * TT);
        const int groups = (n + kGroup - 1) / kGroup;
        const uint32_t kbytes = (uint32_t)groups * EK * kGroup * 2;
        const uint32_t vbytes = (uint32_t)groups * EV * kGroup * 2;
        if (hooks.skip_tile == t && split == hooks.skip_split && b == 0) return;
        const uint32_t dst = smem_u32(stage_base + (size_t)s * STAGE_BYTES);
        mbar_expect_tx(full0 + 8 * s, kbytes + vbytes);
        bulk_g2s(dst, kb + (size_t)t * TT * EK, kbytes, full0 + 8 * s);
        bulk_g2s(dst + KBYTES, vb + (size_t)t * TT * EV, vbytes, full0 + 8 * s);
    };
    // every copy issued for this CTA (tiles below `issued`) lands before it exits
    auto drain = [&](int issued) {
        for (int t = max(0, issued - STAGES); t < issued; ++t) {
            if (hooks.skip_tile == t && split == hooks.skip_split && b == 0) continue;
            if (!mbar_wait(full0 + 8 * (t % STAGES), (t / STAGES) & 1, limit)) raise_error(a.err, kErrTimeout);
        }
    };
    if constexpr (!C::PRODUCER_WARP) {
        if (tid == 0) {                                    // the rest of the first ring
            const int first = min(STAGES, n_tiles);
            for (int t = spec ? 1 : 0; t < first; ++t) issue_tile(t);
            flags[2] = max(first, spec ? 1 : 0);
        }
    }

    // ------------------------------------------------------------ producer
    if (C::PRODUCER_WARP && warp == WARPS) {
        if (lane == 0) {
            int issued = spec ? 1 : 0;
            for (int t = spec ? 1 : 0; t < n_tiles; ++t) {
                const int s = t % STAGES;
                if (t >= STAGES && !mbar_wait(empty0 + 8 * s, ((t / STAGES) - 1) & 1, limit)) {
                    raise_error(a.err, kErrTimeout);
                    flags[0] = 1;
                    break;
                }
                if (flags[0]) break;
                issued = t + 1;
                issue_tile(t);
            }
            drain(issued);
        }
        if (!a.cluster) return;
    } else {

    // rotated, scaled query in fp32 (consumers, while the first copies are in flight):
    // I_{d1} (x) R^(2)(q_pos) on pairs (2m, 2m+1), angles tabulated once per CTA
    if (rotate && tid < D2 / 2) {
        float cth, sth;
        rope_cs_fast(qpos, rope.theta[tid], cth, sth);
        cs[tid] = make_float2(cth, sth);
    }
    asm volatile("bar.sync 1, %0;" ::"n"(WARPS * 32));
    if (a.qf) {
        // q = (1/R_Q) sum_r A^Q_r (x) B^Q_r assembled here from fp32 factors ("Kronecker
        // Product Attention", eq 2); the pairs (2m, 2m+1) of each d2 chunk are rotated after
        // the rank sum (the rotation is linear).  The factors are staged in the query's
        // shared-memory rows (E_Q <= H * Q_LD, checked by the host), the outputs are kept in
        // registers until every thread has read its factors, then written over them.
        // One thread per 8 features of a (head, j1) row.
        constexpr int CH = D2 / 8, ITEMS = HR * D1 * CH;
        constexpr int IPT = (ITEMS + WARPS * 32 - 1) / (WARPS * 32);
        static_assert(C::QF_MAX <= H * C::Q_LD, "query factors staged in the query rows");
#pragma unroll
        for (int k = 0; k < QF_PT; ++k) {
            const int e = tid + k * WARPS * 32;
            if (e < eq) qs[e] = qfv[k];
        }
        asm volatile("bar.sync 1, %0;" ::"n"(WARPS * 32));
        const int qa_b = a.rq * HR1 * D1;                 // first B^Q element of the record
        const float rs = a.qscale / (float)a.rq;
        float acc[IPT][8];
#pragma unroll
        for (int k = 0; k < IPT; ++k) {
#pragma unroll
            for (int u = 0; u < 8; ++u) acc[k][u] = 0.f;
            const int it = tid + k * WARPS * 32;
            if (it < ITEMS) {
                const int head = it / (D1 * CH), rem = it % (D1 * CH), j1 = rem / CH, j2 = (rem % CH) * 8;
                const int i1 = head / H2, i2h = head % H2;
                for (int r = 0; r < a.rq; ++r) {
                    const float av = qs[(r * HR1 + i1) * D1 + j1];
                    const float4 *bq = reinterpret_cast<const float4 *>(qs + qa_b + (r * H2 + i2h) * D2 + j2);
                    const float4 b0 = bq[0], b1 = bq[1];
                    acc[k][0] += av * b0.x;
                    acc[k][1] += av * b0.y;
                    acc[k][2] += av * b0.z;
                    acc[k][3] += av * b0.w;
                    acc[k][4] += av * b1.x;
                    acc[k][5] += av * b1.y;
                    acc[k][6] += av * b1.z;
                    acc[k][7] += av * b1.w;
                }
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(WARPS * 32));
#pragma unroll
        for (int k = 0; k < IPT; ++k) {
            const int it = tid + k * WARPS * 32;
            if (it < ITEMS) {
                const int head = it / (D1 * CH), rem = it % (D1 * CH), j1 = rem / CH, j2 = (rem % CH) * 8;
                float *dst = qs + head * C::Q_LD + j1 * D2 + j2;
#pragma unroll
                for (int u = 0; u < 8; u += 2) {
                    float y0 = acc[k][u], y1 = acc[k][u + 1];
                    if (rotate) {
                        const float2 w = cs[(j2 + u) >> 1];
                        y0 = acc[k][u] * w.x - acc[k][u + 1] * w.y;
                        y1 = acc[k][u] * w.y + acc[k][u + 1] * w.x;
                    }
                    *reinterpret_cast<float2 *>(dst + u) = make_float2(y0 * rs, y1 * rs);
                }
            }
        }
    }
#pragma unroll
    for (int k = 0; k < QPT; ++k) {
        const int i = tid + k * WARPS * 32;
        if (i < HR * DH / 2 && !a.qf) {
            const float2 x = __bfloat1622float2(qv[k]);
            float2 y = x;
            if constexpr (C::ORDER3) {
                // R_{d_b}(q_pos) (x) I_{d_c}: pair m of the b index, for every c index
                if (rotate) {
                    const float2 w = cs[(i % ((C::DB / 2) * C::DC)) / C::DC];
                    y = make_float2(x.x * w.x - x.y * w.y, x.x * w.y + x.y * w.x);
                }
                const int e = o3_pair_feature(i), qh = e / DH;
                qs[qh * C::Q_LD + (e - qh * DH)] = y.x * a.qscale;
                qs[qh * C::Q_LD + (e - qh * DH) + C::DC] = y.y * a.qscale;
            } else {
                if (rotate) {
                    const float2 w = cs[i % (D2 / 2)];
                    y = make_float2(x.x * w.x - x.y * w.y, x.x * w.y + x.y * w.x);
                }
                const int e = 2 * i, qh = e / DH;            // rows padded to Q_LD: no bank conflicts
                *reinterpret_cast<float2 *>(qs + qh * C::Q_LD + (e - qh * DH)) =
                    make_float2(y.x * a.qscale, y.y * a.qscale);
            }
        }
    }
    if constexpr (C::SHARED) {
        // theta_m and (cos, sin)(k theta_m), k < 16, for the in-kernel key rotation
        double *th = reinterpret_cast<double *>(smem + C::OFF_THETA);
        float2 *st = reinterpret_cast<float2 *>(smem + C::OFF_STEP);
        for (int i = tid; i < D2 / 2; i += WARPS * 32) th[i] = rope.theta[i];
        for (int i = tid; i < 16 * (D2 / 2); i += WARPS * 32) {
            const int k = i / (D2 / 2), m = i % (D2 / 2);
            float cth, sth;
            rope_cs_fast((double)k, rope.theta[m], cth, sth);
            st[i] = make_float2(cth, sth);
        }
    }
    if constexpr (HR < H)                                  // padded heads: zero query rows
        for (int i = tid; i < (H - HR) * C::Q_LD; i += WARPS * 32) qs[(size_t)HR * C::Q_LD + i] = 0.f;
    asm volatile("bar.sync 1, %0;" ::"n"(WARPS * 32));

    // ------------------------------------------------------------ consumers
    const int i2 = warp % H2, hs = (warp / H2) % HS, slice = warp / (H2 * HS);
    const int g = lane >> 2, c = lane & 3;
    float *mo = reinterpret_cast<float *>(smem);                   // [SLICES][H][DH] (after the loop)
    constexpr int MO_LD = C::MO_LD;
    float *mm = mo + SLICES * H * MO_LD;                           // [SLICES][H][2]
    float *cp = mm + SLICES * H * 2;                               // merged: [H][DH] o, [H] m, [H] l
    bool aborted = false;
    if constexpr (C::KPA8) {
    // d1 = 8.  Row g of m-tile mt stands for the query row (i1, j1) = (2 mt + (g >> 2),
    // 2 (g & 3)) and row g + 8 for (i1, j1 + 1): a lane's two rows belong to one head, so
    // after the A^K product both add into one score, the sum over j1 is two shuffle
    // levels (lanes g & 3), and every lane then holds the full scores, the weights p
    // and the softmax state of its head for its four tokens (2c, 2c + 1 of each
    // 8-token group).  The A-factor fragments are loaded with ldmatrix from the
    // permuted rows.  The value product P' B^V runs once in fp16: P' = p A^V is
    // rounded once to fp16 (relative 2^-11), B^V (bf16) converts to fp16 exactly in
    // fp16's normal range; a value outside fp16's range makes the partial non-finite,
    // which is reported as a device check.
    // d2 = 8: the score is one m16n8k8 per m-tile (A words 0, 1 of each fragment) and the
    // value product has one 8-column n-tile
    constexpr bool K8 = D2 == 8;
    constexpr int KQ = K8 ? 1 : KS, VQ = K8 ? 2 : 4;
    const int hi1 = g >> 2, jp = 2 * (g & 3);
    uint32_t qa_hi[MT][KQ][4], qa_lo[MT][KQ][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int ks = 0; ks < KQ; ++ks)
#pragma unroll
            for (int v = 0; v < VQ; ++v) {
                const int i1 = 2 * mt + hi1, j1 = jp + (v & 1);
                const int j2 = ks * 16 + 2 * c + ((v & 2) ? 8 : 0);
                const float *src = qs + (i1 * H2 + i2) * C::Q_LD + j1 * D2 + j2;
                split2(make_float2(src[0], src[1]), qa_hi[mt][ks][v], qa_lo[mt][ks][v]);
            }
    // ldmatrix row address (bytes inside a group) of this lane for the A factors: matrix
    // mj = (m-tile 2 mp + (mj >> 1), row half mj & 1) of m-tile pair mp, matrix row mrow
    const int mj = lane >> 3, mrow = lane & 7;
    const uint32_t a_off =
        (uint32_t)(((2 * (mj >> 1) + (mrow >> 2)) * D1 + 2 * (mrow & 3) + (mj & 1)) * 16);
    float o[MT][NT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
    float m_k[MT], l_k[MT];              // running max and this lane's share of the sum, head 2 mt + hi1
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        m_k[mt] = -INFINITY;
        l_k[mt] = 0.f;
    }

    for (int t = 0; t < n_tiles; ++t) {
        const int s = t % STAGES;
        if (!mbar_wait(full0 + 8 * s, (t / STAGES) & 1, limit)) {
            raise_error(a.err, kErrTimeout);
            flags[0] = 1;
            aborted = true;
            break;
        }
        const unsigned char *kt = stage_base + (size_t)s * STAGE_BYTES;
        const unsigned char *vt = kt + KBYTES;
        const int n_valid = min(TT, t1 - t0 - t * TT);
        const int tok_base = slice * CHUNKS * 16;

            // NC chunks of 16 tokens from tok0 on, with one softmax update: the score
            // products of the NC chunks are independent, so a warp has NC of them in
            // flight.  A chunk that ends past the tile's valid tokens (the ragged end of
            // a split, NC = 1) masks its scores and factors; full chunks carry none of
            // that code
            auto chunk = [&](auto tail_c, auto nc_c, const int tok0) {
                constexpr bool TAIL = decltype(tail_c)::value;
                constexpr int NC = decltype(nc_c)::value;
                static_assert(!TAIL || NC == 1, "a ragged chunk runs alone");
                // ---- scores of head 2 mt + hi1, tokens (gi, 2c) and (gi, 2c + 1) of chunk cc
                float2 sc[NC][MT][2];
    #pragma unroll
                for (int cc = 0; cc < NC; ++cc)
    #pragma unroll
                    for (int mt = 0; mt < MT; ++mt) sc[cc][mt][0] = sc[cc][mt][1] = make_float2(0.f, 0.f);
    #pragma unroll
                for (int cc = 0; cc < NC; ++cc)
    #pragma unroll
                for (int r = 0; r < RK; ++r) {
                    const unsigned char *kg0 = kt + (size_t)((tok0 + cc * 16) >> 3) * EK * 16;
    #pragma unroll
                    for (int gi = 0; gi < 2; ++gi) {
                        const unsigned char *grp = kg0 + (size_t)gi * EK * 16;
                        uint32_t bk[KQ][2];
                        const int e_b = A_K + r * H2 * D2 + i2 * D2;
                        if constexpr (K8) {
                            ldsm_x1_t(smem_u32(grp + (size_t)(e_b + (lane & 7)) * 16), bk[0][0]);
                        } else if constexpr (KS % 2 == 0) {
    #pragma unroll
                            for (int kp = 0; kp < KS / 2; ++kp)
                                ldsm_x4_t(smem_u32(grp + (size_t)(e_b + kp * 32 + lane) * 16), bk[2 * kp][0],
                                          bk[2 * kp][1], bk[2 * kp + 1][0], bk[2 * kp + 1][1]);
                        } else {
    #pragma unroll
                            for (int ks = 0; ks < KS; ++ks)
                                ldsm_x2_t(smem_u32(grp + (size_t)(e_b + ks * 16 + (lane & 15)) * 16), bk[ks][0],
                                          bk[ks][1]);
                        }
                        uint32_t ak[MT][2];
                        a_frags<MT, D1>(smem_u32(grp + (size_t)r * MR * 16) + a_off, ak);
    #pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
                            float acc[4] = {0.f, 0.f, 0.f, 0.f};
                            if constexpr (K8) {
                                mma16808(acc, qa_hi[mt][0][0], qa_hi[mt][0][1], bk[0][0]);
                                mma16808(acc, qa_lo[mt][0][0], qa_lo[mt][0][1], bk[0][0]);
                            } else {
    #pragma unroll
                                for (int ks = 0; ks < KS; ++ks) {
                                    mma16816(acc, qa_hi[mt][ks], bk[ks][0], bk[ks][1]);
                                    mma16816(acc, qa_lo[mt][ks], bk[ks][0], bk[ks][1]);
                                }
                            }
                            sc[cc][mt][gi] =
                                ffma2(make_float2(acc[0], acc[1]), unpack_bf16x2(ak[mt][0]), sc[cc][mt][gi]);
                            sc[cc][mt][gi] =
                                ffma2(make_float2(acc[2], acc[3]), unpack_bf16x2(ak[mt][1]), sc[cc][mt][gi]);
                        }
                    }
                }
                // ---- the sum over j1: lanes that differ in g & 3
    #pragma unroll
                for (int off = 4; off <= 8; off <<= 1)
    #pragma unroll
                    for (int cc = 0; cc < NC; ++cc)
    #pragma unroll
                    for (int mt = 0; mt < MT; ++mt)
    #pragma unroll
                        for (int gi = 0; gi < 2; ++gi) {
                            sc[cc][mt][gi].x += __shfl_xor_sync(0xffffffffu, sc[cc][mt][gi].x, off);
                            sc[cc][mt][gi].y += __shfl_xor_sync(0xffffffffu, sc[cc][mt][gi].y, off);
                        }
                if constexpr (TAIL) {
    #pragma unroll
                    for (int gi = 0; gi < 2; ++gi) {
                        const int tk = tok0 + gi * 8 + 2 * c;
    #pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
                            if (tk >= n_valid) sc[0][mt][gi].x = -INFINITY;
                            if (tk + 1 >= n_valid) sc[0][mt][gi].y = -INFINITY;
                        }
                    }
                }
                // ---- online softmax of this lane's head over the NC chunks' tokens
                bool grow = false;
                float alpha[MT];
    #pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    float mx = -INFINITY;
    #pragma unroll
                    for (int cc = 0; cc < NC; ++cc)
                        mx = fmaxf(mx, fmaxf(fmaxf(sc[cc][mt][0].x, sc[cc][mt][0].y),
                                             fmaxf(sc[cc][mt][1].x, sc[cc][mt][1].y)));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                    alpha[mt] = 1.f;
                    if (mx > m_k[mt]) {                     // finite: the chunk has a valid token
                        alpha[mt] = ex2_approx(m_k[mt] - mx);
                        m_k[mt] = mx;
                        grow = true;
                    }
                    const float m_new = m_k[mt];
                    float lsum = 0.f;
    #pragma unroll
                    for (int cc = 0; cc < NC; ++cc) {
    #pragma unroll
                        for (int gi = 0; gi < 2; ++gi) {
                            sc[cc][mt][gi].x = ex2_approx(sc[cc][mt][gi].x - m_new);
                            sc[cc][mt][gi].y = ex2_approx(sc[cc][mt][gi].y - m_new);
                        }
                        lsum += (sc[cc][mt][0].x + sc[cc][mt][0].y) + (sc[cc][mt][1].x + sc[cc][mt][1].y);
                    }
                    l_k[mt] = l_k[mt] * alpha[mt] + lsum;
                }
                if (__any_sync(0xffffffffu, grow)) {
    #pragma unroll
                    for (int mt = 0; mt < MT; ++mt)
    #pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
    #pragma unroll
                            for (int v = 0; v < 4; ++v) o[mt][nt][v] *= alpha[mt];
                }
                // ---- values: P'[(i1, j1), token] = p * A^V_r in fp16 (A operand: rows g, g + 8,
                // tokens 2c, 2c + 1 of group 0 then of group 1)
    #pragma unroll
                for (int cc = 0; cc < NC; ++cc)
    #pragma unroll
                for (int r = 0; r < RV; ++r) {
                    const unsigned char *g0p = vt + (size_t)((tok0 + cc * 16) >> 3) * EV * 16;
                    const unsigned char *g1p = g0p + (size_t)EV * 16;
                    uint32_t av[2][MT][2];
    #pragma unroll
                    for (int gi = 0; gi < 2; ++gi) {
                        a_frags<MT, D1>(smem_u32((gi ? g1p : g0p) + (size_t)r * MR * 16) + a_off, av[gi]);
                    }
                    uint32_t pa[MT][4];
    #pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
    #pragma unroll
                        for (int gi = 0; gi < 2; ++gi)
    #pragma unroll
                            for (int hr = 0; hr < 2; ++hr) {
                                float2 x = fmul2(sc[cc][mt][gi], unpack_bf16x2(av[gi][mt][hr]));
                                if constexpr (TAIL) {   // garbage factors of masked tokens stay out (their weight is 0)
                                    const int tk = tok0 + gi * 8 + 2 * c;
                                    if (tk >= n_valid) x.x = 0.f;
                                    if (tk + 1 >= n_valid) x.y = 0.f;
                                }
                                pa[mt][2 * gi + hr] = pack_h2(x.x, x.y);
                            }
                    }
                    const int e_b = A_V + r * H2 * D2 + i2 * D2;
                    const int mat = lane >> 3, mr = lane & 7;
                    if constexpr (K8) {
                        // one n-tile: matrices (group 0, group 1) of the 8 features, lanes 0..15
                        uint32_t b00, b01;
                        ldsm_x2(smem_u32(((mat & 1) ? g1p : g0p) + (size_t)(e_b + mr) * 16), b00, b01);
                        b00 = bf16x2_to_h2(b00);
                        b01 = bf16x2_to_h2(b01);
                        if constexpr (TAIL) {
                            const int tk = tok0 + 2 * c;
                            b00 = mask_pair(b00, tk < n_valid, tk + 1 < n_valid);
                            b01 = mask_pair(b01, tk + 8 < n_valid, tk + 9 < n_valid);
                        }
    #pragma unroll
                        for (int mt = 0; mt < MT; ++mt) mma16816h(o[mt][0], pa[mt], b00, b01);
                    }
    #pragma unroll
                    for (int np = 0; np < NT / 2; ++np) {
                        const unsigned char *gp = (mat & 1) ? g1p : g0p;
                        uint32_t b00, b01, b10, b11;
                        ldsm_x4(smem_u32(gp + (size_t)(e_b + (2 * np + (mat >> 1)) * 8 + mr) * 16), b00, b01, b10,
                                b11);
                        b00 = bf16x2_to_h2(b00);
                        b01 = bf16x2_to_h2(b01);
                        b10 = bf16x2_to_h2(b10);
                        b11 = bf16x2_to_h2(b11);
                        if constexpr (TAIL) {
                            const int tk = tok0 + 2 * c;
                            b00 = mask_pair(b00, tk < n_valid, tk + 1 < n_valid);
                            b10 = mask_pair(b10, tk < n_valid, tk + 1 < n_valid);
                            b01 = mask_pair(b01, tk + 8 < n_valid, tk + 9 < n_valid);
                            b11 = mask_pair(b11, tk + 8 < n_valid, tk + 9 < n_valid);
                        }
    #pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
                            mma16816h(o[mt][2 * np], pa[mt], b00, b01);
                            mma16816h(o[mt][2 * np + 1], pa[mt], b10, b11);
                        }
                    }
                }
        
            };
            if (n_valid >= tok_base + CHUNKS * 16) {
                chunk(std::false_type{}, std::integral_constant<int, CHUNKS>{}, tok_base);
            } else {
#pragma unroll 1
                for (int ch = 0; ch < CHUNKS; ++ch) {
                    const int tok0 = tok_base + ch * 16;
                    if (tok0 >= n_valid) break;
                    if (tok0 + 16 > n_valid)
                        chunk(std::true_type{}, std::integral_constant<int, 1>{}, tok0);
                    else
                        chunk(std::false_type{}, std::integral_constant<int, 1>{}, tok0);
                }
            }
        __syncwarp();
        if (lane == 0) {
            // the warp is done with stage s: the last of the WARPS releases issues tile
            // t + STAGES into it (acq_rel: every warp's reads of the stage come first)
            uint32_t old;
            asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], 1;"
                         : "=r"(old)
                         : "r"(smem_u32((const void *)(flags + 4 + s)))
                         : "memory");
            if ((old + 1) % WARPS == 0 && t + STAGES < n_tiles && !flags[0]) {
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                issue_tile(t + STAGES);
                flags[2] = t + STAGES + 1;
            }
        }
        if (flags[0]) { aborted = true; break; }
    }

    {   // fp16 operands of the value product: an out-of-range value makes the partial non-finite
        bool fin = true;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int v = 0; v < 4; ++v) fin = fin && isfinite(o[mt][nt][v]);
        if (!fin) raise_error(a.err, kErrDeviceCheck);
    }
    // the sum of each head over the lanes of its tokens (c); lanes g & 3 hold copies
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        l_k[mt] += __shfl_xor_sync(0xffffffffu, l_k[mt], 1);
        l_k[mt] += __shfl_xor_sync(0xffffffffu, l_k[mt], 2);
    }

    // merge the token slices of the CTA through shared memory (reuses the ring)
    asm volatile("bar.sync 1, %0;" ::"n"(WARPS * 32));
    if (tid == 0) drain(flags[2]);               // copies still in flight after an abort
    const bool ok = !(aborted || flags[0]);
    if (!ok && !a.cluster) return;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const int head = (2 * mt + hi1) * H2 + i2;
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            float *dst = mo + ((size_t)slice * H + head) * MO_LD + (jp + hr) * D2;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                *reinterpret_cast<float2 *>(dst + nt * 8 + 2 * c) =
                    make_float2(o[mt][nt][2 * hr], o[mt][nt][2 * hr + 1]);
        }
        if ((lane & 15) == 0) {
            mm[((size_t)slice * H + head) * 2] = m_k[mt];
            mm[((size_t)slice * H + head) * 2 + 1] = l_k[mt];
        }
    }
    } else {
    float *red = scratch + (size_t)warp * C::SCR_FLOATS;   // [16][RED_LD] j1 partials
    float *pbuf = red + 16 * RED_LD;                         // [H1][16] weights
    float *abuf = pbuf + H1 * 16;                            // [H1] rescale factors

    // query fragments (A operand, row = (i1, j1), k = j2), hi and lo parts
    uint32_t qa_hi[MTW][KS][4], qa_lo[MTW][KS][4];
#pragma unroll
    for (int mt = 0; mt < MTW; ++mt)
#pragma unroll
        for (int ks = 0; ks < KS; ++ks)
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const int row = (hs * MTW + mt) * 16 + g + ((v & 1) ? 8 : 0);
                const int j2 = ks * 16 + 2 * c + ((v & 2) ? 8 : 0);
                const int i1 = row / D1, j1 = row % D1;
                const float *src = qs + (i1 * H2 + i2) * C::Q_LD + j1 * D2 + j2;
                if constexpr (C::SHARED || C::ORDER3)
                    split2h(make_float2(src[0], src[1]), qa_hi[mt][ks][v], qa_lo[mt][ks][v]);
                else
                    split2(make_float2(src[0], src[1]), qa_hi[mt][ks][v], qa_lo[mt][ks][v]);
            }
    // shared B: the keys' factors are stored unrotated, so each 16-token chunk rotates
    // its B^K fragments at the tokens' slots ("Kronecker Product Attention", Def 2.3 and
    // Thm 2.4: rotating B rotates the key).  (cos, sin)((p0 + k) theta_m) is formed as
    // (cos, sin)(p0 theta_m) * (cos, sin)(k theta_m), the first per chunk, the second
    // from a per-CTA table of the 16 offsets k.
    const double *theta_s = reinterpret_cast<const double *>(smem + C::OFF_THETA);
    const float2 *step_s = reinterpret_cast<const float2 *>(smem + C::OFF_STEP);
    float2 *base_s = reinterpret_cast<float2 *>(smem + C::OFF_BASE) + (size_t)warp * (D2 / 2);

    float o[MTW][NT][4];
#pragma unroll
    for (int mt = 0; mt < MTW; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
    // softmax state: per owned row (D1 == 1: rows are heads) or per lane head (D1 > 1)
    float m_row[MTW][2], l_row[MTW][2];
#pragma unroll
    for (int mt = 0; mt < MTW; ++mt) {
        m_row[mt][0] = m_row[mt][1] = -INFINITY;
        l_row[mt][0] = l_row[mt][1] = 0.f;
    }
    constexpr int PPL = C::PPL;                 // (head, token) pairs per lane per chunk (D1 > 1)
    const int my_i1 = lane % H1;                // the head this lane scores (D1 > 1)
    float m_h = -INFINITY, l_h = 0.f;

    for (int t = 0; t < n_tiles; ++t) {
        const int s = t % STAGES;
        if (!mbar_wait(full0 + 8 * s, (t / STAGES) & 1, limit)) {
            raise_error(a.err, kErrTimeout);
            flags[0] = 1;
            aborted = true;
            break;
        }
        const unsigned char *kt = stage_base + (size_t)s * STAGE_BYTES;
        const unsigned char *vt = kt + KBYTES;
        const int n_valid = min(TT, t1 - t0 - t * TT);
        const int tok_base = slice * CHUNKS * 16;

#pragma unroll 1
        for (int ch = 0; ch < CHUNKS; ++ch) {
            const int tok0 = tok_base + ch * 16;
            if (tok0 >= n_valid) break;                       // rest of this warp's slice is past the tail
            const bool tail = tok0 + 16 > n_valid;
            const unsigned char *kg0 = kt + (size_t)(tok0 >> 3) * EK * 16;
            float2 rc[2][KS][2];          // shared B: (cos, sin) of this lane's pairs, tokens g and 8 + g
            if constexpr (C::SHARED) {
                const int p0 = t0 + t * TT + tok0;        // slot (= position) of the chunk's first token
                __syncwarp();                             // the previous chunk is done with base_s
                for (int m = lane; m < D2 / 2; m += 32) {
                    float cth, sth;
                    rope_cs_fast((double)p0, theta_s[m], cth, sth);
                    base_s[m] = make_float2(cth, sth);
                }
                __syncwarp();
#pragma unroll
                for (int gi = 0; gi < 2; ++gi)
#pragma unroll
                    for (int ks = 0; ks < KS; ++ks)
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            // fragment word hh of k-step ks holds features 16 ks + 8 hh + 2c, +1
                            const int m = 8 * ks + 4 * hh + c;
                            rc[gi][ks][hh] = cmul(base_s[m], step_s[(gi * 8 + g) * (D2 / 2) + m]);
                        }
            }
            // ---- scores: sc[mt][gi][v] = sum_r A^K_r * (Q_i2 B~^K_r), rows (i1,j1), tokens 2c, 2c+1
            float2 sc[MTW][2][2];
#pragma unroll
            for (int mt = 0; mt < MTW; ++mt)
#pragma unroll
                for (int gi = 0; gi < 2; ++gi) sc[mt][gi][0] = sc[mt][gi][1] = make_float2(0.f, 0.f);
#pragma unroll
            for (int r = 0; r < RK; ++r) {
#pragma unroll
                for (int gi = 0; gi < 2; ++gi) {
                    const unsigned char *grp = kg0 + (size_t)gi * EK * 16;
                    uint32_t bk[KS][2];
                    const int e_b = A_K + r * H2 * D2 + i2 * D2;
                    if constexpr (C::ORDER3) {
                        // the key's features b (x) c of token g, as the B fragment: word 0 of
                        // k-step ks holds features (2ks, 2c), (2ks, 2c+1), word 1 (2ks+1, 2c), (2ks+1, 2c+1)
                        const unsigned char *tg = grp + 2 * g;
                        const float c0 = lds_bf16f(tg + (size_t)(C_K + r * C::DC + 2 * c) * 16);
                        const float c1 = lds_bf16f(tg + (size_t)(C_K + r * C::DC + 2 * c + 1) * 16);
#pragma unroll
                        for (int ks = 0; ks < KS; ++ks) {
                            const float b0 = lds_bf16f(tg + (size_t)(A_K + r * C::DB + 2 * ks) * 16);
                            const float b1 = lds_bf16f(tg + (size_t)(A_K + r * C::DB + 2 * ks + 1) * 16);
                            bk[ks][0] = pack_h2(b0 * c0, b0 * c1);
                            bk[ks][1] = pack_h2(b1 * c0, b1 * c1);
                        }
                    } else if constexpr (KS % 2 == 0) {
#pragma unroll
                        for (int kp = 0; kp < KS / 2; ++kp)
                            ldsm_x4_t(smem_u32(grp + (size_t)(e_b + kp * 32 + lane) * 16), bk[2 * kp][0],
                                      bk[2 * kp][1], bk[2 * kp + 1][0], bk[2 * kp + 1][1]);
                    } else {
#pragma unroll
                        for (int ks = 0; ks < KS; ++ks)
                            ldsm_x2_t(smem_u32(grp + (size_t)(e_b + ks * 16 + (lane & 15)) * 16), bk[ks][0],
                                      bk[ks][1]);
                    }
                    if constexpr (C::SHARED) {
#pragma unroll
                        for (int ks = 0; ks < KS; ++ks) {
                            bk[ks][0] = rotate_to_h2(bk[ks][0], rc[gi][ks][0]);
                            bk[ks][1] = rotate_to_h2(bk[ks][1], rc[gi][ks][1]);
                        }
                    }
#pragma unroll
                    for (int mt = 0; mt < MTW; ++mt) {
                        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int ks = 0; ks < KS; ++ks) {
                            if constexpr (C::SHARED || C::ORDER3) {
                                mma16816h(acc, qa_hi[mt][ks], bk[ks][0], bk[ks][1]);
                                mma16816h(acc, qa_lo[mt][ks], bk[ks][0], bk[ks][1]);
                            } else {
                                mma16816(acc, qa_hi[mt][ks], bk[ks][0], bk[ks][1]);
                                mma16816(acc, qa_lo[mt][ks], bk[ks][0], bk[ks][1]);
                            }
                        }
                        if constexpr (C::SHARED || C::ORDER3) {
                            // a valid token whose fp16 key factors left the fp16 range
                            const int tk = tok0 + gi * 8 + 2 * c;
                            if ((tk < n_valid && !(isfinite(acc[0]) && isfinite(acc[2]))) ||
                                (tk + 1 < n_valid && !(isfinite(acc[1]) && isfinite(acc[3]))))
                                raise_error(a.err, kErrDeviceCheck);
                        }
                        const int row0 = (hs * MTW + mt) * 16 + g;
                        const float2 a0 = unpack_bf16x2(lds_u32(grp + (size_t)(r * MR + row0) * 16 + 4 * c));
                        const float2 a1 = unpack_bf16x2(lds_u32(grp + (size_t)(r * MR + row0 + 8) * 16 + 4 * c));
                        sc[mt][gi][0] = ffma2(make_float2(acc[0], acc[1]), a0, sc[mt][gi][0]);
                        sc[mt][gi][1] = ffma2(make_float2(acc[2], acc[3]), a1, sc[mt][gi][1]);
                    }
                }
            }

            // ---- online softmax for this chunk; afterwards sc holds the weights p
            if constexpr (D1 == 1) {
                // rows are heads: row g of m-tile mt is head mt*16+g, row g+8 head mt*16+g+8
#pragma unroll
                for (int mt = 0; mt < MTW; ++mt)
#pragma unroll
                    for (int hr = 0; hr < 2; ++hr) {
                        if (tail) {
#pragma unroll
                            for (int gi = 0; gi < 2; ++gi) {
                                const int tk = tok0 + gi * 8 + 2 * c;
                                if (tk >= n_valid) sc[mt][gi][hr].x = -INFINITY;
                                if (tk + 1 >= n_valid) sc[mt][gi][hr].y = -INFINITY;
                            }
                        }
                        float mx = fmaxf(fmaxf(sc[mt][0][hr].x, sc[mt][0][hr].y),
                                         fmaxf(sc[mt][1][hr].x, sc[mt][1][hr].y));
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                        const float m_new = fmaxf(m_row[mt][hr], mx);   // finite: chunk has a valid token
                        const float alpha = exp2f(m_row[mt][hr] - m_new);
                        float sum = 0.f;
#pragma unroll
                        for (int gi = 0; gi < 2; ++gi) {
                            sc[mt][gi][hr].x = exp2f(sc[mt][gi][hr].x - m_new);
                            sc[mt][gi][hr].y = exp2f(sc[mt][gi][hr].y - m_new);
                            sum += sc[mt][gi][hr].x + sc[mt][gi][hr].y;
                        }
                        l_row[mt][hr] = l_row[mt][hr] * alpha + sum;
                        m_row[mt][hr] = m_new;
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            o[mt][nt][2 * hr] *= alpha;
                            o[mt][nt][2 * hr + 1] *= alpha;
                        }
                    }
            } else {
                // sum over j1 once per (head, token): partials through the warp's scratch
#pragma unroll
                for (int mt = 0; mt < MTW; ++mt)
#pragma unroll
                    for (int gi = 0; gi < 2; ++gi) {
                        const int tk = gi * 8 + 2 * c, row = (hs * MTW + mt) * 16 + g;
                        red[tk * RED_LD + row] = sc[mt][gi][0].x;
                        red[(tk + 1) * RED_LD + row] = sc[mt][gi][0].y;
                        red[tk * RED_LD + row + 8] = sc[mt][gi][1].x;
                        red[(tk + 1) * RED_LD + row + 8] = sc[mt][gi][1].y;
                    }
                __syncwarp();
                float sp[PPL];
                float mx = -INFINITY;
#pragma unroll
                for (int k = 0; k < PPL; ++k) {
                    const int tk = (lane + 32 * k) / H1;
                    const float *src = red + tk * RED_LD + my_i1 * D1;
                    float v = 0.f;
                    if constexpr (D1 % 4 == 0) {
#pragma unroll
                        for (int j = 0; j < D1; j += 4) {
                            const float4 f = *reinterpret_cast<const float4 *>(src + j);
                            v += (f.x + f.y) + (f.z + f.w);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < D1; ++j) v += src[j];
                    }
                    if (tail && tok0 + tk >= n_valid) v = -INFINITY;
                    sp[k] = v;
                    mx = fmaxf(mx, v);
                }
#pragma unroll
                for (int off = H1; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                const float m_new = fmaxf(m_h, mx);
                const float alpha = exp2f(m_h - m_new);
                float sum = 0.f;
#pragma unroll
                for (int k = 0; k < PPL; ++k) {
                    const float p = exp2f(sp[k] - m_new);
                    sum += p;
                    pbuf[my_i1 * 16 + (lane + 32 * k) / H1] = p;
                }
                l_h = l_h * alpha + sum;
                m_h = m_new;
                if (lane < H1) abuf[lane] = alpha;
                __syncwarp();
#pragma unroll
                for (int mt = 0; mt < MTW; ++mt)
#pragma unroll
                    for (int hr = 0; hr < 2; ++hr) {
                        const int i1 = ((hs * MTW + mt) * 16 + g + 8 * hr) / D1;
                        const float al = abuf[i1];
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            o[mt][nt][2 * hr] *= al;
                            o[mt][nt][2 * hr + 1] *= al;
                        }
#pragma unroll
                        for (int gi = 0; gi < 2; ++gi)
                            sc[mt][gi][hr] = *reinterpret_cast<const float2 *>(pbuf + i1 * 16 + gi * 8 + 2 * c);
                    }
            }

            // ---- values: P'[(i1,j1), k] = p * A^V_r, k = (group, token), hi/lo bf16 parts
            const unsigned char *g0p = vt + (size_t)(tok0 >> 3) * EV * 16;
            const unsigned char *g1p = g0p + (size_t)EV * 16;
#pragma unroll
            for (int r = 0; r < RV; ++r) {
                uint32_t pa_hi[MTW][4], pa_lo[MTW][4];
#pragma unroll
                for (int mt = 0; mt < MTW; ++mt) {
                    const int row0 = (hs * MTW + mt) * 16 + g;
                    const uint32_t w00 = lds_u32(g0p + (size_t)(r * MR + row0) * 16 + 4 * c);
                    const uint32_t w10 = lds_u32(g0p + (size_t)(r * MR + row0 + 8) * 16 + 4 * c);
                    const uint32_t w01 = lds_u32(g1p + (size_t)(r * MR + row0) * 16 + 4 * c);
                    const uint32_t w11 = lds_u32(g1p + (size_t)(r * MR + row0 + 8) * 16 + 4 * c);
                    float2 x0 = fmul2(sc[mt][0][0], unpack_bf16x2(w00));
                    float2 x1 = fmul2(sc[mt][0][1], unpack_bf16x2(w10));
                    float2 x2 = fmul2(sc[mt][1][0], unpack_bf16x2(w01));
                    float2 x3 = fmul2(sc[mt][1][1], unpack_bf16x2(w11));
                    if (tail) {   // keep garbage factors of masked tokens out (their weight is 0)
                        const int tk = tok0 + 2 * c;
                        if (tk >= n_valid) { x0.x = 0.f; x1.x = 0.f; }
                        if (tk + 1 >= n_valid) { x0.y = 0.f; x1.y = 0.f; }
                        if (tk + 8 >= n_valid) { x2.x = 0.f; x3.x = 0.f; }
                        if (tk + 9 >= n_valid) { x2.y = 0.f; x3.y = 0.f; }
                    }
                    if constexpr (C::ORDER3) {       // fp16 operands: the values' b (x) c are fp16
                        split2h(x0, pa_hi[mt][0], pa_lo[mt][0]);
                        split2h(x1, pa_hi[mt][1], pa_lo[mt][1]);
                        split2h(x2, pa_hi[mt][2], pa_lo[mt][2]);
                        split2h(x3, pa_hi[mt][3], pa_lo[mt][3]);
                    } else {
                        split2(x0, pa_hi[mt][0], pa_lo[mt][0]);
                        split2(x1, pa_hi[mt][1], pa_lo[mt][1]);
                        split2(x2, pa_hi[mt][2], pa_lo[mt][2]);
                        split2(x3, pa_hi[mt][3], pa_lo[mt][3]);
                    }
                }
                // B^V: the value record's B, or (shared) the key record's unrotated B
                const int e_b = (C::SHARED ? A_K : A_V) + r * H2 * D2 + i2 * D2;
                const unsigned char *b0p = C::SHARED ? kg0 : g0p;
                const unsigned char *b1p = C::SHARED ? kg0 + (size_t)EK * 16 : g1p;
                const int mat = lane >> 3, mrow = lane & 7;
                // third order: c^V of feature g for this lane's tokens (2c, 2c+1 of both groups)
                float2 cv0 = make_float2(0.f, 0.f), cv1 = cv0;
                if constexpr (C::ORDER3) {
                    cv0 = unpack_bf16x2(lds_u32(g0p + (size_t)(C_V + r * C::DC + g) * 16 + 4 * c));
                    cv1 = unpack_bf16x2(lds_u32(g1p + (size_t)(C_V + r * C::DC + g) * 16 + 4 * c));
                }
#pragma unroll
                for (int np = 0; np < NT / 2; ++np) {
                    const unsigned char *gp = (mat & 1) ? b1p : b0p;
                    uint32_t b00, b01, b10, b11;
                    if constexpr (C::ORDER3) {
                        // features 16 np + g (b index 2np) and 16 np + 8 + g (b index 2np + 1), c index g
                        const int eb = A_V + r * C::DB + 2 * np;
                        const float2 p00 = fmul2(unpack_bf16x2(lds_u32(g0p + (size_t)eb * 16 + 4 * c)), cv0);
                        const float2 p01 = fmul2(unpack_bf16x2(lds_u32(g1p + (size_t)eb * 16 + 4 * c)), cv1);
                        const float2 p10 = fmul2(unpack_bf16x2(lds_u32(g0p + (size_t)(eb + 1) * 16 + 4 * c)), cv0);
                        const float2 p11 = fmul2(unpack_bf16x2(lds_u32(g1p + (size_t)(eb + 1) * 16 + 4 * c)), cv1);
                        b00 = pack_h2(p00.x, p00.y);
                        b01 = pack_h2(p01.x, p01.y);
                        b10 = pack_h2(p10.x, p10.y);
                        b11 = pack_h2(p11.x, p11.y);
                    } else {
                        ldsm_x4(smem_u32(gp + (size_t)(e_b + (2 * np + (mat >> 1)) * 8 + mrow) * 16), b00, b01,
                                b10, b11);
                    }
                    if (tail) {
                        const int tk = tok0 + 2 * c;
                        b00 = mask_pair(b00, tk < n_valid, tk + 1 < n_valid);
                        b10 = mask_pair(b10, tk < n_valid, tk + 1 < n_valid);
                        b01 = mask_pair(b01, tk + 8 < n_valid, tk + 9 < n_valid);
                        b11 = mask_pair(b11, tk + 8 < n_valid, tk + 9 < n_valid);
                    }
#pragma unroll
                    for (int mt = 0; mt < MTW; ++mt) {
                        if constexpr (C::ORDER3) {
                            mma16816h(o[mt][2 * np], pa_hi[mt], b00, b01);
                            mma16816h(o[mt][2 * np], pa_lo[mt], b00, b01);
                            mma16816h(o[mt][2 * np + 1], pa_hi[mt], b10, b11);
                            mma16816h(o[mt][2 * np + 1], pa_lo[mt], b10, b11);
                            continue;
                        }
                        mma16816(o[mt][2 * np], pa_hi[mt], b00, b01);
                        mma16816(o[mt][2 * np], pa_lo[mt], b00, b01);
                        mma16816(o[mt][2 * np + 1], pa_hi[mt], b10, b11);
                        mma16816(o[mt][2 * np + 1], pa_lo[mt], b10, b11);
                    }
                }
            }
            if constexpr (D1 > 1) __syncwarp();    // scratch is rewritten by the next chunk
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * s);
        if (flags[0]) { aborted = true; break; }
    }

    if constexpr (C::ORDER3) {
        // the values' fp16 features b (x) c: an overflow makes the partial non-finite
        bool fin = true;
#pragma unroll
        for (int mt = 0; mt < MTW; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int v = 0; v < 4; ++v) fin = fin && isfinite(o[mt][nt][v]);
        if (!fin) raise_error(a.err, kErrDeviceCheck);
    }

    // l: complete sums per head
    if constexpr (D1 == 1) {
#pragma unroll
        for (int mt = 0; mt < MTW; ++mt)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                float l = l_row[mt][hr];
                l += __shfl_xor_sync(0xffffffffu, l, 1);
                l += __shfl_xor_sync(0xffffffffu, l, 2);
                l_row[mt][hr] = l;
            }
    } else {
#pragma unroll
        for (int off = H1; off < 32; off <<= 1) l_h += __shfl_xor_sync(0xffffffffu, l_h, off);
    }

    // merge the token slices of the CTA through shared memory (reuses the ring)
    asm volatile("bar.sync 1, %0;" ::"n"(WARPS * 32));
    const bool ok = !(aborted || flags[0]);
    if (!ok && !a.cluster) return;
#pragma unroll
    for (int mt = 0; mt < MTW; ++mt)
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const int row = (hs * MTW + mt) * 16 + g + 8 * hr;
            const int i1 = row / D1, j1 = row % D1;
            const int head = i1 * H2 + i2;
            float *dst = mo + ((size_t)slice * H + head) * MO_LD + j1 * D2;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                *reinterpret_cast<float2 *>(dst + nt * 8 + 2 * c) =
                    make_float2(o[mt][nt][2 * hr], o[mt][nt][2 * hr + 1]);
            if constexpr (D1 == 1) {
                if (c == 0) {
                    mm[((size_t)slice * H + head) * 2] = m_row[mt][hr];
                    mm[((size_t)slice * H + head) * 2 + 1] = l_row[mt][hr];
                }
            }
        }
    if constexpr (D1 > 1) {
        if (lane < H1) {
            const int head = lane * H2 + i2;
            mm[((size_t)slice * H + head) * 2] = m_h;
            mm[((size_t)slice * H + head) * 2 + 1] = l_h;
        }
    }
    }  // KPA8
    asm volatile("bar.sync 1, %0;" ::"n"(WARPS * 32));
    float *po = a.part_o + ((size_t)(b * a.n_split + split) * HR) * DH;
    float *pml = a.part_ml + ((size_t)(b * a.n_split + split) * HR) * 2;
    // One float4 column of the merged partial per thread.  Each thread forms the
    // log-sum-exp weights 2^(m_slice - M) of its own head from the slice statistics,
    // so the merge needs no further barrier.
    constexpr int N4 = HR * DH / 4;                  // the cache's heads (padded ones dropped)
    static_assert(DH % 4 == 0 && (MO_LD % 4) == 0 && ((size_t)SLICES * H * (MO_LD + 2)) % 4 == 0,
                  "float4 columns of the slice-merge buffer and of the merged partial");
    for (int c4 = tid; c4 < N4; c4 += WARPS * 32) {
        const int head = (c4 * 4) / DH, col = c4 * 4 - head * DH;
        float4 acc;
        float M, l;
        if constexpr (SLICES > 1) {
            M = -INFINITY;
#pragma unroll
            for (int sl = 0; sl < SLICES; ++sl) M = fmaxf(M, mm[((size_t)sl * H + head) * 2]);
            l = 0.f;
            acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int sl = 0; sl < SLICES; ++sl) {
                const float2 ms = *reinterpret_cast<const float2 *>(mm + ((size_t)sl * H + head) * 2);
                const float w = ms.x == -INFINITY ? 0.f : exp2f(ms.x - M);
                const float4 v = *reinterpret_cast<const float4 *>(mo + ((size_t)sl * H + head) * MO_LD + col);
                l += w * ms.y;
                acc.x += w * v.x;
                acc.y += w * v.y;
                acc.z += w * v.z;
                acc.w += w * v.w;
            }
        } else {
            M = mm[head * 2];
            l = mm[head * 2 + 1];
            acc = *reinterpret_cast<const float4 *>(mo + (size_t)head * MO_LD + col);
        }
        if (a.cluster) {
            *reinterpret_cast<float4 *>(cp + c4 * 4) = acc;
            if (col == 0) {
                cp[HR * DH + head] = M;
                cp[HR * DH + HR + head] = l;
            }
        } else {
            reinterpret_cast<float4 *>(po)[c4] = acc;
            if (col == 0) *reinterpret_cast<float2 *>(pml + 2 * head) = make_float2(M, l);
        }
    }
    if (!a.cluster) {
    if (!a.fused) return;

    // the last CTA of this sequence merges every split (log-sum-exp) into out[b]
    asm volatile("bar.sync 1, %0;" ::"n"(WARPS * 32));
    const int n_b = min(a.n_split, (L + a.tps - 1) / a.tps);   // splits holding tokens of b
    if (tid == 0) {
        // acq_rel at gpu scope: releases the CTA's partial (ordered before this thread
        // by the barrier above) and, for the last arrival, acquires every other CTA's
        int old;
        asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(old) : "l"(a.counters + b) : "memory");
        flags[1] = (old == n_b - 1) ? 1 : 0;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(WARPS * 32));
    if (!flags[1]) return;
    merge_split_partials<HR, DH>(a.part_o, a.part_ml, a.n_split, n_b, b, a.out_scale, a.out, tid, WARPS * 32);
    if (tid == 0) a.counters[b] = 0;                 // ready for the next call
    return;
    }  // global merge
    }  // consumers

    // ---- cluster merge: the CTAs of a cluster are the splits of one sequence. Each
    // keeps its merged partial in shared memory; after a cluster barrier every CTA
    // combines a slice of the outputs, reading its peers' partials over DSMEM.
    cg::cluster_group cl = cg::this_cluster();
    cl.sync();
    if (warp < WARPS) {
        const int n_cl = (int)cl.num_blocks(), rank = (int)cl.block_rank();
        const int per = (HR * DH + n_cl - 1) / n_cl;
        const int lo = rank * per, hi = min(HR * DH, lo + per);
        float *cpl = reinterpret_cast<float *>(smem) + SLICES * H * C::MO_LD + SLICES * H * 2;
        for (int idx = lo + tid; idx < hi; idx += WARPS * 32) {
            const int head = idx / DH;
            float M = -INFINITY;
            for (int r = 0; r < n_cl; ++r) M = fmaxf(M, cl.map_shared_rank(cpl, r)[HR * DH + head]);
            float num = 0.f, den = 0.f;
            for (int r = 0; r < n_cl; ++r) {
                const float *rp = cl.map_shared_rank(cpl, r);
                const float m = rp[HR * DH + head];
                const float w = m == -INFINITY ? 0.f : exp2f(m - M);
                num += w * rp[idx];
                den += w * rp[HR * DH + HR + head];
            }
            a.out[(size_t)b * HR * DH + idx] = den > 0.f ? a.out_scale * num / den : 0.f;
        }
    }
    cl.sync();                                       // peers read this CTA's shared memory
}

template <class C>
cudaError_t launch_cfg(const DecodeArgs &args, int batch, const DecodePlan &p, const RopeTable &rope,
                       const DecodeTestHooks &hooks, cudaStream_t st) {
    const size_t smem = C::smem_bytes();
    cudaError_t e = ensure_dynamic_smem<decode_mma_kernel<C>>(smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3((unsigned)p.n_split, (unsigned)batch);
    lc.blockDim = dim3(C::THREADS);
    lc.dynamicSmemBytes = smem;
    lc.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = args.cluster ? (unsigned)p.n_split : 1u;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    lc.attrs = attr;
    lc.numAttrs = 2;
    return cudaLaunchKernelEx(&lc, decode_mma_kernel<C>, args, rope, hooks);
}

// Can a cluster of `size` CTAs of this variant run on this device?
template <class C>
int cluster_ok_cfg(int size) {
    const size_t smem = C::smem_bytes();
    if (ensure_dynamic_smem<decode_mma_kernel<C>>(smem) != cudaSuccess) return 0;
    if (size > 8 &&
        cudaFuncSetAttribute(decode_mma_kernel<C>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
            cudaSuccess)
        return 0;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3((unsigned)size, 1);
    lc.blockDim = dim3(C::THREADS);
    lc.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)size;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, decode_mma_kernel<C>, &lc) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

}  // namespace

int mma_decode_max_clusters(int variant, int size) {
    switch (variant) {
#define KPA_MMA_CL(IDX, CFG) \
    case IDX:                \
        return cluster_ok_cfg<CFG>(size);
        KPA_MMA_VARIANTS(KPA_MMA_CL)
#undef KPA_MMA_CL
        default:
            return 0;
    }
}

cudaError_t launch_decode_mma(int variant, const DecodeArgs &args, int batch, const DecodePlan &plan,
                              const RopeTable &rope, const DecodeTestHooks &hooks, cudaStream_t st) {
    switch (variant) {
#define KPA_MMA_CASE(IDX, CFG) \
    case IDX:                  \
        return launch_cfg<CFG>(args, batch, plan, rope, hooks, st);
        KPA_MMA_VARIANTS(KPA_MMA_CASE)
#undef KPA_MMA_CASE
        default:
            return cudaErrorInvalidValue;
    }
}

}  // namespace kpa
