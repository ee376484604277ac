// kpa_prefill_mma.cu -- causal prefill in factor space for any Kronecker split of
// order 2 with d_h <= 128 ("Kronecker Product Attention", section 2.2: eq 4 for the
// keys and values of a head, Proposition 2.2 for the scores; the TPA split h1 = h,
// h2 = 1, d1 = 1 of the last paragraph of that section is one case).  The tcgen05
// prefill covers the d1 = 8, d2 = 16, R = 2 split; this kernel takes every other one.
//
// One CTA takes 128 query rows of one head of one sequence (8 warps x 16 rows) and
// walks key slots 0 .. (its last row's position) in tiles of 64:
//   - all threads copy the head's slices of the next tile's factor records into a
//     two-stage ring (cp.async, 16-byte vectors of one element's 8 tokens);
//   - the CTA rebuilds the tile's K_h and V_h = sum_r A_r (x) B_r in fp32, rounded once
//     to fp16, feature-major into shared memory; a shared B is rotated at each slot's
//     position for the keys only (Theorem 2.4); slots past the CTA's last position
//     are written as zeros;
//   - each warp forms S = Q K^T for its 16 rows on mma.sync m16n8k16 (fp16 operands,
//     fp32 accumulators), applies the causal mask and the online softmax in registers
//     and adds P V (P rounded to fp16) into its fp32 output tile.
// The scores carry sm_scale / R_K log2(e) folded into Q before it is rounded to fp16;
// the output is scaled by 1 / R_V.  Rows whose position is outside the cache are
// written as zeros and raise the device-check error; so does an output made non-finite
// by a value outside the fp16 range.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "kpa_f32x2.cuh"
#include "kpa_prefill_mma.cuh"
#include "kpa_sm100.cuh"

namespace kpa {
namespace {

using sm100::cp_async16;
using sm100::smem_u32;
using f32x2::ffma2;
using f32x2::unpack_bf16x2;

constexpr int kRows = 128;     // query rows per CTA
constexpr int kSlots = 64;     // key slots per tile (8 token groups)
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

struct PrefillMmaArgs {
    const __nv_bfloat16 *q;     // dense rotated query [B][n][h][d_h], or null
    const float *qf;            // query factors (when q is null)
    long long qf_stride, qf_seq_stride, qf_tok_stride;
    const int32_t *start_pos;
    const __nv_bfloat16 *kc, *vc;
    float *out;
    int *err;
    int n_tok, cap;
    int h1, h2, d1, d2, dh, rk, rv, rq;
    int ek, ev;                 // elements per key / value record
    int shared;                 // one B for keys and values (cached unrotated)
    int ekh, evh;               // one head's slice of a key / value record, in elements
    int ekp, evp;               // stage stride of a token group's slice, in 16-byte vectors (odd)
    int nch;                    // 4-column chunks of a B row: ceil(d2 / 4)
    float qscale, qf_scale, out_scale;
};

// Shared-memory layout (bytes): K tile, V tile (feature-major, 64 slots = 128 B per
// feature row), then a region that first holds Q and then the factor stages, the
// slice -> record element table and (shared B) the RoPE frequencies.
struct PrefillMmaLayout {
    int ks, vs, x, tab, theta, total;
};

__host__ __device__ inline PrefillMmaLayout prefill_mma_layout(int DH, int ekh, int evh, int ekp, int evp,
                                                               int d2) {
    PrefillMmaLayout L;
    L.ks = 0;
    L.vs = DH * 128;
    L.x = 2 * DH * 128;
    const int qb = kRows * DH * 2, sb = 2 * 8 * (ekp + evp) * 16;
    L.tab = L.x + (qb > sb ? qb : sb);
    L.theta = L.tab + ((ekh + evh) * 4 + 15) / 16 * 16;
    L.total = L.theta + (d2 / 2) * 8;
    return L;
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

__device__ __forceinline__ float ex2f(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}

__device__ __forceinline__ void ldsm4_t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}

// d += a b for one 16 x 8 x 16 tile: a row-major 16 x 16 fp16, b 16 x 8 fp16 (k pairs), d fp32
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void unpack8(const uint4 v, float2 (&x)[4]) {
    x[0] = unpack_bf16x2(v.x);
    x[1] = unpack_bf16x2(v.y);
    x[2] = unpack_bf16x2(v.z);
    x[3] = unpack_bf16x2(v.w);
}

template <int DH>
__global__ void __launch_bounds__(kThreads, 1) prefill_mma_kernel(const PrefillMmaArgs a, const RopeTable rope) {
    static_assert(DH == 64 || DH == 128, "feature tile");
    constexpr int NC = DH / 8;        // 16-byte chunks of a Q row
    constexpr int KS = DH / 16;       // k-steps of Q K^T
    extern __shared__ __align__(128) unsigned char smem[];
    const PrefillMmaLayout L = prefill_mma_layout(DH, a.ekh, a.evh, a.ekp, a.evp, a.d2);
    unsigned char *Ks = smem + L.ks, *Vs = smem + L.vs, *X = smem + L.x;
    int *tab = reinterpret_cast<int *>(smem + L.tab);
    double *theta = reinterpret_cast<double *>(smem + L.theta);
    const int stage_bytes = 8 * (a.ekp + a.evp) * 16;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_qt = (a.n_tok + kRows - 1) / kRows;
    const int qt = n_qt - 1 - (int)blockIdx.x;                   // longest rows first
    const int head = blockIdx.y, b = blockIdx.z;
    const int h = a.h1 * a.h2, i1 = head / a.h2, i2 = head % a.h2;
    const int q0 = qt * kRows;
    const int last_row = min(q0 + kRows, a.n_tok) - 1;
    const int start = a.start_pos[b];
    if (tid == 0 && (start < 0 || (long long)start + last_row >= a.cap)) raise_error(a.err, kErrDeviceCheck);

    float *out_b = a.out + ((size_t)b * a.n_tok) * h * a.dh;
    if (start < 0) {                                             // no row has a valid position
        for (int idx = tid; idx < (last_row - q0 + 1) * a.dh; idx += kThreads) {
            const int r = idx / a.dh, f = idx - r * a.dh;
            out_b[((size_t)(q0 + r) * h + head) * a.dh + f] = 0.f;
        }
        return;
    }
    const int max_slot = (int)min((long long)start + last_row, (long long)a.cap - 1);
    const int n_kt = max_slot / kSlots + 1;

    // ---- prologue: slice table, frequencies, zero feature rows d_h .. DH-1, Q tile
    for (int e = tid; e < a.ekh + a.evh; e += kThreads) {
        const bool v = e >= a.ekh;
        const int ee = v ? e - a.ekh : e, R = v ? a.rv : a.rk;
        int off;
        if (ee < R * a.d1)
            off = (ee / a.d1) * a.h1 * a.d1 + i1 * a.d1 + ee % a.d1;
        else {
            const int e2 = ee - R * a.d1;
            off = R * a.h1 * a.d1 + (e2 / a.d2) * a.h2 * a.d2 + i2 * a.d2 + e2 % a.d2;
        }
        tab[e] = off;
    }
    if (a.shared)
        for (int m = tid; m < a.d2 / 2; m += kThreads) theta[m] = rope.theta[m];
    for (int idx = tid; idx < (DH - a.dh) * 8 * 2; idx += kThreads) {
        const int row = a.dh + (idx >> 4), c = idx & 7;
        *reinterpret_cast<uint4 *>(((idx >> 3) & 1 ? Vs : Ks) + row * 128 + c * 16) = make_uint4(0, 0, 0, 0);
    }
    if (a.q) {
        for (int idx = tid; idx < kRows * NC; idx += kThreads) {
            const int row = idx / NC, c = idx % NC, f0 = c * 8, tok = q0 + row;
            uint32_t w[4] = {0u, 0u, 0u, 0u};
            if (tok < a.n_tok && f0 < a.dh) {
                const uint32_t *src = reinterpret_cast<const uint32_t *>(
                    a.q + (((size_t)b * a.n_tok + tok) * h + head) * a.dh + f0);
#pragma unroll
                for (int p = 0; p < 4; ++p)
                    if (f0 + 2 * p < a.dh) {
                        const float2 x = unpack_bf16x2(__ldg(src + p));
                        w[p] = pack_h2(x.x * a.qscale, x.y * a.qscale);
                    }
            }
            *reinterpret_cast<uint4 *>(X + row * DH * 2 + ((c ^ (row & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    } else {
        for (int idx = tid; idx < kRows * NC; idx += kThreads)
            reinterpret_cast<uint4 *>(X)[idx] = make_uint4(0, 0, 0, 0);
        __syncthreads();
        // row t's query (1/R_Q) sum_r A^Q_r (x) B^Q_r in fp32 (eq 2), scaled, rounded once
        for (int idx = tid; idx < kRows * a.d1; idx += kThreads) {
            const int row = idx % kRows, j1 = idx / kRows, tok = q0 + row;
            if (tok >= a.n_tok) continue;
            const float *src = a.qf + (long long)b * a.qf_seq_stride + (long long)tok * a.qf_tok_stride;
            float aq[kPrefillQfMaxRq];
#pragma unroll
            for (int r = 0; r < kPrefillQfMaxRq; ++r)
                aq[r] = r < a.rq ? __ldg(src + (long long)(r * a.h1 * a.d1 + i1 * a.d1 + j1) * a.qf_stride) : 0.f;
            for (int j2 = 0; j2 < a.d2; j2 += 2) {
                float x0 = 0.f, x1 = 0.f;
#pragma unroll
                for (int r = 0; r < kPrefillQfMaxRq; ++r)
                    if (r < a.rq) {
                        const float *bp =
                            src + (long long)(a.rq * a.h1 * a.d1 + r * a.h2 * a.d2 + i2 * a.d2 + j2) * a.qf_stride;
                        x0 += aq[r] * __ldg(bp);
                        x1 += aq[r] * __ldg(bp + a.qf_stride);
                    }
                const int f = j1 * a.d2 + j2;
                *reinterpret_cast<uint32_t *>(X + row * DH * 2 + (((f >> 3) ^ (row & 7)) << 4) + (f & 7) * 2) =
                    pack_h2(x0 * a.qf_scale, x1 * a.qf_scale);
            }
        }
    }
    __syncthreads();
    // Q fragments of this warp's 16 rows, all k-steps, kept in registers
    uint32_t qa[KS][4];
    {
        const int row = warp * 16 + (lane & 15);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks)
            ldsm4(smem_u32(X + row * DH * 2 + (((2 * ks + (lane >> 4)) ^ (row & 7)) << 4)), qa[ks]);
    }
    __syncthreads();                                             // X becomes the factor stages

    const size_t gseq = (size_t)b * (a.cap / 8);                 // first token group of the sequence
    auto issue = [&](int t) {
        unsigned char *st = X + (t & 1) * stage_bytes;
        const int g_valid = min(8, max_slot / 8 - t * 8 + 1);    // groups holding slots <= max_slot
        for (int idx = tid; idx < 8 * a.ekh; idx += kThreads) {
            const int g = idx & 7, e = idx >> 3;
            if (g < g_valid)
                cp_async16(smem_u32(st + (g * a.ekp + e) * 16),
                           a.kc + ((gseq + t * 8 + g) * a.ek + tab[e]) * 8);
        }
        unsigned char *sv = st + 8 * a.ekp * 16;
        for (int idx = tid; idx < 8 * a.evh; idx += kThreads) {
            const int g = idx & 7, e = idx >> 3;
            if (g < g_valid)
                cp_async16(smem_u32(sv + (g * a.evp + e) * 16),
                           a.vc + ((gseq + t * 8 + g) * a.ev + tab[a.ekh + e]) * 8);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    const int wrow0 = q0 + warp * 16;
    const bool warp_live = wrow0 < a.n_tok;
    const int warp_last_pos = min(start + min(wrow0 + 15, a.n_tok - 1), max_slot);
    const int pos0 = start + wrow0 + (lane >> 2), pos1 = pos0 + 8;   // positions of this lane's two rows
    float o[DH / 8][4];
#pragma unroll
    for (int nt = 0; nt < DH / 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    const int n_items = 8 * a.d1 * a.nch;                        // rebuild items per plane
    issue(0);
    for (int t = 0; t < n_kt; ++t) {
        if (t + 1 < n_kt) {
            issue(t + 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();                                         // stage t landed; tile t-1 fully used

        // ---- rebuild K_h, V_h of tile t: item = (token group g, row j1, 4 columns of B)
        {
            const unsigned char *st = X + (t & 1) * stage_bytes;
            const uint4 *sk = reinterpret_cast<const uint4 *>(st);
            const uint4 *sv = reinterpret_cast<const uint4 *>(st + 8 * a.ekp * 16);
            for (int it = tid; it < 2 * n_items; it += kThreads) {
                const bool isv = it >= n_items;
                const int i = isv ? it - n_items : it;
                const int g = i & 7, rest = i >> 3;
                const int j1 = rest / a.nch, c = rest - j1 * a.nch;
                const int R = isv ? a.rv : a.rk;
                const uint4 *A = isv ? sv + g * a.evp : sk + g * a.ekp;
                const uint4 *B = (isv && !a.shared) ? sv + g * a.evp + a.rv * a.d1 : sk + g * a.ekp + a.rk * a.d1;
                const bool rot = a.shared && !isv;
                const int slot0 = t * kSlots + g * 8;
                float2 cs[2][4], sn[2][4];
                if (rot) {
#pragma unroll
                    for (int p = 0; p < 2; ++p)
                        if (c * 4 + 2 * p < a.d2) {
                            const double th = theta[c * 2 + p];
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                rope_cs_fast((double)(slot0 + 2 * k), th, cs[p][k].x, sn[p][k].x);
                                rope_cs_fast((double)(slot0 + 2 * k + 1), th, cs[p][k].y, sn[p][k].y);
                            }
                        }
                }
                float2 acc[4][4];
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int k = 0; k < 4; ++k) acc[u][k] = make_float2(0.f, 0.f);
                for (int r = 0; r < R; ++r) {
                    float2 av[4];
                    unpack8(A[r * a.d1 + j1], av);
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        const int j2 = c * 4 + 2 * p;
                        if (j2 < a.d2) {                         // d2 is even: j2 + 1 < d2 as well
                            float2 x0[4], x1[4];
                            unpack8(B[r * a.d2 + j2], x0);
                            unpack8(B[r * a.d2 + j2 + 1], x1);
                            if (rot) {
#pragma unroll
                                for (int k = 0; k < 4; ++k) {
                                    const float2 y0 = make_float2(x0[k].x * cs[p][k].x - x1[k].x * sn[p][k].x,
                                                                  x0[k].y * cs[p][k].y - x1[k].y * sn[p][k].y);
                                    const float2 y1 = make_float2(x0[k].x * sn[p][k].x + x1[k].x * cs[p][k].x,
                                                                  x0[k].y * sn[p][k].y + x1[k].y * cs[p][k].y);
                                    x0[k] = y0;
                                    x1[k] = y1;
                                }
                            }
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                acc[2 * p][k] = ffma2(av[k], x0[k], acc[2 * p][k]);
                                acc[2 * p + 1][k] = ffma2(av[k], x1[k], acc[2 * p + 1][k]);
                            }
                        }
                    }
                }
                unsigned char *dst = isv ? Vs : Ks;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int j2 = c * 4 + u;
                    if (j2 < a.d2) {
                        if (slot0 + 7 > max_slot) {
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                if (slot0 + 2 * k > max_slot) acc[u][k].x = 0.f;
                                if (slot0 + 2 * k + 1 > max_slot) acc[u][k].y = 0.f;
                            }
                        }
                        const int f = j1 * a.d2 + j2;
                        *reinterpret_cast<uint4 *>(dst + f * 128 + ((g ^ (f & 7)) << 4)) =
                            make_uint4(pack_h2(acc[u][0].x, acc[u][0].y), pack_h2(acc[u][1].x, acc[u][1].y),
                                       pack_h2(acc[u][2].x, acc[u][2].y), pack_h2(acc[u][3].x, acc[u][3].y));
                    }
                }
            }
        }
        __syncthreads();                                         // K_h, V_h of tile t complete

        if (!warp_live || t * kSlots > warp_last_pos) continue;  // every row of the warp is before the tile
        // ---- S = Q K^T (16 rows x 64 slots)
        float s[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            const int f = ks * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t kb[4];
                const int chunk = 2 * np + (lane >> 4);
                ldsm4_t(smem_u32(Ks + f * 128 + ((chunk ^ (f & 7)) << 4)), kb);
                mma_f16(s[2 * np], qa[ks], kb[0], kb[1]);
                mma_f16(s[2 * np + 1], qa[ks], kb[2], kb[3]);
            }
        }
        // ---- causal mask and online softmax (base 2: the scores carry log2 e)
        if (t * kSlots + kSlots - 1 > start + wrow0) {
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const int j = t * kSlots + nt * 8 + 2 * (lane & 3);
                if (j > pos0) s[nt][0] = -INFINITY;
                if (j + 1 > pos0) s[nt][1] = -INFINITY;
                if (j > pos1) s[nt][2] = -INFINITY;
                if (j + 1 > pos1) s[nt][3] = -INFINITY;
            }
        }
        float mx0 = m0, mx1 = m1;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            mx0 = fmaxf(mx0, fmaxf(s[nt][0], s[nt][1]));
            mx1 = fmaxf(mx1, fmaxf(s[nt][2], s[nt][3]));
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float ref0 = mx0 == -INFINITY ? 0.f : mx0, ref1 = mx1 == -INFINITY ? 0.f : mx1;
        const float al0 = m0 == -INFINITY ? 0.f : ex2f(m0 - ref0), al1 = m1 == -INFINITY ? 0.f : ex2f(m1 - ref1);
        m0 = mx0;
        m1 = mx1;
        float ps0 = 0.f, ps1 = 0.f;
        uint32_t pa[8][2];                                      // P as fp16 pairs, A-fragment order
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            const float p0 = ex2f(s[nt][0] - ref0), p1 = ex2f(s[nt][1] - ref0);
            const float p2 = ex2f(s[nt][2] - ref1), p3 = ex2f(s[nt][3] - ref1);
            ps0 += p0 + p1;
            ps1 += p2 + p3;
            pa[nt][0] = pack_h2(p0, p1);
            pa[nt][1] = pack_h2(p2, p3);
        }
        l0 = l0 * al0 + ps0;
        l1 = l1 * al1 + ps1;
#pragma unroll
        for (int nt = 0; nt < DH / 8; ++nt) {
            o[nt][0] *= al0;
            o[nt][1] *= al0;
            o[nt][2] *= al1;
            o[nt][3] *= al1;
        }
        // ---- O += P V
#pragma unroll
        for (int kk = 0; kk < kSlots / 16; ++kk) {
            const uint32_t pf[4] = {pa[2 * kk][0], pa[2 * kk][1], pa[2 * kk + 1][0], pa[2 * kk + 1][1]};
            const int chunk = 2 * kk + ((lane >> 3) & 1);
#pragma unroll
            for (int np = 0; np < DH / 16; ++np) {
                uint32_t vb[4];
                const int f = (2 * np + (lane >> 4)) * 8 + (lane & 7);
                ldsm4(smem_u32(Vs + f * 128 + ((chunk ^ (f & 7)) << 4)), vb);
                mma_f16(o[2 * np], pf, vb[0], vb[1]);
                mma_f16(o[2 * np + 1], pf, vb[2], vb[3]);
            }
        }
    }

    // ---- normalise and store the rows this warp owns
    if (!warp_live) return;
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const int row0 = wrow0 + (lane >> 2), row1 = row0 + 8;
    const bool ok0 = row0 < a.n_tok && pos0 < a.cap, ok1 = row1 < a.n_tok && pos1 < a.cap;
    const float f0 = l0 > 0.f ? a.out_scale / l0 : 0.f, f1 = l1 > 0.f ? a.out_scale / l1 : 0.f;
    bool finite = true;
#pragma unroll
    for (int nt = 0; nt < DH / 8; ++nt) {
        const int f = nt * 8 + 2 * (lane & 3);
        if (f < a.dh) {
            const float2 y0 = ok0 ? make_float2(o[nt][0] * f0, o[nt][1] * f0) : make_float2(0.f, 0.f);
            const float2 y1 = ok1 ? make_float2(o[nt][2] * f1, o[nt][3] * f1) : make_float2(0.f, 0.f);
            if (row0 < a.n_tok) {
                *reinterpret_cast<float2 *>(out_b + ((size_t)row0 * h + head) * a.dh + f) = y0;
                finite = finite && isfinite(y0.x) && isfinite(y0.y);
            }
            if (row1 < a.n_tok) {
                *reinterpret_cast<float2 *>(out_b + ((size_t)row1 * h + head) * a.dh + f) = y1;
                finite = finite && isfinite(y1.x) && isfinite(y1.y);
            }
        }
    }
    // a value outside the fp16 range (a rebuilt K or V element, or P) makes rows non-finite
    if (__any_sync(0xffffffffu, !finite) && lane == 0) raise_error(a.err, kErrDeviceCheck);
}

struct SliceDims {
    int DH, ekh, evh, ekp, evp;
};

SliceDims slice_dims(const Dims &d) {
    SliceDims s;
    s.DH = d.dh <= 64 ? 64 : 128;
    s.ekh = d.rk * (d.d1 + d.d2);
    s.evh = d.shared ? d.rv * d.d1 : d.rv * (d.d1 + d.d2);
    s.ekp = s.ekh | 1;                       // odd stride: the 8 groups' vectors fall in distinct banks
    s.evp = s.evh | 1;
    return s;
}

}  // namespace

size_t prefill_mma_smem_bytes(const Dims &d) {
    if (d.order == 3 || d.dh > 128 || d.dh < 2 || d.d2 % 2 != 0) return 0;
    const SliceDims s = slice_dims(d);
    return (size_t)prefill_mma_layout(s.DH, s.ekh, s.evh, s.ekp, s.evp, d.d2).total;
}

bool prefill_mma_supported(const Dims &d) {
    const size_t b = prefill_mma_smem_bytes(d);
    return b > 0 && b <= 227 * 1024;
}

cudaError_t launch_prefill_mma(const Dims &d, int batch, int n_tok, const void *q, const PrefillQf &qf,
                               const int32_t *start_pos, const void *kc, const void *vc, int cap,
                               float qscale, float out_scale, float *out, const RopeTable &rope, int *err,
                               cudaStream_t st) {
    if (!prefill_mma_supported(d)) return cudaErrorInvalidValue;
    if (qf.ptr && (qf.rq < 1 || qf.rq > kPrefillQfMaxRq)) return cudaErrorInvalidValue;
    const SliceDims s = slice_dims(d);
    PrefillMmaArgs a;
    a.q = qf.ptr ? nullptr : static_cast<const __nv_bfloat16 *>(q);
    a.qf = qf.ptr;
    a.qf_stride = qf.stride;
    a.qf_seq_stride = qf.seq_stride;
    a.qf_tok_stride = qf.tok_stride;
    a.rq = qf.rq;
    a.start_pos = start_pos;
    a.kc = static_cast<const __nv_bfloat16 *>(kc);
    a.vc = static_cast<const __nv_bfloat16 *>(vc);
    a.out = out;
    a.err = err;
    a.n_tok = n_tok;
    a.cap = cap;
    a.h1 = d.h1;
    a.h2 = d.h2;
    a.d1 = d.d1;
    a.d2 = d.d2;
    a.dh = d.dh;
    a.rk = d.rk;
    a.rv = d.rv;
    a.ek = d.ek;
    a.ev = d.ev;
    a.shared = d.shared;
    a.ekh = s.ekh;
    a.evh = s.evh;
    a.ekp = s.ekp;
    a.evp = s.evp;
    a.nch = (d.d2 + 3) / 4;
    a.qscale = qscale;
    a.qf_scale = qf.rq > 0 ? qscale / (float)qf.rq : 0.f;
    a.out_scale = out_scale;
    const size_t smem = prefill_mma_smem_bytes(d);
    cudaError_t e = s.DH == 64 ? ensure_dynamic_smem<prefill_mma_kernel<64>>(smem)
                               : ensure_dynamic_smem<prefill_mma_kernel<128>>(smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((n_tok + kRows - 1) / kRows), (unsigned)d.h, (unsigned)batch);
    if (s.DH == 64)
        prefill_mma_kernel<64><<<grid, kThreads, smem, st>>>(a, rope);
    else
        prefill_mma_kernel<128><<<grid, kThreads, smem, st>>>(a, rope);
    return cudaGetLastError();
}

}  // namespace kpa
