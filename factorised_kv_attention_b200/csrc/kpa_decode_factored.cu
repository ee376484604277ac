// kpa_decode_factored.cu -- TPA decode from the query factors with the factored score
// (CUDA cores).
//
// "Kronecker Product Attention", Prop 2.2 (eq 6) with d1 = 1, h2 = 1 -- the FlashTPA
// decoding form of the "Tensor Product Attention Is All You Need" explainer: with the
// query kept as its factors A^Q (R_Q x h) and B^Q (R_Q x d_h, rotated at q_pos), the
// score of head h against cached token t is
//   score[h] = 1/(R_Q R_K) sum_{r, r'} A^Q_r[h] A^K_r'(t)[h] (B^Q_r . B~^K_r'(t)),
// so per token the head-shared dots P[r, r'] = B^Q_r . B~^K_r'(t) (R_Q R_K d_h
// multiply-adds) are formed once and mixed per head (h R_Q R_K), instead of contracting
// an assembled h x d_h query (h R_K d_h).  The values are as in the other kernels:
// O[h] += p[h] (1/R_V) sum_r A^V_r(t)[h] B^V_r(t).
//
// One CTA per (split, sequence), 8 warps, 32-token tiles copied with cp.async at a
// padded group stride, double buffered.  Per tile: the dots P (lane = token, warp =
// a share of the (r, r') pairs), the per-head mix and online softmax (lane = token,
// warp = its heads w, w + 8, ...), each tile's B^V widened once to fp32 (4 tokens per
// float4), and the value accumulation (lane = feature, warp = its heads).  Each head
// lives in one warp, so the CTA's partial (o, m, l) needs no merge inside the CTA; the
// split combine merges the splits.
#include "kpa_decode_factored.cuh"
#include "kpa_internal.cuh"
#include "kpa_sm100.cuh"

namespace kpa {
namespace {

using sm100::cp_async16;

constexpr int kFqThreads = 256;
constexpr int kFqTile = 32;           // tokens per tile (4 groups)
constexpr int kFqMaxHpw = 4;          // heads per warp (h <= 32)
constexpr int kFqMaxPairs = 32;       // R_Q R_K
constexpr int kFqMaxR = 4;            // R_K, R_V

struct FactoredArgs {
    const float *qf;
    long long qf_stride, qf_seq_stride;
    const int32_t *q_pos;
    const __nv_bfloat16 *kc, *vc;
    int cap;
    const int32_t *seq_len;
    int max_len, tps, n_split;
    int h, rq, rk, rv;
    float qscale;                     // sm_scale / (R_Q R_K) * log2(e)
    float *part_o, *part_ml;
    int *err;
};

// element e of token t in a tile of 8-token groups at byte stride g; a bf16 widened by a shift
__device__ __forceinline__ float tile_elem(const unsigned char *tile, int g, int t, int e) {
    return __uint_as_float((uint32_t)*reinterpret_cast<const unsigned short *>(tile + (t >> 3) * g + (e * kGroup + (t & 7)) * 2)
                           << 16);
}

// Shared-memory layout (bytes), for h heads, d_h, R_Q, R_K, R_V.
struct FqLayout {
    size_t bq, aq, pt, wv, bv, cs, tiles, bytes;
    int pld, gk, gv;
    __host__ __device__ FqLayout(int h, int dh, int rq, int rk, int rv) {
        pld = rq * rk + 1;                                        // odd row stride: no bank conflicts
        gk = rk * (h + dh) * kGroup * 2 + 16;                     // padded group strides
        gv = rv * (h + dh) * kGroup * 2 + 16;
        bq = 0;                                                   // [R_Q][d_h] rotated B^Q
        aq = bq + (size_t)rq * dh * 4;                            // [R_Q][h] scaled A^Q
        pt = aq + (size_t)rq * h * 4;                             // [32][pld] dots
        wv = pt + (size_t)kFqTile * pld * 4;                      // [h][R_V][32] p a^V
        bv = (wv + (size_t)h * rv * kFqTile * 4 + 15) / 16 * 16;  // [R_V][8][d_h] float4 (4 tokens)
        cs = bv + (size_t)rv * kFqTile * dh * 4;                  // [d_h / 2] (cos, sin)
        tiles = (cs + (size_t)(dh / 2) * 8 + 15) / 16 * 16;
        bytes = tiles + 2 * (size_t)(4 * gk + 4 * gv);
    }
};

template <int DH, int NP_>
__global__ void __launch_bounds__(kFqThreads, 2) decode_factored_kernel(FactoredArgs a, RopeTable rope) {
    constexpr int JPL = DH / 32;                                  // features per lane
    const int H = a.h, RQ = a.rq, RK = a.rk, RV = a.rv, NP = NP_ ? NP_ : RQ * RK;
    const int EK = RK * (H + DH), EV = RV * (H + DH);
    const FqLayout lay(H, DH, RQ, RK, RV);
    const int GK = lay.gk, GV = lay.gv, TILE_BYTES = 4 * GK + 4 * GV, PLD = lay.pld;
    extern __shared__ float4 smem4[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(smem4);
    float *bq = reinterpret_cast<float *>(sm + lay.bq);
    float *aq = reinterpret_cast<float *>(sm + lay.aq);
    float *pt = reinterpret_cast<float *>(sm + lay.pt);
    float *wv = reinterpret_cast<float *>(sm + lay.wv);
    float4 *bvs = reinterpret_cast<float4 *>(sm + lay.bv);
    float2 *cs = reinterpret_cast<float2 *>(sm + lay.cs);
    unsigned char *tiles = sm + lay.tiles;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.y, split = blockIdx.x;
    int L = a.seq_len[b];
    if (L > a.max_len || L < 0) {
        if (split == 0 && tid == 0) raise_error(a.err, kErrDeviceCheck);
        L = L < 0 ? 0 : a.max_len;
    }
    const int t0 = split * a.tps;
    if (t0 >= L) return;                                          // empty split: the combine skips it
    const int t1 = split == a.n_split - 1 ? L : min(t0 + a.tps, L);
    const int n_tiles = (t1 - t0 + kFqTile - 1) / kFqTile;
    const unsigned char *kbase = reinterpret_cast<const unsigned char *>(a.kc + ((size_t)b * a.cap + t0) * EK);
    const unsigned char *vbase = reinterpret_cast<const unsigned char *>(a.vc + ((size_t)b * a.cap + t0) * EV);

    auto issue = [&](int t, int buf) {
        const int n = min(kFqTile, t1 - t0 - t * kFqTile);
        const int groups = (n + kGroup - 1) / kGroup;
        const int ck = EK * kGroup * 2 / 16, cv = EV * kGroup * 2 / 16;
        const uint32_t dst = (uint32_t)__cvta_generic_to_shared(tiles + (size_t)buf * TILE_BYTES);
        const unsigned char *ks = kbase + (size_t)t * kFqTile * EK * 2;
        const unsigned char *vs = vbase + (size_t)t * kFqTile * EV * 2;
        for (int c = tid; c < groups * (ck + cv); c += kFqThreads) {
            if (c < groups * ck) {
                const int g = c / ck, k = c % ck;
                cp_async16(dst + g * GK + k * 16, ks + ((size_t)g * ck + k) * 16);
            } else {
                const int c2 = c - groups * ck, g = c2 / cv, k = c2 % cv;
                cp_async16(dst + 4 * GK + g * GV + k * 16, vs + ((size_t)g * cv + k) * 16);
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    issue(0, 0);

    // query factors: A^Q scaled, B^Q rotated by R(q_pos) on the pairs (2m, 2m+1)
    const bool rotate = a.q_pos != nullptr;
    if (rotate && tid < DH / 2) {
        float c, s;
        rope_cs((double)a.q_pos[b], rope.theta[tid], c, s);
        cs[tid] = make_float2(c, s);
    }
    __syncthreads();
    const float *qfb = a.qf + (size_t)b * a.qf_seq_stride;
    for (int e = tid; e < RQ * H; e += kFqThreads) aq[e] = __ldg(qfb + (size_t)e * a.qf_stride) * a.qscale;
    for (int i = tid; i < RQ * DH / 2; i += kFqThreads) {
        const int r = i / (DH / 2), m = i % (DH / 2);
        const size_t e0 = (size_t)RQ * H + (size_t)r * DH + 2 * m;
        float x0 = __ldg(qfb + e0 * a.qf_stride), x1 = __ldg(qfb + (e0 + 1) * a.qf_stride);
        if (rotate) {
            const float2 w = cs[m];
            const float y0 = x0 * w.x - x1 * w.y, y1 = x0 * w.y + x1 * w.x;
            x0 = y0;
            x1 = y1;
        }
        bq[r * DH + 2 * m] = x0;
        bq[r * DH + 2 * m + 1] = x1;
    }

    float m_run[kFqMaxHpw], l_part[kFqMaxHpw], acc[kFqMaxHpw][JPL];
#pragma unroll
    for (int k = 0; k < kFqMaxHpw; ++k) {
        m_run[k] = -INFINITY;
        l_part[k] = 0.f;
#pragma unroll
        for (int i = 0; i < JPL; ++i) acc[k][i] = 0.f;
    }
    const int bk0 = RK * H, bv0 = RV * H;                         // first B element of a record

    for (int t = 0; t < n_tiles; ++t) {
        const int buf = t & 1;
        if (t + 1 < n_tiles) {
            issue(t + 1, buf ^ 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();                                          // tile t (and the query) ready
        const unsigned char *kt = tiles + (size_t)buf * TILE_BYTES;
        const unsigned char *vt = kt + 4 * GK;
        const int n_valid = min(kFqTile, t1 - t0 - t * kFqTile);
        const bool valid = lane < n_valid;

        // ---- head-shared dots P[t][r R_K + r'] = B^Q_r . B~^K_r'(t) (lane = token)
        for (int rk = 0; rk < RK; ++rk) {
            float bk[DH];
#pragma unroll
            for (int j = 0; j < DH; ++j) bk[j] = tile_elem(kt, GK, lane, bk0 + rk * DH + j);
            for (int p = warp; p < NP; p += 8) {
                if (p % RK != rk) continue;
                const float4 *bqr = reinterpret_cast<const float4 *>(bq + (p / RK) * DH);
                float d0 = 0.f, d1 = 0.f;
#pragma unroll
                for (int j = 0; j < DH / 4; j += 2) {
                    const float4 u = bqr[j], v = bqr[j + 1];
                    d0 = fmaf(u.x, bk[4 * j], d0);
                    d1 = fmaf(u.y, bk[4 * j + 1], d1);
                    d0 = fmaf(u.z, bk[4 * j + 2], d0);
                    d1 = fmaf(u.w, bk[4 * j + 3], d1);
                    d0 = fmaf(v.x, bk[4 * j + 4], d0);
                    d1 = fmaf(v.y, bk[4 * j + 5], d1);
                    d0 = fmaf(v.z, bk[4 * j + 6], d0);
                    d1 = fmaf(v.w, bk[4 * j + 7], d1);
                }
                pt[lane * PLD + p] = d0 + d1;
            }
        }
        // each tile's B^V widened once: [R_V][8][d_h] x 4 tokens (0 past the tile's end)
        for (int it = tid; it < RV * (kFqTile / 4) * DH; it += kFqThreads) {
            const int r = it / ((kFqTile / 4) * DH), rem = it % ((kFqTile / 4) * DH);
            const int t4 = rem / DH, j = rem % DH;
            float4 v;
            v.x = 4 * t4 + 0 < n_valid ? tile_elem(vt, GV, 4 * t4 + 0, bv0 + r * DH + j) : 0.f;
            v.y = 4 * t4 + 1 < n_valid ? tile_elem(vt, GV, 4 * t4 + 1, bv0 + r * DH + j) : 0.f;
            v.z = 4 * t4 + 2 < n_valid ? tile_elem(vt, GV, 4 * t4 + 2, bv0 + r * DH + j) : 0.f;
            v.w = 4 * t4 + 3 < n_valid ? tile_elem(vt, GV, 4 * t4 + 3, bv0 + r * DH + j) : 0.f;
            bvs[(r * (kFqTile / 4) + t4) * DH + j] = v;
        }
        __syncthreads();

        // ---- rank mix, online softmax and the weights p a^V (lane = token)
#pragma unroll
        for (int k = 0; k < kFqMaxHpw; ++k) {
            const int h = warp + 8 * k;
            if (h >= H) break;
            float s = 0.f;
            for (int rk = 0; rk < RK; ++rk) {
                float mix = 0.f;
                if constexpr (NP_ != 0) {
#pragma unroll
                    for (int rq = 0; rq < NP_; ++rq)
                        if (rq < RQ) mix = fmaf(aq[rq * H + h], pt[lane * PLD + rq * RK + rk], mix);
                } else {
                    for (int rq = 0; rq < RQ; ++rq) mix = fmaf(aq[rq * H + h], pt[lane * PLD + rq * RK + rk], mix);
                }
                s = fmaf(tile_elem(kt, GK, lane, rk * H + h), mix, s);
            }
            s = valid ? s : -INFINITY;
            float mx = s;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float m_new = fmaxf(m_run[k], mx);                 // finite: the tile has a valid token
            const float alpha = exp2f(m_run[k] - m_new);
            const float p = valid ? exp2f(s - m_new) : 0.f;
            l_part[k] = fmaf(l_part[k], alpha, p);
            m_run[k] = m_new;
            for (int r = 0; r < RV; ++r)
                wv[(h * RV + r) * kFqTile + lane] = valid ? p * tile_elem(vt, GV, lane, r * H + h) : 0.f;
#pragma unroll
            for (int i = 0; i < JPL; ++i) acc[k][i] *= alpha;
        }
        __syncwarp();

        // ---- values (lane = feature): O[h, j] += sum_{t, r} w[h, r, t] B^V_r(t)[j]
        const int n4 = (n_valid + 3) / 4;
        for (int t4 = 0; t4 < n4; ++t4)
            for (int r = 0; r < RV; ++r) {
                float4 bvv[JPL], w4[kFqMaxHpw];
#pragma unroll
                for (int i = 0; i < JPL; ++i) bvv[i] = bvs[(r * (kFqTile / 4) + t4) * DH + lane + 32 * i];
#pragma unroll
                for (int k = 0; k < kFqMaxHpw; ++k)
                    w4[k] = warp + 8 * k < H ? reinterpret_cast<const float4 *>(wv + ((warp + 8 * k) * RV + r) * kFqTile)[t4]
                                             : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int k = 0; k < kFqMaxHpw; ++k)
#pragma unroll
                    for (int i = 0; i < JPL; ++i) {
                        float x = acc[k][i];
                        x = fmaf(w4[k].x, bvv[i].x, x);
                        x = fmaf(w4[k].y, bvv[i].y, x);
                        x = fmaf(w4[k].z, bvv[i].z, x);
                        acc[k][i] = fmaf(w4[k].w, bvv[i].w, x);
                    }
            }
        __syncthreads();                                          // buffers are refilled next iteration
    }

    // ---- unnormalised partial (o, m, l) of this split
    float *po = a.part_o + ((size_t)(b * a.n_split + split) * H) * DH;
    float *pml = a.part_ml + ((size_t)(b * a.n_split + split) * H) * 2;
#pragma unroll
    for (int k = 0; k < kFqMaxHpw; ++k) {
        const int h = warp + 8 * k;
        if (h >= H) break;
        float l = l_part[k];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
#pragma unroll
        for (int i = 0; i < JPL; ++i) po[h * DH + lane + 32 * i] = acc[k][i];
        if (lane == 0) *reinterpret_cast<float2 *>(pml + 2 * h) = make_float2(m_run[k], l);
    }
}

template <class F>
auto with_factored_kernel(int rq, int rk, F &&f) {
    if (rq * rk == 16) return f(decode_factored_kernel<64, 16>);
    return f(decode_factored_kernel<64, 0>);
}

}  // namespace

bool factored_decode_supported(const Dims &d, int rq) {
    return d.order == 2 && !d.shared && d.h2 == 1 && d.d1 == 1 && d.dh == 64 && d.h <= 8 * kFqMaxHpw && rq > 0 &&
           rq * d.rk <= kFqMaxPairs && d.rk <= kFqMaxR && d.rv <= kFqMaxR &&
           FqLayout(d.h, d.dh, rq, d.rk, d.rv).bytes <= 200 * 1024;
}

int factored_ctas_per_sm(const Dims &d, int rq) {
    const size_t smem = FqLayout(d.h, d.dh, rq, d.rk, d.rv).bytes;
    return with_factored_kernel(rq, d.rk, [&](auto kernel) -> int {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) {
            cudaGetLastError();
            return 1;
        }
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kFqThreads, smem) != cudaSuccess) {
            cudaGetLastError();
            return 1;
        }
        return n > 0 ? n : 1;
    });
}

cudaError_t launch_decode_factored(const Dims &d, int rq, int batch, const float *qf, long long qf_stride,
                                   long long qf_seq_stride, const int32_t *q_pos, const void *kc, const void *vc,
                                   int cap, const int32_t *seq_len, int max_len, float qscale, const DecodePlan &p,
                                   float *part_o, float *part_ml, const RopeTable &rope, int *err, cudaStream_t st) {
    FactoredArgs a;
    a.qf = qf;
    a.qf_stride = qf_stride;
    a.qf_seq_stride = qf_seq_stride;
    a.q_pos = q_pos;
    a.kc = static_cast<const __nv_bfloat16 *>(kc);
    a.vc = static_cast<const __nv_bfloat16 *>(vc);
    a.cap = cap;
    a.seq_len = seq_len;
    a.max_len = max_len;
    a.tps = p.tokens_per_split;
    a.n_split = p.n_split;
    a.h = d.h;
    a.rq = rq;
    a.rk = d.rk;
    a.rv = d.rv;
    a.qscale = qscale;
    a.part_o = part_o;
    a.part_ml = part_ml;
    a.err = err;
    const size_t smem = FqLayout(d.h, d.dh, rq, d.rk, d.rv).bytes;
    const dim3 grid((unsigned)p.n_split, (unsigned)batch);
    return with_factored_kernel(rq, d.rk, [&](auto kernel) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kernel<<<grid, kFqThreads, smem, st>>>(a, rope);
        return cudaGetLastError();
    });
}

}  // namespace kpa
