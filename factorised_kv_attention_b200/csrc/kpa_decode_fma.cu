// kpa_decode_fma.cu -- factor-space decode on the CUDA cores (any shape, fp32 or bf16).
//
// One CTA = one (sequence, split) and all heads.  The split's slots are walked in
// shared-memory tiles; per tile (Proposition 2.2 with a dense query, scored
// directly from the factors):
//   score(i1,i2) = sum_r sum_j1 A^K_r[i1,j1] * (sum_j2 q[i1,i2,j1,j2] B~^K_r[i2,j2])
//   online softmax per head in the log2 domain (running max m and sum l),
//   o(i1,i2)[j1,j2] += p * sum_r A^V_r[i1,j1] B^V_r[i2,j2].
// 1/R_K and the softmax scale are folded into the rotated query, 1/R_V into the
// combine.  The CTA leaves an unnormalised partial (o, m, l) per head; the
// combine pass merges the splits with a log-sum-exp ("online log-sum-exp",
// FlashTPA decoding in the Tensor Product Attention explainer).
//
// This kernel is the general fallback (fp32 caches, shapes outside the
// tensor-core kernel's cover).
#include "kpa_internal.cuh"

namespace kpa {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ int elem(int tok, int e, int E) {
    return ((tok >> 3) * E + e) * kGroup + (tok & 7);
}

template <typename T>
__device__ __forceinline__ void copy_tile(T *dst, const T *src, size_t elems) {
    // elems * sizeof(T) is a multiple of 16 (8-token groups)
    const size_t n16 = elems * sizeof(T) / 16;
    const uint4 *s = reinterpret_cast<const uint4 *>(src);
    uint4 *o = reinterpret_cast<uint4 *>(dst);
    for (size_t i = threadIdx.x; i < n16; i += blockDim.x) o[i] = __ldg(s + i);
}

template <typename T, int OPT>
__global__ void __launch_bounds__(kThreads)
decode_fma_kernel(Dims d, const T *__restrict__ q, const int32_t *__restrict__ q_pos,
                  const T *__restrict__ kc, const T *__restrict__ vc, int cap,
                  const int32_t *__restrict__ seq_len, int max_len, float qscale, int tps,
                  int tile, int n_split, float *__restrict__ part_o,
                  float *__restrict__ part_ml, RopeTable rope, int *err) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int b = blockIdx.y, split = blockIdx.x, tid = threadIdx.x;
    const int h = d.h, dh = d.dh;

    int L = seq_len[b];
    if (L > max_len || L < 0) {
        if (split == 0 && tid == 0) raise_error(err, kErrDeviceCheck);
        L = L < 0 ? 0 : max_len;
    }
    const int t0 = split * tps;
    if (t0 >= L) return;                          // empty split: the combine skips it
    const int t1 = split == n_split - 1 ? L : min(t0 + tps, L);   // the last split runs to the end

    float *qr = reinterpret_cast<float *>(smem);  // [h][dh] rotated, scaled query
    float *pr = qr + h * dh;                      // [h][tile] scores, then weights
    float *m_run = pr + h * tile;
    float *l_run = m_run + h;
    float *alpha = l_run + h;
    size_t off = (size_t)(h * dh + h * tile + 3 * h) * sizeof(float);
    off = (off + 15) & ~(size_t)15;
    T *kt = reinterpret_cast<T *>(smem + off);    // [tile/8][ek][8]
    T *vt = kt + (size_t)tile * d.ek;             // [tile/8][ev][8]

    // rotate the query: I_{d1} (x) R^(2)(q_pos), pairs (2m, 2m+1) of each d2 chunk
    const T *qb = q + (size_t)b * h * dh;
    const bool rotate = q_pos != nullptr;
    const double qp = rotate ? (double)q_pos[b] : 0.0;
    for (int i = tid; i < h * dh / 2; i += kThreads) {
        const float x0 = to_f32(qb[2 * i]), x1 = to_f32(qb[2 * i + 1]);
        float y0 = x0, y1 = x1;
        if (rotate) {
            const int m = ((2 * i) % d.d2) >> 1;
            float c, s;
            rope_cs(qp, rope.theta[m], c, s);
            y0 = x0 * c - x1 * s;
            y1 = x0 * s + x1 * c;
        }
        qr[2 * i] = y0 * qscale;
        qr[2 * i + 1] = y1 * qscale;
    }
    for (int i = tid; i < h; i += kThreads) {
        m_run[i] = -INFINITY;
        l_run[i] = 0.f;
    }
    float o[OPT];
#pragma unroll
    for (int k = 0; k < OPT; ++k) o[k] = 0.f;

    const T *kb = kc + (size_t)b * cap * d.ek;
    const T *vb = vc + (size_t)b * cap * d.ev;
    const int a_k = d.rk * d.h1 * d.d1, a_v = d.rv * d.h1 * d.d1;

    for (int s0 = t0; s0 < t1; s0 += tile) {
        const int n = min(tile, t1 - s0);
        const int groups = (n + kGroup - 1) / kGroup;
        __syncthreads();                          // previous tile fully consumed
        copy_tile(kt, kb + (size_t)s0 * d.ek, (size_t)groups * d.ek * kGroup);
        copy_tile(vt, vb + (size_t)s0 * d.ev, (size_t)groups * d.ev * kGroup);
        __syncthreads();

        // scores, log2 domain (qscale carries sm_scale / R_K * log2 e)
        for (int idx = tid; idx < h * tile; idx += kThreads) {
            const int head = idx / tile, tok = idx % tile;
            float sc = -INFINITY;
            if (tok < n) {
                const int i1 = head / d.h2, i2 = head % d.h2;
                float acc = 0.f;
                for (int r = 0; r < d.rk; ++r) {
                    const int a_base = r * d.h1 * d.d1 + i1 * d.d1;
                    const int b_base = a_k + r * d.h2 * d.d2 + i2 * d.d2;
                    for (int j1 = 0; j1 < d.d1; ++j1) {
                        const float *qrow = qr + head * dh + j1 * d.d2;
                        float inner = 0.f;
                        for (int j2 = 0; j2 < d.d2; ++j2)
                            inner += qrow[j2] * to_f32(kt[elem(tok, b_base + j2, d.ek)]);
                        acc += to_f32(kt[elem(tok, a_base + j1, d.ek)]) * inner;
                    }
                }
                sc = acc;
            }
            pr[head * tile + tok] = sc;
        }
        __syncthreads();

        // online softmax, one thread per head
        for (int head = tid; head < h; head += kThreads) {
            float *row = pr + head * tile;
            const float m_old = m_run[head];
            float mx = m_old;
            for (int tok = 0; tok < n; ++tok) mx = fmaxf(mx, row[tok]);
            const float al = (m_old == -INFINITY) ? 0.f : exp2f(m_old - mx);
            float sum = 0.f;
            for (int tok = 0; tok < n; ++tok) {
                const float p = exp2f(row[tok] - mx);
                row[tok] = p;
                sum += p;
            }
            l_run[head] = l_run[head] * al + sum;
            m_run[head] = mx;
            alpha[head] = al;
        }
        __syncthreads();

        // values: o += p * sum_r A^V_r[i1,j1] B^V_r[i2,j2]
#pragma unroll
        for (int k = 0; k < OPT; ++k) {
            const int idx = tid + k * kThreads;
            if (idx < h * dh) {
                const int head = idx / dh, f = idx % dh;
                const int i1 = head / d.h2, i2 = head % d.h2;
                const int j1 = f / d.d2, j2 = f % d.d2;
                const float *prow = pr + head * tile;
                float acc = 0.f;
                for (int tok = 0; tok < n; ++tok) {
                    float v = 0.f;
                    for (int r = 0; r < d.rv; ++r)
                        v += to_f32(vt[elem(tok, r * d.h1 * d.d1 + i1 * d.d1 + j1, d.ev)]) *
                             to_f32(vt[elem(tok, a_v + r * d.h2 * d.d2 + i2 * d.d2 + j2, d.ev)]);
                    acc += prow[tok] * v;
                }
                o[k] = o[k] * alpha[head] + acc;
            }
        }
    }

    float *po = part_o + ((size_t)(b * n_split + split) * h) * dh;
#pragma unroll
    for (int k = 0; k < OPT; ++k) {
        const int idx = tid + k * kThreads;
        if (idx < h * dh) po[idx] = o[k];
    }
    __syncthreads();
    float *pml = part_ml + ((size_t)(b * n_split + split) * h) * 2;
    for (int head = tid; head < h; head += kThreads) {
        pml[2 * head] = m_run[head];
        pml[2 * head + 1] = l_run[head];
    }
}

template <typename T, int OPT>
cudaError_t launch_t(const Dims &d, int batch, const void *q, const int32_t *q_pos,
                     const void *kc, const void *vc, int cap, const int32_t *seq_len,
                     int max_len, float qscale, const DecodePlan &p, float *part_o,
                     float *part_ml, const RopeTable &rope, int *err, cudaStream_t st,
                     size_t smem) {
    auto kern = decode_fma_kernel<T, OPT>;
    cudaError_t e = ensure_dynamic_smem<decode_fma_kernel<T, OPT>>(smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)p.n_split, (unsigned)batch);
    kern<<<grid, kThreads, smem, st>>>(d, (const T *)q, q_pos, (const T *)kc, (const T *)vc, cap,
                                       seq_len, max_len, qscale, p.tokens_per_split, p.tile,
                                       p.n_split, part_o, part_ml, rope, err);
    return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch_opt(const Dims &d, int batch, const void *q, const int32_t *q_pos,
                         const void *kc, const void *vc, int cap, const int32_t *seq_len,
                         int max_len, float qscale, const DecodePlan &p, float *part_o,
                         float *part_ml, const RopeTable &rope, int *err, cudaStream_t st,
                         size_t smem) {
    const int need = (d.h * d.dh + kThreads - 1) / kThreads;
#define KPA_OPT_CASE(N)                                                                      \
    if (need <= N)                                                                           \
        return launch_t<T, N>(d, batch, q, q_pos, kc, vc, cap, seq_len, max_len, qscale, p, \
                              part_o, part_ml, rope, err, st, smem);
    KPA_OPT_CASE(1)
    KPA_OPT_CASE(2)
    KPA_OPT_CASE(4)
    KPA_OPT_CASE(8)
    KPA_OPT_CASE(16)
    KPA_OPT_CASE(32)
#undef KPA_OPT_CASE
    return cudaErrorInvalidValue;
}

}  // namespace

size_t decode_fma_smem_bytes(const Dims &d, kpa_dtype dt, int tile) {
    size_t off = (size_t)(d.h * d.dh + d.h * tile + 3 * d.h) * sizeof(float);
    off = (off + 15) & ~(size_t)15;
    const size_t es = dt == KPA_BF16 ? 2 : 4;
    return off + (size_t)tile * (d.ek + d.ev) * es;
}

cudaError_t launch_decode_fma(const Dims &d, kpa_dtype dt, int batch, const void *q,
                              const int32_t *q_pos, const void *kc, const void *vc, int cap,
                              const int32_t *seq_len, int max_len, float qscale,
                              const DecodePlan &plan, float *part_o, float *part_ml,
                              const RopeTable &rope, int *err, cudaStream_t st, int /*sms*/) {
    const size_t smem = decode_fma_smem_bytes(d, dt, plan.tile);
    if (dt == KPA_BF16)
        return dispatch_opt<__nv_bfloat16>(d, batch, q, q_pos, kc, vc, cap, seq_len, max_len,
                                           qscale, plan, part_o, part_ml, rope, err, st, smem);
    return dispatch_opt<float>(d, batch, q, q_pos, kc, vc, cap, seq_len, max_len, qscale, plan,
                               part_o, part_ml, rope, err, st, smem);
}

// ---------------------------------------------------------------------------
// Split combine: out = (1/R_V) * sum_i 2^(m_i - M) o_i / sum_i 2^(m_i - M) l_i.
// One block per (head, sequence, chunk of up to 16 features).  The block's threads
// take (feature, split phase) pairs; right after the wait on the decode, each thread
// requests its partial outputs (every 32nd split, up to kCombinePre of them into
// registers) and the first threads the splits' (m, l), all in one round trip to L2.
// The maximum, the weights and their sum are then formed in shared memory, each
// thread weighs the outputs it already holds, and the phases are added through shared
// memory.
// Launched as a programmatic dependent of the decode kernel: it becomes resident
// while the decode's last CTAs still run and waits for them before reading.
namespace {

constexpr int kCombineThreads = 512;
constexpr int kCombineMaxSplits = 4096;
constexpr int kCombineFeatures = 16;
constexpr int kCombinePre = 8;           // partial outputs per thread requested up front

__global__ void __launch_bounds__(kCombineThreads)
decode_combine_kernel(Dims d, const int32_t *__restrict__ seq_len, int max_len, int tps,
                      int n_split, const float *__restrict__ part_o,
                      const float *__restrict__ part_ml, float out_scale,
                      float *__restrict__ out, float *__restrict__ lse, float lse_scale) {
    __shared__ float w[kCombineMaxSplits];
    __shared__ float red[kCombineThreads / 32];
    __shared__ float s_max, s_den;
    const int fch = d.dh < kCombineFeatures ? d.dh : kCombineFeatures;    // features per block
    const int n_chunks = (d.dh + fch - 1) / fch;
    const int head = blockIdx.x / n_chunks, f0 = (blockIdx.x % n_chunks) * fch;
    const int b = blockIdx.y, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    asm volatile("griddepcontrol.wait;" ::: "memory");        // the decode's partials are complete
    asm volatile("griddepcontrol.launch_dependents;");
    int L = seq_len[b];
    L = L < 0 ? 0 : (L > max_len ? max_len : L);
    const int ns = min(n_split, (L + tps - 1) / tps);
    float *dst = out + ((size_t)b * d.h + head) * d.dh + f0;
    const int nf = min(fch, d.dh - f0);
    if (ns == 0 || ns > kCombineMaxSplits) {
        for (int f = tid; f < nf; f += kCombineThreads) dst[f] = 0.f;
        if (lse && f0 == 0 && tid == 0) lse[(size_t)b * d.h + head] = -INFINITY;   // no scores
        return;
    }
    // (feature, phase) pairs: the phases of one feature take every P-th split
    const int P = kCombineThreads / fch;
    const int f = tid % fch, phase = tid / fch;
    const bool worker = phase < P && f < nf;
    const float *po = part_o + ((size_t)b * n_split * d.h + head) * d.dh + f0 + f;
    const size_t po_stride = (size_t)d.h * d.dh;
    float pre[kCombinePre];
#pragma unroll
    for (int k = 0; k < kCombinePre; ++k) {
        const int i = phase + k * P;
        pre[k] = worker && i < ns ? __ldcg(po + (size_t)i * po_stride) : 0.f;
    }
    const float2 *ml = reinterpret_cast<const float2 *>(part_ml) + (size_t)b * n_split * d.h + head;
    float M = -INFINITY;
    float2 mine[kCombineMaxSplits / kCombineThreads];
#pragma unroll
    for (int k = 0; k < kCombineMaxSplits / kCombineThreads; ++k) {
        const int i = tid + k * kCombineThreads;
        mine[k] = i < ns ? __ldcg(ml + (size_t)i * d.h) : make_float2(-INFINITY, 0.f);
        M = fmaxf(M, mine[k].x);
    }
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    if (lane == 0) red[wid] = M;
    __syncthreads();
    if (tid == 0) {
        float t = red[0];
        for (int k = 1; k < kCombineThreads / 32; ++k) t = fmaxf(t, red[k]);
        s_max = t;
    }
    __syncthreads();
    M = s_max;
    float den = 0.f;
#pragma unroll
    for (int k = 0; k < kCombineMaxSplits / kCombineThreads; ++k) {
        const int i = tid + k * kCombineThreads;
        if (i < ns) {
            const float wi = mine[k].x == -INFINITY ? 0.f : exp2f(mine[k].x - M);
            w[i] = wi;
            den += wi * mine[k].y;
        }
    }
    for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
    __syncthreads();                                       // red reused; w complete
    if (lane == 0) red[wid] = den;
    __syncthreads();
    if (tid == 0) {
        float t = 0.f;
        for (int k = 0; k < kCombineThreads / 32; ++k) t += red[k];
        s_den = t;
        if (lse && f0 == 0) lse[(size_t)b * d.h + head] = t > 0.f ? (M + log2f(t)) * lse_scale : -INFINITY;
    }
    float num = 0.f;
    if (worker) {
#pragma unroll
        for (int k = 0; k < kCombinePre; ++k) {
            const int i = phase + k * P;
            if (i < ns) num += w[i] * pre[k];
        }
#pragma unroll 4
        for (int i = phase + kCombinePre * P; i < ns; i += P) num += w[i] * __ldcg(po + (size_t)i * po_stride);
    }
    __syncthreads();                                       // s_den set; every w read
    float *acc = w;                                        // reuse: [P][fch] partial sums
    if (phase < P) acc[phase * fch + f] = num;
    __syncthreads();
    for (int ff = tid; ff < nf; ff += kCombineThreads) {
        float t = 0.f;
        for (int ph = 0; ph < P; ++ph) t += acc[ph * fch + ff];
        dst[ff] = s_den > 0.f ? out_scale * t / s_den : 0.f;
    }
}

}  // namespace

cudaError_t launch_decode_combine(const Dims &d, int batch, const int32_t *seq_len,
                                  int max_len, const DecodePlan &plan, const float *part_o,
                                  const float *part_ml, float out_scale, float *out,
                                  cudaStream_t st, float *lse, float lse_scale) {
    if (plan.n_split > kCombineMaxSplits) return cudaErrorInvalidValue;
    const int fch = d.dh < kCombineFeatures ? d.dh : kCombineFeatures;
    const long long blocks = (long long)d.h * ((d.dh + fch - 1) / fch);
    if (blocks > 0x7fffffffLL || batch > 65535) return cudaErrorInvalidValue;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3((unsigned)blocks, (unsigned)batch);
    lc.blockDim = dim3(kCombineThreads);
    lc.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    return cudaLaunchKernelEx(&lc, decode_combine_kernel, d, seq_len, max_len, plan.tokens_per_split, plan.n_split,
                              part_o, part_ml, out_scale, out, lse, lse_scale);
}

namespace {

// One block per (head, sequence), one thread per feature: the parts' weights
// exp(lse_p - LSE) are formed once per block in shared memory.
constexpr int kMergeMaxParts = 4096;

__global__ void __launch_bounds__(1024)
merge_lse_kernel(int heads, int d_h, int n_parts, const float *__restrict__ outs, const float *__restrict__ lses,
                 float *__restrict__ out, float *__restrict__ lse_out) {
    __shared__ float w[kMergeMaxParts];
    __shared__ float s_max, s_den;
    const int head = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
    const size_t bh = (size_t)b * heads + head, per_part = (size_t)gridDim.y * heads;
    if (tid == 0) {
        float M = -INFINITY;
        for (int p = 0; p < n_parts; ++p) M = fmaxf(M, lses[p * per_part + bh]);
        float den = 0.f;
        for (int p = 0; p < n_parts; ++p) {
            const float l = lses[p * per_part + bh];
            const float wp = l == -INFINITY ? 0.f : expf(l - M);
            w[p] = wp;
            den += wp;
        }
        s_max = M;
        s_den = den;
        if (lse_out) lse_out[bh] = den > 0.f ? M + logf(den) : -INFINITY;
    }
    __syncthreads();
    const float inv = s_den > 0.f ? 1.f / s_den : 0.f;
    for (int f = tid; f < d_h; f += blockDim.x) {
        float acc = 0.f;
        for (int p = 0; p < n_parts; ++p)
            if (w[p] != 0.f) acc = fmaf(w[p], outs[(p * per_part + bh) * d_h + f], acc);
        out[bh * d_h + f] = acc * inv;
    }
}

}  // namespace

cudaError_t launch_merge_lse(int batch, int heads, int d_h, int n_parts, const float *outs, const float *lses,
                             float *out, float *lse_out, cudaStream_t st) {
    if (n_parts > kMergeMaxParts || d_h > 1024) return cudaErrorInvalidValue;
    const int threads = d_h < 32 ? 32 : (d_h + 31) / 32 * 32;
    merge_lse_kernel<<<dim3((unsigned)heads, (unsigned)batch), threads, 0, st>>>(heads, d_h, n_parts, outs, lses, out,
                                                                                 lse_out);
    return cudaGetLastError();
}

}  // namespace kpa
