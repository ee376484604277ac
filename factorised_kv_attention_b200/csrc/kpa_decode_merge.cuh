// kpa_decode_merge.cuh -- merge of a sequence's split partials, done by the last CTA
// of the sequence inside the tensor-core decode kernels.
#pragma once

#include "kpa_internal.cuh"

namespace kpa {

// out[b] = out_scale * (sum_i w_i o_i) / (sum_i w_i l_i), w_i = 2^(m_i - M), M = max_i m_i,
// over the n_b splits of sequence b that hold tokens: the log-sum-exp merge of the
// per-split online-softmax partials (o_i unnormalised, (m_i, l_i) per head, base 2).
// One float4 output column per thread (threads tid < nthr).  The column of up to PF
// splits and its head's (m, l) of those splits are requested together, so the merge
// takes one round trip to L2; the weights are formed per thread.
template <int H, int DH>
__device__ __forceinline__ void merge_split_partials(const float *part_o, const float *part_ml, int n_split,
                                                     int n_b, int b, float out_scale, float *out, int tid,
                                                     int nthr) {
    static_assert(DH % 4 == 0, "float4 columns");
    constexpr int N4 = H * DH / 4;
    constexpr int PF = 16;
    const float4 *pob4 = reinterpret_cast<const float4 *>(part_o + (size_t)b * n_split * H * DH);
    const float2 *pmb2 = reinterpret_cast<const float2 *>(part_ml + (size_t)b * n_split * H * 2);
    for (int c4 = tid; c4 < N4; c4 += nthr) {
        const int head = (c4 * 4) / DH;
        float4 pre[PF];
        float2 st[PF];
#pragma unroll
        for (int i = 0; i < PF; ++i)
            if (i < n_b) {
                pre[i] = __ldcg(pob4 + (size_t)i * N4 + c4);
                st[i] = __ldcg(pmb2 + (size_t)i * H + head);
            }
        float M = -INFINITY;
#pragma unroll
        for (int i = 0; i < PF; ++i)
            if (i < n_b) M = fmaxf(M, st[i].x);
        for (int i = PF; i < n_b; ++i) M = fmaxf(M, __ldcg(pmb2 + (size_t)i * H + head).x);
        float d = 0.f;
        float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < PF; ++i)
            if (i < n_b) {
                const float w = st[i].x == -INFINITY ? 0.f : exp2f(st[i].x - M);
                d += w * st[i].y;
                num.x += w * pre[i].x;
                num.y += w * pre[i].y;
                num.z += w * pre[i].z;
                num.w += w * pre[i].w;
            }
#pragma unroll 4
        for (int i = PF; i < n_b; ++i) {
            const float2 sv = __ldcg(pmb2 + (size_t)i * H + head);
            const float4 v = __ldcg(pob4 + (size_t)i * N4 + c4);
            const float w = sv.x == -INFINITY ? 0.f : exp2f(sv.x - M);
            d += w * sv.y;
            num.x += w * v.x;
            num.y += w * v.y;
            num.z += w * v.z;
            num.w += w * v.w;
        }
        const float f = d > 0.f ? out_scale / d : 0.f;
        reinterpret_cast<float4 *>(out + (size_t)b * H * DH)[c4] =
            make_float4(num.x * f, num.y * f, num.z * f, num.w * f);
    }
}

}  // namespace kpa
