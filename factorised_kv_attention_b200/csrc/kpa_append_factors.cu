// kpa_append_factors.cu -- write factor records into the interleaved cache.
//
// "Kronecker Product Attention", section 2.5 and Theorem 2.4: the cache keeps
// A^K, A^V and B^V as projected and B^K rotated at the token's position by
// R_theta^(2)(pos); nothing else is rotated.  With one B shared by keys and values
// ("Tensor Product Attention Is All You Need", section 5) B is stored unrotated and
// the value record holds A^V only.  A third-order TPA record [a | b | c] has its b
// factors rotated instead (R_{d_b}(pos) (x) I_{d_c}, the same paper's Appendix C).
//
// One CTA owns one 8-token cache group of one plane of one sequence: it reads the
// (up to) 8 natural-layout records of that group, rotates the B^K pairs and
// stores the group element-major, token-minor, so a fully covered group is
// written with one 16-byte store per element (bf16) and no read-modify-write.
#include "kpa_internal.cuh"

namespace kpa {
namespace {

__device__ __forceinline__ int64_t floor_div8(int64_t a) { return a >= 0 ? a / 8 : -((-a + 7) / 8); }

template <typename T> struct Pack8;
template <> struct Pack8<__nv_bfloat16> {
    // 8 bf16 = one 16-byte store
    static __device__ __forceinline__ void store(__nv_bfloat16 *dst, const __nv_bfloat16 (&v)[8]) {
        uint4 u;
        __nv_bfloat162 *p = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
        for (int k = 0; k < 4; ++k) p[k] = __halves2bfloat162(v[2 * k], v[2 * k + 1]);
        *reinterpret_cast<uint4 *>(dst) = u;
    }
};
template <> struct Pack8<float> {
    static __device__ __forceinline__ void store(float *dst, const float (&v)[8]) {
        *reinterpret_cast<float4 *>(dst) = make_float4(v[0], v[1], v[2], v[3]);
        *reinterpret_cast<float4 *>(dst + 4) = make_float4(v[4], v[5], v[6], v[7]);
    }
};

template <typename T>
__global__ void __launch_bounds__(256)
append_factors_kernel(Dims d, int n_tok, const T *__restrict__ kf, const T *__restrict__ vf,
                      const int32_t *__restrict__ start_pos, const int32_t *__restrict__ pos_offset, int cap,
                      T *__restrict__ kc, T *__restrict__ vc, RopeTable rope, int *err) {
    __shared__ float2 cs[kGroup][kMaxHalfD2];   // (cos, sin) per token of the group, per m

    const int b = blockIdx.y;
    const bool is_k = blockIdx.z == 0;
    const int E = is_k ? d.ek : d.ev;
    const int64_t start = start_pos[b];
    const int64_t g = floor_div8(start) + blockIdx.x;
    const int64_t s_lo = max(g * kGroup, start);
    const int64_t s_hi = min(g * kGroup + kGroup, start + (int64_t)n_tok);
    if (s_lo >= s_hi) return;                     // past the last group of this sequence
    if (s_lo < 0 || s_hi > cap) {
        if (threadIdx.x == 0) raise_error(err, kErrDeviceCheck);
    }
    const int64_t v_lo = max(s_lo, (int64_t)0), v_hi = min(s_hi, (int64_t)cap);
    if (v_lo >= v_hi) return;                     // nothing of this group lies in the cache
    const bool full = (v_lo == g * kGroup) && (v_hi == g * kGroup + kGroup);

    const T *src = (is_k ? kf : vf) + ((size_t)b * n_tok) * E;
    T *dst = (is_k ? kc : vc) + ((size_t)b * cap) * E + (size_t)g * E * kGroup;

    // the rotated factor: B^K (length d2, after the A factors), or for a third-order
    // record [a | b | c] the b factors (length d1, after the a factors)
    const int R = is_k ? d.rk : d.rv;
    const int period = d.order == 3 ? d.d1 : d.d2;
    const int half = period / 2;
    const int a_size = d.order == 3 ? R * d.h1 : R * d.h1 * d.d1;
    const int rot_end = d.order == 3 ? a_size + R * d.d1 : E;
    const bool rot_k = is_k && !d.shared;         // a shared B is stored unrotated
    if (rot_k) {
        // the position of slot s is s, or s + pos_offset[b] for a cache that holds a range of
        // a longer sequence
        const int64_t off = pos_offset ? (int64_t)pos_offset[b] : 0;
        for (int i = threadIdx.x; i < kGroup * half; i += blockDim.x) {
            const int k = i / half, m = i % half;
            float c, s;
            rope_cs((double)(g * kGroup + k + off), rope.theta[m], c, s);
            cs[k][m] = make_float2(c, s);
        }
        __syncthreads();
    }

    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const bool rot = rot_k && e >= a_size && e < rot_end;
        int partner = e, j2 = 0;
        if (rot) {
            j2 = (e - a_size) % period;
            partner = (j2 & 1) ? e - 1 : e + 1;
        }
        T vals[kGroup];
#pragma unroll
        for (int k = 0; k < kGroup; ++k) {
            const int64_t s = g * kGroup + k;
            vals[k] = T(0.f);
            if (s < v_lo || s >= v_hi) continue;
            const T *row = src + (size_t)(s - start) * E;
            if (!rot) {
                vals[k] = row[e];
            } else {
                const float self = to_f32(row[e]), other = to_f32(row[partner]);
                const float2 w = cs[k][j2 >> 1];
                // pair (x0, x1) -> (x0 c - x1 s, x0 s + x1 c)
                const float r = (j2 & 1) ? (other * w.y + self * w.x) : (self * w.x - other * w.y);
                vals[k] = from_f32<T>(r);
            }
        }
        T *out = dst + (size_t)e * kGroup;
        if (full) {
            Pack8<T>::store(out, vals);
        } else {
#pragma unroll
            for (int k = 0; k < kGroup; ++k) {
                const int64_t s = g * kGroup + k;
                if (s >= v_lo && s < v_hi) out[k] = vals[k];
            }
        }
    }
}

}  // namespace

cudaError_t launch_append_factors(const Dims &d, kpa_dtype dt, int batch, int n_tok,
                                  const void *kf, const void *vf, const int32_t *start_pos,
                                  const int32_t *pos_offset, int cap, void *kc, void *vc, const RopeTable &rope,
                                  int *err, cudaStream_t st) {
    // a run of n_tok slots touches at most n_tok/8 + 2 groups
    dim3 grid((unsigned)(n_tok / kGroup + 2), (unsigned)batch, 2);
    if (dt == KPA_BF16)
        append_factors_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
            d, n_tok, (const __nv_bfloat16 *)kf, (const __nv_bfloat16 *)vf, start_pos, pos_offset, cap,
            (__nv_bfloat16 *)kc, (__nv_bfloat16 *)vc, rope, err);
    else
        append_factors_kernel<float><<<grid, 256, 0, st>>>(d, n_tok, (const float *)kf,
                                                           (const float *)vf, start_pos, pos_offset, cap,
                                                           (float *)kc, (float *)vc, rope, err);
    return cudaGetLastError();
}

}  // namespace kpa
