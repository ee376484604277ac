// kpa_decode_order3.cu -- decode over a third-order TPA factor cache (CUDA cores).
//
// Third-order TPA ("Tensor Product Attention Is All You Need", Appendix C, as the
// explainer page summarises it): the key of head h at slot t is
//   K_t[h, :] = (1/R_K) sum_r a^K_r(t)[h] (b~^K_r(t) (x) c^K_r(t)),
// b in R^{d_b}, c in R^{d_c}, d_h = d_b d_c (b's index the slower one), with RoPE
// acting on b alone (R_{d_b}(t) (x) I_{d_c}, Theorem C.1); the cache stores b~^K
// already rotated.  Values likewise, unrotated.  Per cached token and head:
//   score   = sum_r a^K_r[h] sum_jb b~_r[jb] sum_jc Qs[h, jb d_c + jc] c_r[jc]
//   values  O[h, (jb, jc)] += sum_r (p[h] a^V_r[h]) b^V_r[jb] c^V_r[jc]
// where Qs is the query rotated by R_{d_b}(q_pos) (x) I_{d_c} and scaled by
// sm_scale / R_K * log2(e).  This kernel computes them as written, on the CUDA cores
// (a d_b x d_c bilinear form per head and a rank-R_V outer-product update), for the
// shapes and element types the tensor-core decode does not take: d_b = d_c = 8 in bf16
// runs there instead, with the features b (x) c formed in registers.  Here the FP32
// work, not HBM, bounds the decode: a record is only R (h + d_b + d_c) numbers.
//
// One CTA per (split, sequence), 8 warps.  A tile of 32 tokens (4 cache groups)
// is copied with cp.async into shared memory at a padded group stride, double
// buffered.  Warp w owns heads w, w + 8, ...: lane = token for the scores and the
// online softmax (so the running maximum and the weights p a^V stay in the warp),
// lane = output feature for the value accumulation.  Each CTA leaves an
// unnormalised partial (o, m, l) per head; the split combine merges them.
#include "kpa_internal.cuh"
#include "kpa_sm100.cuh"

namespace kpa {
namespace {

using sm100::cp_async16;

constexpr int kO3Threads = 256;
constexpr int kO3Tile = kOrder3Tile;  // tokens per tile (4 groups)
constexpr int kO3MaxHpw = 4;         // heads per warp (h <= 32)
constexpr int kO3MaxJpl = 8;         // output features per lane (d_h <= 256)
constexpr int kO3MaxDb = 16, kO3MaxDc = 16;

struct Order3Args {
    const void *q;
    const int32_t *q_pos;
    const void *kc, *vc;
    int cap;
    const int32_t *seq_len;
    int max_len, tps, n_split;
    int h, db, dc, rk, rv, ek, ev;
    float qscale;
    float *part_o, *part_ml;
    int *err;
};

// Shared memory: the query [h][d_h], the weights p a^V [h][R_V][32], the value outer
// products b^V (x) c^V of a tile [R_V][8][d_h][4] (4 tokens per float4), the rotation
// table, then the two tile buffers.
__host__ __device__ __forceinline__ size_t o3_bc_offset(int h, int dh, int rv) {
    return ((size_t)h * dh + (size_t)h * rv * kO3Tile) * 4;
}
__host__ __device__ __forceinline__ size_t o3_tiles_offset(int h, int dh, int rv) {
    return (o3_bc_offset(h, dh, rv) + (size_t)rv * kO3Tile * dh * 4 + (kO3MaxDb / 2) * 8 + 15) / 16 * 16;
}

template <typename T> __device__ __forceinline__ float ld_f32(const unsigned char *p);
template <> __device__ __forceinline__ float ld_f32<float>(const unsigned char *p) {
    return *reinterpret_cast<const float *>(p);
}
// a bf16 is the top half of its fp32 value: widen with a shift (integer pipe, exact)
template <> __device__ __forceinline__ float ld_f32<__nv_bfloat16>(const unsigned char *p) {
    return __uint_as_float((uint32_t)*reinterpret_cast<const unsigned short *>(p) << 16);
}

template <typename T>
__device__ __forceinline__ float elem(const unsigned char *tile, int gstride, int tok, int e) {
    return ld_f32<T>(tile + (tok >> 3) * gstride + (e * kGroup + (tok & 7)) * (int)sizeof(T));
}

// DB_, DC_: d_b and d_c at compile time (0: taken from the arguments, loops bounded by
// the largest supported sizes); HPW: heads per warp, ceil(h / 8).
template <typename T, int DB_, int DC_, int HPW>
__global__ void __launch_bounds__(kO3Threads) decode_order3_kernel(Order3Args a, RopeTable rope) {
    constexpr int MDB = DB_ ? DB_ : kO3MaxDb, MDC = DC_ ? DC_ : kO3MaxDc;      // loop bounds
    constexpr int JPL = DB_ && DC_ ? (DB_ * DC_ + 31) / 32 : kO3MaxJpl;         // features per lane
    const int H = a.h, DB = DB_ ? DB_ : a.db, DC = DC_ ? DC_ : a.dc, DH = DB * DC;
    const int RK = a.rk, RV = a.rv, EK = a.ek, EV = a.ev;
    const int GK = EK * kGroup * (int)sizeof(T) + 16, GV = EV * kGroup * (int)sizeof(T) + 16;
    const int TILE_BYTES = 4 * GK + 4 * GV;
    extern __shared__ float4 smem4[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(smem4);
    float *qs = reinterpret_cast<float *>(sm);                                       // [H][DH]
    float *wv = reinterpret_cast<float *>(sm + (size_t)H * DH * 4);                  // [H][RV][32] p a^V
    float4 *bcs = reinterpret_cast<float4 *>(sm + o3_bc_offset(H, DH, RV));       // [RV][8][DH] x 4 tokens
    float2 *cs = reinterpret_cast<float2 *>(sm + o3_bc_offset(H, DH, RV) + (size_t)RV * kO3Tile * DH * 4);
    unsigned char *tiles = sm + o3_tiles_offset(H, DH, RV);                          // 16-byte aligned

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.y, split = blockIdx.x;
    int L = a.seq_len[b];
    if (L > a.max_len || L < 0) {
        if (split == 0 && tid == 0) raise_error(a.err, kErrDeviceCheck);
        L = L < 0 ? 0 : a.max_len;
    }
    const int t0 = split * a.tps;
    if (t0 >= L) return;                                    // empty split: the combine skips it
    const int t1 = split == a.n_split - 1 ? L : min(t0 + a.tps, L);
    const int n_tiles = (t1 - t0 + kO3Tile - 1) / kO3Tile;
    const unsigned char *kbase = static_cast<const unsigned char *>(a.kc) + ((size_t)b * a.cap + t0) * EK * sizeof(T);
    const unsigned char *vbase = static_cast<const unsigned char *>(a.vc) + ((size_t)b * a.cap + t0) * EV * sizeof(T);

    // tile t: its groups (16-byte chunks) into buffer `buf` at the padded strides
    auto issue = [&](int t, int buf) {
        const int n = min(kO3Tile, t1 - t0 - t * kO3Tile);
        const int groups = (n + kGroup - 1) / kGroup;
        const int ck = EK * kGroup * (int)sizeof(T) / 16, cv = EV * kGroup * (int)sizeof(T) / 16;
        const uint32_t dst = (uint32_t)__cvta_generic_to_shared(tiles + (size_t)buf * TILE_BYTES);
        const unsigned char *ks = kbase + (size_t)t * kO3Tile * EK * sizeof(T);
        const unsigned char *vs = vbase + (size_t)t * kO3Tile * EV * sizeof(T);
        for (int c = tid; c < groups * (ck + cv); c += kO3Threads) {
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

    // the query rotated by R_{d_b}(q_pos) (x) I_{d_c} (pairs (2m, 2m+1) of b's index, for
    // every c index) and scaled
    const bool rotate = a.q_pos != nullptr;
    if (rotate && tid < DB / 2) {
        float c, s;
        rope_cs((double)a.q_pos[b], rope.theta[tid], c, s);
        cs[tid] = make_float2(c, s);
    }
    __syncthreads();
    const T *qb = static_cast<const T *>(a.q) + (size_t)b * H * DH;
    for (int i = tid; i < H * (DB / 2) * DC; i += kO3Threads) {
        const int h = i / ((DB / 2) * DC), rem = i % ((DB / 2) * DC), m = rem / DC, jc = rem % DC;
        const int e0 = h * DH + (2 * m) * DC + jc, e1 = e0 + DC;
        float x0 = to_f32(qb[e0]), x1 = to_f32(qb[e1]);
        if (rotate) {
            const float2 w = cs[m];
            const float y0 = x0 * w.x - x1 * w.y, y1 = x0 * w.y + x1 * w.x;
            x0 = y0;
            x1 = y1;
        }
        qs[e0] = x0 * a.qscale;
        qs[e1] = x1 * a.qscale;
    }

    float m_run[HPW], l_part[HPW], acc[HPW][JPL];
#pragma unroll
    for (int k = 0; k < HPW; ++k) {
        m_run[k] = -INFINITY;
        l_part[k] = 0.f;
#pragma unroll
        for (int i = 0; i < JPL; ++i) acc[k][i] = 0.f;
    }
    const int a_k = RK * H, b_k = a_k + RK * DB;           // first b, first c of a key record
    const int a_v = RV * H, c_v = a_v + RV * DB;            // first b, first c of a value record
    // this lane's output features j = lane + 32 i: byte offsets of b^V_0[j / d_c] and
    // c^V_0[j % d_c] inside a group (token 0), fixed for the whole split
    int vb_off[JPL], vc_off[JPL];
#pragma unroll
    for (int i = 0; i < JPL; ++i) {
        const int j = min(lane + 32 * i, DH - 1);
        vb_off[i] = (a_v + j / DC) * kGroup * (int)sizeof(T);
        vc_off[i] = (c_v + j % DC) * kGroup * (int)sizeof(T);
    }

    for (int t = 0; t < n_tiles; ++t) {
        const int buf = t & 1;
        if (t + 1 < n_tiles) {
            issue(t + 1, buf ^ 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();                                    // tile t (and, at t = 0, the query) ready
        const unsigned char *kt = tiles + (size_t)buf * TILE_BYTES;
        const unsigned char *vt = kt + 4 * GK;
        const int n_valid = min(kO3Tile, t1 - t0 - t * kO3Tile);
        const bool valid = lane < n_valid;

        // ---- scores (lane = token) and the online softmax of this warp's heads
        float sc[HPW];
#pragma unroll
        for (int k = 0; k < HPW; ++k) sc[k] = 0.f;
        for (int r = 0; r < RK; ++r) {
            float bf[MDB], cf[MDC];
#pragma unroll
            for (int j = 0; j < MDB; ++j) bf[j] = j < DB ? elem<T>(kt, GK, lane, a_k + r * DB + j) : 0.f;
#pragma unroll
            for (int j = 0; j < MDC; ++j) cf[j] = j < DC ? elem<T>(kt, GK, lane, b_k + r * DC + j) : 0.f;
#pragma unroll
            for (int k = 0; k < HPW; ++k) {
                const int h = warp + 8 * k;
                if (h < H) {
                    const float *qh = qs + h * DH;
                    float u = 0.f;
#pragma unroll
                    for (int jb = 0; jb < MDB; ++jb) {
                        if (jb < DB) {
                            float inner = 0.f;
#pragma unroll
                            for (int jc = 0; jc < MDC; ++jc)
                                if (jc < DC) inner = fmaf(qh[jb * DC + jc], cf[jc], inner);
                            u = fmaf(bf[jb], inner, u);
                        }
                    }
                    sc[k] = fmaf(elem<T>(kt, GK, lane, r * H + h), u, sc[k]);
                }
            }
        }
#pragma unroll
        for (int k = 0; k < HPW; ++k) {
            const int h = warp + 8 * k;
            if (h >= H) break;
            const float s = valid ? sc[k] : -INFINITY;
            float mx = s;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float m_new = fmaxf(m_run[k], mx);         // finite: the tile has a valid token
            const float alpha = exp2f(m_run[k] - m_new);
            const float p = valid ? exp2f(s - m_new) : 0.f;
            l_part[k] = fmaf(l_part[k], alpha, p);
            m_run[k] = m_new;
            for (int r = 0; r < RV; ++r)
                wv[(h * RV + r) * kO3Tile + lane] = valid ? p * elem<T>(vt, GV, lane, r * H + h) : 0.f;
#pragma unroll
            for (int i = 0; i < JPL; ++i) acc[k][i] *= alpha;
        }
        __syncwarp();

        // ---- values (lane = output feature): O[h, j] += sum_r w[h, r] b^V_r[j / d_c] c^V_r[j % d_c]
        if constexpr (DB_ != 0 && DC_ != 0) {
            // every thread forms outer products b^V_r (x) c^V_r for 4 tokens at a time
            // (float4 over the tokens), then each warp reads them with one 16-byte load per
            // (4 tokens, rank, feature) and its weights with one per (4 tokens, rank, head)
            constexpr int DHC = DB_ * DC_;
            for (int it = tid; it < RV * (kO3Tile / 4) * DHC; it += kO3Threads) {
                const int r = it / ((kO3Tile / 4) * DHC), rem = it % ((kO3Tile / 4) * DHC);
                const int t4 = rem / DHC, j = rem % DHC;
                float4 v;
                float *vp = reinterpret_cast<float *>(&v);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int t2 = 4 * t4 + u;
                    // slots past the tile's end may hold any bits: their product is 0
                    vp[u] = t2 < n_valid ? elem<T>(vt, GV, t2, a_v + r * DB_ + j / DC_) *
                                               elem<T>(vt, GV, t2, c_v + r * DC_ + j % DC_)
                                         : 0.f;
                }
                bcs[(r * (kO3Tile / 4) + t4) * DHC + j] = v;
            }
            __syncthreads();
            const int n4 = (n_valid + 3) / 4;                // weights past n_valid are 0
            for (int t4 = 0; t4 < n4; ++t4)
                for (int r = 0; r < RV; ++r) {
                    float4 bc[JPL], w[HPW];
#pragma unroll
                    for (int i = 0; i < JPL; ++i)
                        bc[i] = bcs[(r * (kO3Tile / 4) + t4) * DHC + min(lane + 32 * i, DHC - 1)];
#pragma unroll
                    for (int k = 0; k < HPW; ++k)
                        w[k] = warp + 8 * k < H
                                   ? reinterpret_cast<const float4 *>(wv + ((warp + 8 * k) * RV + r) * kO3Tile)[t4]
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int k = 0; k < HPW; ++k)
#pragma unroll
                        for (int i = 0; i < JPL; ++i) {
                            float a = acc[k][i];
                            a = fmaf(w[k].x, bc[i].x, a);
                            a = fmaf(w[k].y, bc[i].y, a);
                            a = fmaf(w[k].z, bc[i].z, a);
                            acc[k][i] = fmaf(w[k].w, bc[i].w, a);
                        }
                }
        } else {
            // (four tokens per step, so their loads are in flight together)
            for (int tt = 0; tt < n_valid; tt += 4) {
                const int cnt = min(4, n_valid - tt);
                for (int r = 0; r < RV; ++r) {
                    const int rb = r * DB * kGroup * (int)sizeof(T), rc = r * DC * kGroup * (int)sizeof(T);
                    float bc[4][JPL], w[4][HPW];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int t2 = tt + (u < cnt ? u : 0);          // a repeated token gets weight 0
                        const unsigned char *vg = vt + (t2 >> 3) * GV + (t2 & 7) * (int)sizeof(T);
#pragma unroll
                        for (int i = 0; i < JPL; ++i)
                            bc[u][i] = ld_f32<T>(vg + vb_off[i] + rb) * ld_f32<T>(vg + vc_off[i] + rc);
#pragma unroll
                        for (int k = 0; k < HPW; ++k)
                            w[u][k] = (u < cnt && warp + 8 * k < H) ? wv[((warp + 8 * k) * RV + r) * kO3Tile + t2] : 0.f;
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u)
#pragma unroll
                        for (int k = 0; k < HPW; ++k)
#pragma unroll
                            for (int i = 0; i < JPL; ++i) acc[k][i] = fmaf(w[u][k], bc[u][i], acc[k][i]);
                }
            }
        }
        __syncthreads();                                    // buffer `buf` is refilled next iteration
    }

    // ---- unnormalised partial (o, m, l) of this split
    float *po = a.part_o + ((size_t)(b * a.n_split + split) * H) * DH;
    float *pml = a.part_ml + ((size_t)(b * a.n_split + split) * H) * 2;
#pragma unroll
    for (int k = 0; k < HPW; ++k) {
        const int h = warp + 8 * k;
        if (h >= H) break;
        float l = l_part[k];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
#pragma unroll
        for (int i = 0; i < JPL; ++i) {
            const int j = lane + 32 * i;
            if (j < DH) po[h * DH + j] = acc[k][i];
        }
        if (lane == 0) *reinterpret_cast<float2 *>(pml + 2 * h) = make_float2(m_run[k], l);
    }
}

size_t order3_smem_bytes(const Dims &d, kpa_dtype dt) {
    const size_t es = dt == KPA_BF16 ? 2 : 4;
    const size_t tile = 4 * (d.ek * kGroup * es + 16) + 4 * (d.ev * kGroup * es + 16);
    return o3_tiles_offset(d.h, d.dh, d.rv) + 2 * tile;       // includes the outer products
}

}  // namespace

bool order3_decode_supported(const Dims &d, kpa_dtype dt) {
    return d.order == 3 && d.h2 == 1 && d.h <= 8 * kO3MaxHpw && d.d1 <= kO3MaxDb && d.d2 <= kO3MaxDc &&
           d.d1 % 2 == 0 && d.dh <= 32 * kO3MaxJpl && d.rk <= 64 && d.rv <= 64 &&
           order3_smem_bytes(d, dt) <= 200 * 1024;
}

// CTAs of the kernel this shape runs that one SM holds at once (occupancy query).
int order3_ctas_per_sm(const Dims &d, kpa_dtype dt) {
    const size_t smem = order3_smem_bytes(d, dt);
    const bool b8x8 = d.d1 == 8 && d.d2 == 8 && d.h <= 16;
    auto query = [&](auto kernel) -> int {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) {
            cudaGetLastError();
            return 1;
        }
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kO3Threads, smem) != cudaSuccess) {
            cudaGetLastError();
            return 1;
        }
        return n > 0 ? n : 1;
    };
    if (dt == KPA_BF16)
        return b8x8 ? query(decode_order3_kernel<__nv_bfloat16, 8, 8, 2>)
                    : query(decode_order3_kernel<__nv_bfloat16, 0, 0, kO3MaxHpw>);
    return b8x8 ? query(decode_order3_kernel<float, 8, 8, 2>) : query(decode_order3_kernel<float, 0, 0, kO3MaxHpw>);
}

cudaError_t launch_decode_order3(const Dims &d, kpa_dtype dt, int batch, const void *q, const int32_t *q_pos,
                                 const void *kc, const void *vc, int cap, const int32_t *seq_len, int max_len,
                                 float qscale, const DecodePlan &p, float *part_o, float *part_ml,
                                 const RopeTable &rope, int *err, cudaStream_t st) {
    Order3Args a;
    a.q = q;
    a.q_pos = q_pos;
    a.kc = kc;
    a.vc = vc;
    a.cap = cap;
    a.seq_len = seq_len;
    a.max_len = max_len;
    a.tps = p.tokens_per_split;
    a.n_split = p.n_split;
    a.h = d.h;
    a.db = d.d1;
    a.dc = d.d2;
    a.rk = d.rk;
    a.rv = d.rv;
    a.ek = d.ek;
    a.ev = d.ev;
    a.qscale = qscale;
    a.part_o = part_o;
    a.part_ml = part_ml;
    a.err = err;
    const size_t smem = order3_smem_bytes(d, dt);
    const dim3 grid((unsigned)p.n_split, (unsigned)batch);
    // d_b = d_c = 8 with h <= 16 (the benchmark shape) has its own instantiation; any other
    // covered shape runs the general one
    auto run = [&](auto kernel) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kernel<<<grid, kO3Threads, smem, st>>>(a, rope);
        return cudaGetLastError();
    };
    const bool b8x8 = d.d1 == 8 && d.d2 == 8 && d.h <= 16;
    if (dt == KPA_BF16)
        return b8x8 ? run(decode_order3_kernel<__nv_bfloat16, 8, 8, 2>) : run(decode_order3_kernel<__nv_bfloat16, 0, 0, kO3MaxHpw>);
    return b8x8 ? run(decode_order3_kernel<float, 8, 8, 2>) : run(decode_order3_kernel<float, 0, 0, kO3MaxHpw>);
}

}  // namespace kpa
