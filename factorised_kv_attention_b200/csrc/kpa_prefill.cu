// kpa_prefill.cu -- causal chunked attention in factor space on the tcgen05 tensor cores.
//
// Row t of sequence b is the query at position start_pos[b] + t; it attends to cache
// slots 0 .. start_pos[b] + t.  Keys and values exist only as factors in the cache
// ("Kronecker Product Attention", eqs 3-4, B^K pre-rotated per Theorem 2.4); each
// 128-token K and V tile of one head is rebuilt on chip,
//     K[s][(j1,j2)] = sum_r A^K_r(s)[i1,j1] B~^K_r(s)[i2,j2]     (1/R_K folded into the scale)
//     V[s][(j1,j2)] = sum_r A^V_r(s)[i1,j1] B^V_r(s)[i2,j2]      (1/R_V folded into the output)
// straight into the 128-byte-swizzled K-major layouts that tcgen05.mma reads, and is
// never written to device memory.  The tensor-core operands are fp16 (K, V and P
// are rounded once to an 11-bit significand, 4x finer than bf16; the bf16 Q tile is
// converted in place); a value outside the fp16 range is reported as
// KPA_ERR_DEVICE_CHECK.  Then, per tile (FlashAttention-style):
//     S = Q K^T on the tensor cores into TMEM; the softmax warps (one query row per
//     thread) read S, apply the causal mask and the online softmax, write P in bf16
//     back to shared memory and, when a row's running max grew, rescale that row of
//     the TMEM output accumulator; then O += P V on the tensor cores, in TMEM.
// Warps 0-3: softmax / output rows.  Warps 4-7: K/V reconstruction (one tile ahead,
// double-buffered).  Warp 8: TMEM allocation, the Q tile's TMA load, MMA issue.
#include <cudaTypedefs.h>

#include <cuda_fp16.h>

#include "kpa_internal.cuh"
#include "kpa_sm100.cuh"

namespace kpa {

struct PrefillArgs {
    int batch, n_tok, cap;
    const int32_t *start_pos;
    const __nv_bfloat16 *kc, *vc;
    float *out;
    float qscale;       // sm_scale / R_K * log2(e)
    float out_scale;    // 1 / R_V
    int h1, h2;
    int *err;
    unsigned long long wait_limit_ns;
};

namespace {

using namespace sm100;

constexpr int TQ = 128, TK = 128;
constexpr int kThreads = 288;
constexpr uint32_t kTmemCols = 256;        // S: columns 0..127, O accumulator: 128..255

template <int D1_, int D2_, int RK_, int RV_>
struct PrefillCfg {
    static constexpr int D1 = D1_, D2 = D2_, RK = RK_, RV = RV_;
    static constexpr int DH = D1 * D2;
    static constexpr int NH = DH / 64;             // 64-feature halves of a row
    static_assert(DH == 64 || DH == 128, "head dim 64 or 128");
    static_assert(D2 % 8 == 0, "d2 must be a multiple of 8");
    static constexpr uint32_t Q_BYTES = TQ * DH * 2;
    static constexpr uint32_t K_BYTES = TK * DH * 2;
    static constexpr uint32_t V_BYTES = DH * TK * 2;
    static constexpr uint32_t P_BYTES = TQ * TK * 2;
    static constexpr size_t OFF_Q = 0;
    static constexpr size_t OFF_K = OFF_Q + Q_BYTES;                 // 2 buffers
    static constexpr size_t OFF_V = OFF_K + 2 * K_BYTES;             // 2 buffers
    static constexpr size_t OFF_P = OFF_V + 2 * V_BYTES;
    static constexpr size_t OFF_BAR = OFF_P + P_BYTES;
    static constexpr size_t SMEM = 1024 + OFF_BAR + 64;
};

// Byte offset of element k (0..63) of row `row` in a 128-byte-swizzled K-major block.
__device__ __forceinline__ uint32_t sw128(int row, int k) {
    return (uint32_t)row * 128 + ((((uint32_t)k >> 3) ^ ((uint32_t)row & 7)) << 4) + ((uint32_t)k & 7) * 2;
}

constexpr float kHalfMax = 65504.f;

// Eight floats as fp16; `big` records whether any lies outside the fp16 range.
__device__ __forceinline__ uint4 pack8(const float (&x)[8], bool &big) {
    uint4 u;
    uint32_t *p = reinterpret_cast<uint32_t *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        big |= fabsf(x[2 * i]) > kHalfMax || fabsf(x[2 * i + 1]) > kHalfMax;
        __half2 h = __floats2half2_rn(x[2 * i], x[2 * i + 1]);
        p[i] = *reinterpret_cast<uint32_t *>(&h);
    }
    return u;
}

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <class C>
__global__ void __launch_bounds__(kThreads, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tmq, PrefillArgs a) {
    constexpr int D1 = C::D1, D2 = C::D2, RK = C::RK, RV = C::RV, DH = C::DH, NH = C::NH;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);    // q, s, pv
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 3);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_qt = (a.n_tok + TQ - 1) / TQ;
    const int qt = n_qt - 1 - (int)blockIdx.x;                // longest rows first
    const int head = blockIdx.y, b = blockIdx.z;
    const int h = a.h1 * a.h2, i1 = head / a.h2, i2 = head % a.h2;
    const int q0 = qt * TQ;
    const int start = a.start_pos[b];
    int max_slot = start + min(q0 + TQ, a.n_tok) - 1;          // last slot any row of the tile sees
    if (max_slot >= a.cap || start < 0) {
        if (tid == 0) raise_error(a.err, kErrDeviceCheck);
        max_slot = min(max_slot, a.cap - 1);
    }
    const int n_kt = max_slot >= 0 ? max_slot / TK + 1 : 0;
    const uint32_t bar_q = smem_u32(bars), bar_s = bar_q + 8, bar_pv = bar_q + 16;
    const uint64_t limit = a.wait_limit_ns;

    if (tid == 0) {
        mbar_init(bar_q, 1);
        mbar_init(bar_s, 1);
        mbar_init(bar_pv, 1);
        mbar_fence_init();
    }
    if (warp == 8) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (tid == 8 * 32) {           // the Q tile: rows q0.. of sequence b, this head's DH columns
        mbar_expect_tx(bar_q, C::Q_BYTES);
#pragma unroll
        for (int hh = 0; hh < NH; ++hh)
            tma_load_2d(smem_u32(smem + C::OFF_Q + hh * TQ * 128), &tmq, head * DH + hh * 64, b * a.n_tok + q0, bar_q);
    }

    const int ek = RK * (a.h1 * D1 + a.h2 * D2), ev = RV * (a.h1 * D1 + a.h2 * D2);
    const __nv_bfloat16 *kcb = a.kc + (size_t)b * a.cap * ek;
    const __nv_bfloat16 *vcb = a.vc + (size_t)b * a.cap * ev;

    // ---- reconstruction of tile kt into buffer kt % 2 (warps 4..7)
    auto rebuild = [&](int kt) {
        const int rt = tid - 128;
        bool big = false;
        unsigned char *kbuf = smem + C::OFF_K + (kt & 1) * C::K_BYTES;
        unsigned char *vbuf = smem + C::OFF_V + (kt & 1) * C::V_BYTES;
        // K: thread = token row
        {
            const int slot = kt * TK + rt;
            float A[RK][D1], B[RK][D2];
            const bool live = slot <= max_slot;
            if (live) {
                const __nv_bfloat16 *base = kcb + ((size_t)(slot / kGroup) * ek) * kGroup + (slot % kGroup);
#pragma unroll
                for (int r = 0; r < RK; ++r) {
#pragma unroll
                    for (int j1 = 0; j1 < D1; ++j1)
                        A[r][j1] = __bfloat162float(base[(size_t)(r * a.h1 * D1 + i1 * D1 + j1) * kGroup]);
#pragma unroll
                    for (int j2 = 0; j2 < D2; ++j2)
                        B[r][j2] = __bfloat162float(
                            base[(size_t)(RK * a.h1 * D1 + r * a.h2 * D2 + i2 * D2 + j2) * kGroup]);
                }
            }
#pragma unroll
            for (int j1 = 0; j1 < D1; ++j1)
#pragma unroll
                for (int c8 = 0; c8 < D2; c8 += 8) {
                    float x[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        float acc = 0.f;
                        if (live) {
#pragma unroll
                            for (int r = 0; r < RK; ++r) acc += A[r][j1] * B[r][c8 + u];
                        }
                        x[u] = acc;
                    }
                    const int f = j1 * D2 + c8;                          // first feature of the chunk
                    *reinterpret_cast<uint4 *>(kbuf + (f / 64) * (TK * 128) + sw128(rt, f % 64)) = pack8(x, big);
                }
        }
        // V^T: thread = feature row f, tokens in 16-byte groups of 8
        if (rt < DH) {
            const int f = rt, j1 = f / D2, j2 = f % D2;
#pragma unroll 4
            for (int g = 0; g < TK / kGroup; ++g) {
                const int slot0 = kt * TK + g * kGroup;
                float x[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) x[u] = 0.f;
                if (slot0 <= max_slot) {
                    const __nv_bfloat16 *gb = vcb + (size_t)(slot0 / kGroup) * ev * kGroup;
#pragma unroll
                    for (int r = 0; r < RV; ++r) {
                        const uint4 av = *reinterpret_cast<const uint4 *>(gb + (size_t)(r * a.h1 * D1 + i1 * D1 + j1) * kGroup);
                        const uint4 bv = *reinterpret_cast<const uint4 *>(
                            gb + (size_t)(RV * a.h1 * D1 + r * a.h2 * D2 + i2 * D2 + j2) * kGroup);
                        const __nv_bfloat162 *ap = reinterpret_cast<const __nv_bfloat162 *>(&av);
                        const __nv_bfloat162 *bp = reinterpret_cast<const __nv_bfloat162 *>(&bv);
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const float2 af = __bfloat1622float2(ap[u]), bf = __bfloat1622float2(bp[u]);
                            x[2 * u] += af.x * bf.x;
                            x[2 * u + 1] += af.y * bf.y;
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        if (slot0 + u > max_slot) x[u] = 0.f;
                }
                const int tk = g * kGroup;                               // first token of the chunk
                *reinterpret_cast<uint4 *>(vbuf + (tk / 64) * (DH * 128) + sw128(f, tk % 64)) = pack8(x, big);
            }
        }
        if (big) raise_error(a.err, kErrDeviceCheck);
        fence_async_smem();        // visible to the tensor cores
    };

    if (warp >= 4 && warp < 8 && n_kt > 0) rebuild(0);

    // softmax-row state (warps 0..3)
    const int row = (warp & 3) * 32 + lane;
    const int pos = start + q0 + row;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;

    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // the bf16 Q tile becomes fp16 in place once its copy has landed
    if (warp < 4) {
        if (!mbar_wait(bar_q, 0, limit)) {
            raise_error(a.err, kErrTimeout);
            ok = false;
        }
        bool big = false;
        uint4 *qt4 = reinterpret_cast<uint4 *>(smem + C::OFF_Q);
        for (int i = tid; i < (int)(C::Q_BYTES / 16); i += 128) {
            uint4 u = qt4[i];
            uint32_t *w = reinterpret_cast<uint32_t *>(&u);
            float x[8];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&w[k]));
                x[2 * k] = f.x;
                x[2 * k + 1] = f.y;
            }
            qt4[i] = pack8(x, big);
        }
        if (big) raise_error(a.err, kErrDeviceCheck);
        fence_async_smem();
    }
    if (warp < 4 || warp == 8) asm volatile("bar.sync 1, 160;" ::: "memory");

    const uint32_t idesc_s = umma_idesc_f16_f32(TQ, TK), idesc_o = umma_idesc_f16_f32(TQ, DH);
    const uint32_t srow = tmem + ((uint32_t)((warp & 3) * 32) << 16);    // this row's S columns
    const uint32_t orow = srow + 128;                                     // this row's O columns
    for (int kt = 0; kt < n_kt; ++kt) {
        const int buf = kt & 1;
        if (tid == 8 * 32) {                                           // S = Q K^T
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < DH / 16; ++k) {
                const uint64_t qd = umma_desc_k_sw128(smem_u32(smem + C::OFF_Q + (k / 4) * TQ * 128)) + 2 * (k % 4);
                const uint64_t kd = umma_desc_k_sw128(
                                        smem_u32(smem + C::OFF_K + buf * C::K_BYTES + (k / 4) * TK * 128)) +
                                    2 * (k % 4);
                umma_bf16(tmem, qd, kd, idesc_s, k > 0);
            }
            umma_commit(bar_s);
        }
        if (warp >= 4 && warp < 8 && kt + 1 < n_kt) rebuild(kt + 1);
        if (warp < 4) {
            if (!mbar_wait(bar_s, kt & 1, limit)) {
                raise_error(a.err, kErrTimeout);
                ok = false;
            }
            tc_fence_after();
            const int slot0 = kt * TK;
            float mx = -INFINITY;
#pragma unroll 1
            for (int c = 0; c < TK / 16; ++c) {
                float v[16];
                tmem_ld16(srow + c * 16, v);
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (slot0 + c * 16 + j <= pos) mx = fmaxf(mx, v[j] * a.qscale);
            }
            const float m_new = fmaxf(m_run, mx);
            const float alpha = m_run == -INFINITY ? 0.f : exp2f(m_run - m_new);
            float sum = 0.f;
            unsigned char *pbuf = smem + C::OFF_P;
#pragma unroll 1
            for (int c = 0; c < TK / 16; ++c) {
                float v[16];
                tmem_ld16(srow + c * 16, v);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int slot = slot0 + c * 16 + j;
                    v[j] = (slot <= pos && m_new != -INFINITY) ? exp2f(v[j] * a.qscale - m_new) : 0.f;
                    sum += v[j];
                }
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float x[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) x[u] = v[hh * 8 + u];
                    const int tk = c * 16 + hh * 8;
                    bool unused = false;
                    *reinterpret_cast<uint4 *>(pbuf + (tk / 64) * (TQ * 128) + sw128(row, tk % 64)) = pack8(x, unused);
                }
            }
            l_run = l_run * alpha + sum;
            m_run = m_new;
            // the accumulator row follows the new max before P V is added to it
            // (tcgen05.ld/st are warp-collective: the warp rescales if any of its rows must)
            if (kt > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
                for (int c = 0; c < DH / 16; ++c) {
                    float v[16];
                    tmem_ld16(orow + c * 16, v);
#pragma unroll
                    for (int j = 0; j < 16; ++j) v[j] *= alpha;
                    tmem_st16(orow + c * 16, v);
                }
                tmem_st_wait();
            }
            fence_async_smem();
            tc_fence_before();
        }
        if (warp < 4 || warp == 8) asm volatile("bar.sync 1, 160;" ::: "memory");     // P written
        if (tid == 8 * 32) {                                           // O += P V
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < TK / 16; ++k) {
                const uint64_t pd = umma_desc_k_sw128(smem_u32(smem + C::OFF_P + (k / 4) * TQ * 128)) + 2 * (k % 4);
                const uint64_t vd = umma_desc_k_sw128(
                                        smem_u32(smem + C::OFF_V + buf * C::V_BYTES + (k / 4) * DH * 128)) +
                                    2 * (k % 4);
                umma_bf16(tmem + 128, pd, vd, idesc_o, kt > 0 || k > 0);
            }
            umma_commit(bar_pv);
        }
        if (warp < 4 && !mbar_wait(bar_pv, kt & 1, limit)) {
            raise_error(a.err, kErrTimeout);
            ok = false;
        }
        tc_fence_before();
        __syncthreads();           // next tile rebuilt; S, P and the accumulator free again
        tc_fence_after();
    }

    if (warp < 4) {
        const bool write = q0 + row < a.n_tok && ok && n_kt > 0;
        const float inv = l_run > 0.f ? a.out_scale / l_run : 0.f;
        float *dst = a.out + (((size_t)b * a.n_tok + q0 + row) * h + head) * DH;
#pragma unroll 1
        for (int c = 0; c < DH / 16; ++c) {
            float v[16];
            tmem_ld16(orow + c * 16, v);                                // warp-collective
            if (write)
#pragma unroll
                for (int j = 0; j < 16; j += 4)
                    *reinterpret_cast<float4 *>(dst + c * 16 + j) =
                        make_float4(v[j] * inv, v[j + 1] * inv, v[j + 2] * inv, v[j + 3] * inv);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

using PrefillKpaH4x4D8x16R2 = PrefillCfg<8, 16, 2, 2>;

bool make_q_map(CUtensorMap *map, const void *q, uint64_t rows, uint64_t cols) {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) != cudaSuccess ||
            qr != cudaDriverEntryPointSuccess)
            return false;
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)TQ};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(q), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool prefill_supported(const Dims &d) {
    return d.d1 == PrefillKpaH4x4D8x16R2::D1 && d.d2 == PrefillKpaH4x4D8x16R2::D2 &&
           d.rk == PrefillKpaH4x4D8x16R2::RK && d.rv == PrefillKpaH4x4D8x16R2::RV;
}

cudaError_t launch_prefill(const Dims &d, int batch, int n_tok, const void *q, const int32_t *start_pos,
                           const void *kc, const void *vc, int cap, float qscale, float out_scale,
                           float *out, int *err, unsigned long long wait_limit_ns, cudaStream_t st) {
    using C = PrefillKpaH4x4D8x16R2;
    if (!prefill_supported(d)) return cudaErrorInvalidValue;
    PrefillArgs a;
    a.batch = batch;
    a.n_tok = n_tok;
    a.cap = cap;
    a.start_pos = start_pos;
    a.kc = static_cast<const __nv_bfloat16 *>(kc);
    a.vc = static_cast<const __nv_bfloat16 *>(vc);
    a.out = out;
    a.qscale = qscale;
    a.out_scale = out_scale;
    a.h1 = d.h1;
    a.h2 = d.h2;
    a.err = err;
    a.wait_limit_ns = wait_limit_ns;
    CUtensorMap tmq;
    if (!make_q_map(&tmq, q, (uint64_t)batch * n_tok, (uint64_t)d.h * d.dh)) return cudaErrorInvalidValue;
    cudaError_t e = ensure_dynamic_smem<prefill_kernel<C>>(C::SMEM);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((n_tok + TQ - 1) / TQ), (unsigned)d.h, (unsigned)batch);
    prefill_kernel<C><<<grid, kThreads, C::SMEM, st>>>(tmq, a);
    return cudaGetLastError();
}

}  // namespace kpa
