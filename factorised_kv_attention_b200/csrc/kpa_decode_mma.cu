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
// STAGES-deep shared-memory ring with cp.async.bulk (TMA, no multicast) and
// mbarrier transaction counts; consumer warps read the 8-token groups, whose
// element-major/token-minor layout makes every fragment load a conflict-free
// 16-byte row (ldmatrix) or 32-bit word (two adjacent tokens).  Every wait is
// bounded; on expiry the kernel records KPA_ERR_TIMEOUT, drains its copies and
// returns.
#include "kpa_internal.cuh"
#include "kpa_mma_decode.cuh"

namespace kpa {
namespace {

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of an mbarrier, for at most limit_ns nanoseconds.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15) == 0 && globaltimer() - t0 > limit_ns) return false;
    }
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
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

__device__ __forceinline__ uint32_t pack_bf16(float lo_elem, float hi_elem) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo_elem, hi_elem);
    return *reinterpret_cast<uint32_t *>(&v);
}

// x ~= hi + lo with both parts bf16; returns the packed pairs for (x0, x1).
__device__ __forceinline__ void split_pack(float x0, float x1, uint32_t &hi, uint32_t &lo) {
    const __nv_bfloat16 h0 = __float2bfloat16_rn(x0), h1 = __float2bfloat16_rn(x1);
    __nv_bfloat162 H = __halves2bfloat162(h0, h1);
    hi = *reinterpret_cast<uint32_t *>(&H);
    lo = pack_bf16(x0 - __bfloat162float(h0), x1 - __bfloat162float(h1));
}

__device__ __forceinline__ float2 lds_bf16x2(const unsigned char *p) {
    const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162 *>(p);
    return __bfloat1622float2(v);
}

__device__ __forceinline__ uint32_t mask_pair(uint32_t v, bool keep0, bool keep1) {
    return (keep0 ? (v & 0xffffu) : 0u) | (keep1 ? (v & 0xffff0000u) : 0u);
}

// ------------------------------------------------------------------- kernel
template <class C>
__global__ void __launch_bounds__((C::WARPS + 1) * 32, 1)
decode_mma_kernel(const __nv_bfloat16 *__restrict__ q, const int32_t *__restrict__ q_pos,
                  const __nv_bfloat16 *__restrict__ kc, const __nv_bfloat16 *__restrict__ vc,
                  int cap, const int32_t *__restrict__ seq_len, int max_len, float qscale,
                  int tps, int n_split, float *__restrict__ part_o, float *__restrict__ part_ml,
                  RopeTable rope, int *err, DecodeTestHooks hooks) {
    constexpr int MA = C::MA, D1 = C::D1, D2 = C::D2, RK = C::RK, RV = C::RV, H2 = C::H2;
    constexpr int H1 = MA / D1, H = H1 * H2, DH = D1 * D2;
    constexpr int MT = MA / 16, KS = D2 / 16, NT = D2 / 8;
    constexpr int EK = C::EK, EV = C::EV;
    constexpr int WARPS = C::WARPS, SLICES = C::SLICES, CHUNKS = C::CHUNKS, STAGES = C::STAGES;
    constexpr int TT = C::TT;
    constexpr int KBYTES = TT * EK * 2, STAGE_BYTES = C::STAGE_BYTES;

    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char *stage_base = smem;                                     // STAGES x (K | V)
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);  // full, empty
    float *qs = reinterpret_cast<float *>(bars + 2 * STAGES);             // [H][DH] query
    volatile int *abort_flag = reinterpret_cast<volatile int *>(qs + H * DH);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.y, split = blockIdx.x;

    int L = seq_len[b];
    if (L > max_len || L < 0) {
        if (split == 0 && tid == 0) raise_error(err, kErrDeviceCheck);
        L = L < 0 ? 0 : max_len;
    }
    const int t0 = split * tps;
    if (t0 >= L) return;                                   // empty split
    const int t1 = min(t0 + tps, L);
    const int n_tiles = (t1 - t0 + TT - 1) / TT;

    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + STAGES);
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, WARPS);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // rotated, scaled query in fp32 (consumer threads; the producer starts right away)
    if (warp < WARPS) {
        const __nv_bfloat16 *qb = q + (size_t)b * H * DH;
        const bool rotate = q_pos != nullptr;
        const double qp = rotate ? (double)q_pos[b] : 0.0;
        for (int i = tid; i < H * DH / 2; i += WARPS * 32) {
            const float x0 = __bfloat162float(qb[2 * i]), x1 = __bfloat162float(qb[2 * i + 1]);
            float y0 = x0, y1 = x1;
            if (rotate) {
                float c, s;
                rope_cs(qp, rope.theta[((2 * i) % D2) >> 1], c, s);
                y0 = x0 * c - x1 * s;
                y1 = x0 * s + x1 * c;
            }
            qs[2 * i] = y0 * qscale;
            qs[2 * i + 1] = y1 * qscale;
        }
    }
    __syncthreads();

    const uint64_t limit = hooks.wait_limit_ns;
    const __nv_bfloat16 *kb = kc + ((size_t)b * cap + t0) * EK;   // group-aligned (t0 % 8 == 0)
    const __nv_bfloat16 *vb = vc + ((size_t)b * cap + t0) * EV;

    // ------------------------------------------------------------ producer
    if (warp == WARPS) {
        if (lane == 0) {
            int issued = 0;
            bool ok = true;
            for (int t = 0; t < n_tiles && ok; ++t) {
                const int s = t % STAGES;
                if (t >= STAGES) {
                    if (!mbar_wait_bounded(empty0 + 8 * s, ((t / STAGES) - 1) & 1, limit)) {
                        raise_error(err, kErrTimeout);
                        *abort_flag = 1;
                        ok = false;
                        break;
                    }
                }
                if (*abort_flag) break;
                const int n = min(TT, t1 - t0 - t * TT);
                const int groups = (n + kGroup - 1) / kGroup;
                const uint32_t kbytes = (uint32_t)groups * EK * kGroup * 2;
                const uint32_t vbytes = (uint32_t)groups * EV * kGroup * 2;
                if (hooks.skip_tile == t && split == hooks.skip_split && b == 0) {
                    issued = t + 1;          // test hook: this tile never arrives
                    continue;
                }
                const uint32_t dst = smem_u32(stage_base + (size_t)s * STAGE_BYTES);
                mbar_expect_tx(full0 + 8 * s, kbytes + vbytes);
                bulk_g2s(dst, kb + (size_t)t * TT * EK, kbytes, full0 + 8 * s);
                bulk_g2s(dst + KBYTES, vb + (size_t)t * TT * EV, vbytes, full0 + 8 * s);
                issued = t + 1;
            }
            // drain: every copy this thread issued must land before the CTA exits
            for (int t = max(0, issued - STAGES); t < issued; ++t) {
                if (hooks.skip_tile == t && split == hooks.skip_split && b == 0) continue;
                if (!mbar_wait_bounded(full0 + 8 * (t % STAGES), (t / STAGES) & 1, limit))
                    raise_error(err, kErrTimeout);
            }
        }
        return;
    }

    // ------------------------------------------------------------ consumers
    const int i2 = warp % H2, slice = warp / H2;
    const int g = lane >> 2, c = lane & 3;

    // query fragments (A operand, row = (i1, j1), k = j2), hi and lo parts
    uint32_t qa_hi[MT][KS][4], qa_lo[MT][KS][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int ks = 0; ks < KS; ++ks)
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const int row = mt * 16 + g + ((v & 1) ? 8 : 0);
                const int j2 = ks * 16 + 2 * c + ((v & 2) ? 8 : 0);
                const int i1 = row / D1, j1 = row % D1;
                const float *src = qs + (i1 * H2 + i2) * DH + j1 * D2 + j2;
                split_pack(src[0], src[1], qa_hi[mt][ks][v], qa_lo[mt][ks][v]);
            }

    // running softmax state per owned row (rows g and g+8 of each m-tile), per lane
    float m_run[MT][2], l_run[MT][2];
    float o[MT][NT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        m_run[mt][0] = m_run[mt][1] = -INFINITY;
        l_run[mt][0] = l_run[mt][1] = 0.f;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
    }

    constexpr int A_K = RK * MA;                 // start of B^K in a key record
    constexpr int A_V = RV * MA;
    bool aborted = false;

    for (int t = 0; t < n_tiles; ++t) {
        const int s = t % STAGES;
        if (!mbar_wait_bounded(full0 + 8 * s, (t / STAGES) & 1, limit)) {
            raise_error(err, kErrTimeout);
            *abort_flag = 1;
            aborted = true;
            break;
        }
        const unsigned char *kt = stage_base + (size_t)s * STAGE_BYTES;
        const unsigned char *vt = kt + KBYTES;
        const int n_valid = min(TT, t1 - t0 - t * TT);           // tokens of this tile
        const int tok_base = slice * CHUNKS * 16;                 // this warp's first token

        float sc[CHUNKS][MT][2][4];                               // scores, then weights
#pragma unroll
        for (int ch = 0; ch < CHUNKS; ++ch) {
            const int tok0 = tok_base + ch * 16;
            const int grp0 = tok0 >> 3;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int gi = 0; gi < 2; ++gi)
#pragma unroll
                    for (int v = 0; v < 4; ++v) sc[ch][mt][gi][v] = 0.f;
            if (tok0 >= n_valid) continue;                        // whole chunk past the tail
#pragma unroll
            for (int r = 0; r < RK; ++r) {
#pragma unroll
                for (int gi = 0; gi < 2; ++gi) {
                    const unsigned char *grp = kt + (size_t)(grp0 + gi) * EK * 16;
                    // B~^K_r(token)[i2, :] as the B operand: rows j2, 8 tokens each (.trans)
                    uint32_t bk[KS][2];
                    const int e_b = A_K + r * H2 * D2 + i2 * D2;
                    if constexpr (KS % 2 == 0) {
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
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int ks = 0; ks < KS; ++ks) {
                            mma16816(acc, qa_hi[mt][ks], bk[ks][0], bk[ks][1]);
                            mma16816(acc, qa_lo[mt][ks], bk[ks][0], bk[ks][1]);
                        }
                        // times A^K_r(token)[i1, j1] for rows g and g+8, tokens 2c and 2c+1
                        const int row0 = mt * 16 + g;
                        const float2 a0 = lds_bf16x2(grp + (size_t)(r * MA + row0) * 16 + 4 * c);
                        const float2 a1 = lds_bf16x2(grp + (size_t)(r * MA + row0 + 8) * 16 + 4 * c);
                        sc[ch][mt][gi][0] += acc[0] * a0.x;
                        sc[ch][mt][gi][1] += acc[1] * a0.y;
                        sc[ch][mt][gi][2] += acc[2] * a1.x;
                        sc[ch][mt][gi][3] += acc[3] * a1.y;
                    }
                }
            }
            // sum over j1: rows of one head are D1 consecutive rows
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int gi = 0; gi < 2; ++gi) {
                    float *v = sc[ch][mt][gi];
                    if constexpr (D1 == 16) {
                        v[0] += v[2]; v[1] += v[3];
                    }
#pragma unroll
                    for (int off = 4; off < 4 * (D1 < 8 ? D1 : 8); off <<= 1) {
#pragma unroll
                        for (int k = 0; k < 4; ++k) v[k] += __shfl_xor_sync(0xffffffffu, v[k], off);
                    }
                    if constexpr (D1 == 16) {
                        v[2] = v[0]; v[3] = v[1];
                    }
                    // tokens past the tile's valid range
                    const int tk = tok0 + gi * 8 + 2 * c;
                    if (tk >= n_valid) { v[0] = -INFINITY; v[2] = -INFINITY; }
                    if (tk + 1 >= n_valid) { v[1] = -INFINITY; v[3] = -INFINITY; }
                }
        }
        // chunks entirely past the tail
#pragma unroll
        for (int ch = 0; ch < CHUNKS; ++ch)
            if (tok_base + ch * 16 >= n_valid)
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int gi = 0; gi < 2; ++gi)
#pragma unroll
                        for (int v = 0; v < 4; ++v) sc[ch][mt][gi][v] = -INFINITY;

        // online softmax over this tile (log2 domain), per owned row
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                float mx = -INFINITY;
#pragma unroll
                for (int ch = 0; ch < CHUNKS; ++ch)
#pragma unroll
                    for (int gi = 0; gi < 2; ++gi)
                        mx = fmaxf(mx, fmaxf(sc[ch][mt][gi][2 * hr], sc[ch][mt][gi][2 * hr + 1]));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                const float m_new = fmaxf(m_run[mt][hr], mx);
                const float alpha = (m_run[mt][hr] == -INFINITY) ? 0.f : exp2f(m_run[mt][hr] - m_new);
                float sum = 0.f;
#pragma unroll
                for (int ch = 0; ch < CHUNKS; ++ch)
#pragma unroll
                    for (int gi = 0; gi < 2; ++gi)
#pragma unroll
                        for (int k = 0; k < 2; ++k) {
                            float &x = sc[ch][mt][gi][2 * hr + k];
                            x = (m_new == -INFINITY) ? 0.f : exp2f(x - m_new);
                            sum += x;
                        }
                l_run[mt][hr] = l_run[mt][hr] * alpha + sum;
                m_run[mt][hr] = m_new;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    o[mt][nt][2 * hr] *= alpha;
                    o[mt][nt][2 * hr + 1] *= alpha;
                }
            }

        // values
#pragma unroll
        for (int ch = 0; ch < CHUNKS; ++ch) {
            const int tok0 = tok_base + ch * 16;
            if (tok0 >= n_valid) continue;
            const int grp0 = tok0 >> 3;
            const bool tail = tok0 + 16 > n_valid;
            const unsigned char *g0p = vt + (size_t)grp0 * EV * 16;
            const unsigned char *g1p = g0p + (size_t)EV * 16;
#pragma unroll
            for (int r = 0; r < RV; ++r) {
                // A operand: P'[(i1,j1), k] = p * A^V_r, k = (group, token); hi/lo split
                uint32_t pa_hi[MT][4], pa_lo[MT][4];
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    const int row0 = mt * 16 + g;
                    const float2 a00 = lds_bf16x2(g0p + (size_t)(r * MA + row0) * 16 + 4 * c);
                    const float2 a10 = lds_bf16x2(g0p + (size_t)(r * MA + row0 + 8) * 16 + 4 * c);
                    const float2 a01 = lds_bf16x2(g1p + (size_t)(r * MA + row0) * 16 + 4 * c);
                    const float2 a11 = lds_bf16x2(g1p + (size_t)(r * MA + row0 + 8) * 16 + 4 * c);
                    const float *p0 = sc[ch][mt][0], *p1 = sc[ch][mt][1];
                    // weights of masked tokens are exactly 0; keep garbage factors out
                    const float w00 = p0[0] != 0.f ? p0[0] * a00.x : 0.f;
                    const float w01 = p0[1] != 0.f ? p0[1] * a00.y : 0.f;
                    const float w10 = p0[2] != 0.f ? p0[2] * a10.x : 0.f;
                    const float w11 = p0[3] != 0.f ? p0[3] * a10.y : 0.f;
                    const float w20 = p1[0] != 0.f ? p1[0] * a01.x : 0.f;
                    const float w21 = p1[1] != 0.f ? p1[1] * a01.y : 0.f;
                    const float w30 = p1[2] != 0.f ? p1[2] * a11.x : 0.f;
                    const float w31 = p1[3] != 0.f ? p1[3] * a11.y : 0.f;
                    split_pack(w00, w01, pa_hi[mt][0], pa_lo[mt][0]);
                    split_pack(w10, w11, pa_hi[mt][1], pa_lo[mt][1]);
                    split_pack(w20, w21, pa_hi[mt][2], pa_lo[mt][2]);
                    split_pack(w30, w31, pa_hi[mt][3], pa_lo[mt][3]);
                }
                const int e_b = A_V + r * H2 * D2 + i2 * D2;
                const int mat = lane >> 3, mrow = lane & 7;
#pragma unroll
                for (int np = 0; np < NT / 2; ++np) {
                    // B operand: B^V_r(token)[i2, j2], rows j2 (8 tokens each), no transpose
                    const unsigned char *gp = (mat & 1) ? g1p : g0p;
                    uint32_t b00, b01, b10, b11;
                    ldsm_x4(smem_u32(gp + (size_t)(e_b + (2 * np + (mat >> 1)) * 8 + mrow) * 16), b00, b01,
                            b10, b11);
                    if (tail) {
                        const int tk = tok0 + 2 * c;
                        b00 = mask_pair(b00, tk < n_valid, tk + 1 < n_valid);
                        b10 = mask_pair(b10, tk < n_valid, tk + 1 < n_valid);
                        b01 = mask_pair(b01, tk + 8 < n_valid, tk + 9 < n_valid);
                        b11 = mask_pair(b11, tk + 8 < n_valid, tk + 9 < n_valid);
                    }
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        mma16816(o[mt][2 * np], pa_hi[mt], b00, b01);
                        mma16816(o[mt][2 * np], pa_lo[mt], b00, b01);
                        mma16816(o[mt][2 * np + 1], pa_hi[mt], b10, b11);
                        mma16816(o[mt][2 * np + 1], pa_lo[mt], b10, b11);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * s);
        if (*abort_flag) { aborted = true; break; }
    }

    // l: sum over the four lanes (c) that share a row
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            float l = l_run[mt][hr];
            l += __shfl_xor_sync(0xffffffffu, l, 1);
            l += __shfl_xor_sync(0xffffffffu, l, 2);
            l_run[mt][hr] = l;
        }

    // merge the token slices of the CTA through shared memory (reuses the ring)
    asm volatile("bar.sync 1, %0;" ::"n"(WARPS * 32));
    if (aborted || *abort_flag) return;
    float *mo = reinterpret_cast<float *>(smem);                   // [SLICES][H][DH]
    float *mm = mo + SLICES * H * DH;                              // [SLICES][H][2]
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const int row = mt * 16 + g + 8 * hr;
            const int i1 = row / D1, j1 = row % D1;
            const int head = i1 * H2 + i2;
            float *dst = mo + ((size_t)slice * H + head) * DH + j1 * D2;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                *reinterpret_cast<float2 *>(dst + nt * 8 + 2 * c) =
                    make_float2(o[mt][nt][2 * hr], o[mt][nt][2 * hr + 1]);
            if (c == 0 && j1 == 0) {
                mm[((size_t)slice * H + head) * 2] = m_run[mt][hr];
                mm[((size_t)slice * H + head) * 2 + 1] = l_run[mt][hr];
            }
        }
    asm volatile("bar.sync 1, %0;" ::"n"(WARPS * 32));
    float *po = part_o + ((size_t)(b * n_split + split) * H) * DH;
    float *pml = part_ml + ((size_t)(b * n_split + split) * H) * 2;
    for (int idx = tid; idx < H * DH; idx += WARPS * 32) {
        const int head = idx / DH;
        float M = -INFINITY;
#pragma unroll
        for (int sl = 0; sl < SLICES; ++sl) M = fmaxf(M, mm[((size_t)sl * H + head) * 2]);
        float acc = 0.f, l = 0.f;
#pragma unroll
        for (int sl = 0; sl < SLICES; ++sl) {
            const float ms = mm[((size_t)sl * H + head) * 2];
            const float wgt = ms == -INFINITY ? 0.f : exp2f(ms - M);
            acc += wgt * mo[((size_t)sl * H) * DH + idx];
            l += wgt * mm[((size_t)sl * H + head) * 2 + 1];
        }
        po[idx] = acc;
        if (idx % DH == 0) {
            pml[2 * head] = M;
            pml[2 * head + 1] = l;
        }
    }
}

template <class C>
cudaError_t launch_cfg(int batch, const void *q, const int32_t *q_pos, const void *kc,
                       const void *vc, int cap, const int32_t *seq_len, int max_len, float qscale,
                       const DecodePlan &p, float *part_o, float *part_ml, const RopeTable &rope,
                       int *err, const DecodeTestHooks &hooks, cudaStream_t st) {
    auto kern = decode_mma_kernel<C>;
    const size_t smem = C::smem_bytes();
    cudaError_t e = ensure_dynamic_smem(kern, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)p.n_split, (unsigned)batch);
    kern<<<grid, (C::WARPS + 1) * 32, smem, st>>>(
        (const __nv_bfloat16 *)q, q_pos, (const __nv_bfloat16 *)kc, (const __nv_bfloat16 *)vc, cap,
        seq_len, max_len, qscale, p.tokens_per_split, p.n_split, part_o, part_ml, rope, err, hooks);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_mma(int variant, int batch, const void *q, const int32_t *q_pos,
                              const void *kc, const void *vc, int cap, const int32_t *seq_len,
                              int max_len, float qscale, const DecodePlan &plan, float *part_o,
                              float *part_ml, const RopeTable &rope, int *err,
                              const DecodeTestHooks &hooks, cudaStream_t st) {
    switch (variant) {
#define KPA_MMA_CASE(IDX, CFG)                                                                     \
    case IDX:                                                                                      \
        return launch_cfg<CFG>(batch, q, q_pos, kc, vc, cap, seq_len, max_len, qscale, plan, part_o, \
                               part_ml, rope, err, hooks, st);
        KPA_MMA_VARIANTS(KPA_MMA_CASE)
#undef KPA_MMA_CASE
        default:
            return cudaErrorInvalidValue;
    }
}

}  // namespace kpa
