// kpa_decode_tc.cu -- TPA decode with both contractions on the tcgen05 tensor cores.
//
// TPA is the degenerate split of KPA (h1 = h, d1 = 1, h2 = 1): the cached key of
// head h is K_t[h, :] = (1/R_K) sum_r A^K_r(t)[h] B~^K_r(t) with B~ rotated at the
// key's slot, and the value likewise without rotation ("Kronecker Product
// Attention", Def 2.1 and Thm 2.4; "Tensor Product Attention Is All You Need",
// eq 2-3).  Per 128-token tile of one split:
//
//   score   U_r[t, n] = sum_j B~^K_r(t)[j] Qs[n, j], n = (head, hi | lo part of the
//           rotated, scaled query).  M = 128 tokens, N = 2h, K = d_h; A is the
//           cache tile as it lands (tokens are the contiguous dimension of each
//           8-token group: an MN-major operand), B the query in shared memory.
//           score[t, h] = sum_r A^K_r(t)[h] (U_r[t, (h, hi)] + U_r[t, (h, lo)]).
//   values  O_tile[(r, j), n] = sum_t B^V_r(t)[j] P'[t, n], n = (r', head, hi | lo),
//           P'_r'[t, h] = p[t, h] A^V_r'(t)[h] split into bf16 hi + lo.  M = R_V d_h =
//           128 (both ranks' value factors, K-major: within a group each element's
//           8 tokens are contiguous), N = 2 R_V h, K = tokens.  Only the blocks
//           r = r' of the product are read.
//
// Online softmax per head over the tile (base 2, the scale folded into the query);
// the CTA's 128 tokens share one running maximum per head, exchanged through shared
// memory once per tile.  Each tile's value product lands in its own tensor-memory
// buffer and is added to registers with that tile's rescale factor, so nothing in
// tensor memory is ever rescaled.
//
// Warps: 0-7 read the score rows of tensor-memory lanes 32 (w % 4) .. +31 (one token
// per thread) for heads 8 (w / 4) .. +7, form P', and accumulate the value rows of
// the same lanes (one (rank, feature) row per thread) for the same heads; warp 8
// streams the cache with bulk copies into a two-stage ring (each 8-token group at a
// padded stride, so per-token reads of the A factors hit distinct banks); warp 9
// owns tensor memory and issues the MMAs.  Every wait is bounded; a wait that runs
// out records KPA_ERR_TIMEOUT, and the CTA drains its copies and MMAs, frees its
// tensor memory and returns.
#include "kpa_decode_merge.cuh"
#include "kpa_internal.cuh"
#include "kpa_mma_decode.cuh"
#include "kpa_sm100.cuh"

namespace kpa {
namespace {

using namespace sm100;

// Compile-time shape of the kernel: TPA with h heads, head dimension d_h, rank R
// for keys and values.
template <int H_, int D2_, int R_>
struct TcDecodeCfg {
    static constexpr int H = H_, D2 = D2_, R = R_, DH = D2_;
    static constexpr int EK = R * (H + D2), EV = R * (H + D2);   // elements per key / value record
    static constexpr int A_K = R * H, A_V = R * H;               // first B element of a record
    static constexpr int TT = 128, GROUPS = TT / kGroup;         // tokens per tile, groups per tile
    static constexpr int GP = EK * kGroup * 2 + 16;              // padded group stride (bytes), keys
    static constexpr int GPV = EV * kGroup * 2 + 16;             // ... values
    static constexpr int KT_BYTES = GROUPS * GP, STAGE_BYTES = KT_BYTES + GROUPS * GPV;
    static constexpr int HB = H / 8;                             // blocks of 8 heads
    static constexpr int SW = 4 * HB;                            // softmax warps
    static constexpr int THREADS = (SW + 2) * 32;
    static constexpr int SN = 2 * H;                             // score columns per rank
    static constexpr int ON = R * SN;                            // value-product columns
    static constexpr int P_SBO = (TT / 8) * 128;                 // P': bytes between 8-column blocks
    static constexpr int P_BYTES = TT * ON * 2;
    static constexpr int Q_SBO = (D2 / 8) * 128;                 // query: bytes between 8-row blocks
    static constexpr int Q_BYTES = SN * D2 * 2;
    static constexpr int TMEM_S = 0, TMEM_O = 2 * R * SN, TMEM_COLS = 256;
    static constexpr size_t OFF_P = 2 * (size_t)STAGE_BYTES;
    static constexpr size_t OFF_Q = OFF_P + 2 * (size_t)P_BYTES;
    static constexpr size_t OFF_CS = OFF_Q + Q_BYTES;
    static constexpr size_t OFF_XM = OFF_CS + (D2 / 2) * 8;       // [2][4][H] tile maxima
    static constexpr size_t OFF_LP = OFF_XM + 2 * 4 * H * 4;      // [4][H] denominators
    static constexpr size_t OFF_OB = OFF_LP + 4 * H * 4;          // [H][DH] rank-1 half of O
    static constexpr size_t OFF_BARS = OFF_OB + (size_t)H * DH * 4;
    static constexpr size_t OFF_TMEM = OFF_BARS + 12 * 8;
    static constexpr size_t OFF_FLAGS = OFF_TMEM + 8;
    static constexpr size_t smem_bytes() { return OFF_FLAGS + 16; }
    static_assert(R == 2 && R * D2 == 128, "the value product stacks both ranks' d_h rows into M = 128");
    static_assert(H == 16, "two blocks of 8 heads: eight softmax warps");
    static_assert(D2 % 16 == 0 && SN % 16 == 0 && ON % 16 == 0 && ON <= 256, "MMA shapes");
    static_assert(TMEM_O + 2 * ON <= TMEM_COLS, "tensor memory columns");
    static_assert(GP % 16 == 0 && GPV % 16 == 0 && (OFF_P % 16) == 0 && (OFF_Q % 16) == 0, "16-byte rows");
    static_assert(smem_bytes() <= 227 * 1024, "shared memory");
};

using TcTpaH16D64R2 = TcDecodeCfg<16, 64, 2>;

// Shared-memory descriptor of an operand in the no-swizzle layout: 8 x 16-byte core
// matrices (128 contiguous bytes), `lbo` bytes apart along K, `sbo` bytes apart along
// M or N, whichever operand major-ness the instruction descriptor states.
__device__ __forceinline__ uint64_t desc_plain(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | ((uint64_t)1 << 46);
}

__device__ __forceinline__ float warp_max(float v) {
    float r;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
    return r;
}

// Named barrier 1 over the softmax warps; returns the OR of `pred` over them.
template <int N>
__device__ __forceinline__ bool softmax_bar_or(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "n"(N)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ float lds_bf16(const unsigned char *p) {
    return __uint_as_float((uint32_t)*reinterpret_cast<const unsigned short *>(p) << 16);
}

// (x.x, x.y) -> bf16 hi + lo pairs (low half = x.x); hi + lo equals x to ~2^-16.
__device__ __forceinline__ void split_bf16(float x0, float x1, uint32_t &hi, uint32_t &lo) {
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(hi) : "f"(x1), "f"(x0));
    const float r0 = x0 - __uint_as_float(hi << 16), r1 = x1 - __uint_as_float(hi & 0xffff0000u);
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(lo) : "f"(r1), "f"(r0));
}

// Bounded wait that also gives up once another role has aborted the CTA.
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, uint64_t limit_ns, volatile int *flags,
                                              int *err) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15) == 0) {
            if (flags[0]) return false;
            if (globaltimer() - t0 > limit_ns) {
                raise_error(err, kErrTimeout);
                flags[0] = 1;
                return false;
            }
        }
    }
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1) decode_tc_kernel(DecodeArgs a, RopeTable rope, DecodeTestHooks hooks) {
    constexpr int H = C::H, D2 = C::D2, R = C::R, DH = C::DH, TT = C::TT, EK = C::EK, EV = C::EV;
    constexpr int SW = C::SW, SN = C::SN, ON = C::ON;
    constexpr int PRODUCER = SW, ISSUER = SW + 1;
    // score: M = 128 tokens (A MN-major), N = 2h; values: M = 128 rows, N = 2 R h (B MN-major)
    constexpr uint32_t IDESC_S = umma_idesc_bf16_f32(128, SN) | (1u << 15);
    constexpr uint32_t IDESC_O = umma_idesc_bf16_f32(128, ON) | (1u << 16);

    extern __shared__ __align__(1024) unsigned char smem[];
    const uint32_t full0 = smem_u32(smem + C::OFF_BARS);   // [2] tile landed
    const uint32_t empty0 = full0 + 16;                      // [2] stage free (value MMAs done)
    const uint32_t sfull0 = full0 + 32;                      // [2] score product in tensor memory
    const uint32_t pfull0 = full0 + 48;                      // [2] P' written (one arrival per softmax warp)
    const uint32_t ofull0 = full0 + 64;                      // [2] value product in tensor memory
    const uint32_t done_bar = full0 + 80;                    // every MMA of the CTA completed
    volatile int *flags = reinterpret_cast<volatile int *>(smem + C::OFF_FLAGS);   // abort, last CTA
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_TMEM);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.y, split = blockIdx.x;
    const int t0 = split * a.tps;
    const __nv_bfloat16 *kb = a.kc + ((size_t)b * a.cap + t0) * EK;   // group-aligned (t0 % 8 == 0)
    const __nv_bfloat16 *vb = a.vc + ((size_t)b * a.cap + t0) * EV;
    // tile t of this split, its first n slots: every group into the stage at its padded stride
    auto issue_tile = [&](int t, int n, uint32_t bar) {
        const int groups = (n + kGroup - 1) / kGroup;
        const uint32_t dst = smem_u32(smem + (size_t)(t & 1) * C::STAGE_BYTES);
        mbar_expect_tx(bar, (uint32_t)groups * (EK + EV) * kGroup * 2);
        for (int g = 0; g < groups; ++g) {
            const size_t tok = (size_t)t * TT + (size_t)g * kGroup;
            bulk_g2s(dst + g * C::GP, kb + tok * EK, EK * kGroup * 2, bar);
            bulk_g2s(dst + C::KT_BYTES + g * C::GPV, vb + tok * EV, EV * kGroup * 2, bar);
        }
    };

    if (tid == PRODUCER * 32) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
            mbar_init(sfull0 + 8 * s, 1);
            mbar_init(pfull0 + 8 * s, SW);
            mbar_init(ofull0 + 8 * s, 1);
        }
        mbar_init(done_bar, 1);
        flags[0] = 0;
        flags[1] = 0;
        mbar_fence_init();
    }
    // launched with programmatic stream serialization: wait for the previous grid before
    // reading any input, and let the next grid be scheduled now
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");

    // The first tile's copy starts before the sequence length is known: slots
    // [t0, t0 + TT) clipped to max_len are inside the cache whatever the length.
    const int spec_n = min(TT, a.max_len - t0);
    const bool spec = spec_n > 0 && !(hooks.skip_tile == 0 && split == hooks.skip_split && b == 0);
    if (tid == PRODUCER * 32 && spec) issue_tile(0, spec_n, full0);

    const bool rotate = a.q_pos != nullptr;
    int L = a.seq_len[b];
    const double qpos = rotate ? (double)a.q_pos[b] : 0.0;
    constexpr int QPT = (H * DH / 2) / (SW * 32);   // query pairs per softmax thread
    static_assert(QPT * SW * 32 == H * DH / 2, "query pairs spread evenly");
    __nv_bfloat162 qv[QPT];
    if (warp < SW) {
        const __nv_bfloat162 *qb = reinterpret_cast<const __nv_bfloat162 *>(a.q + (size_t)b * H * DH);
#pragma unroll
        for (int k = 0; k < QPT; ++k) qv[k] = qb[tid + k * SW * 32];
    }
    if (L > a.max_len || L < 0) {
        if (split == 0 && tid == 0) raise_error(a.err, kErrDeviceCheck);
        L = L < 0 ? 0 : a.max_len;
    }
    const uint64_t limit = hooks.wait_limit_ns;
    if (t0 >= L) {                                       // empty split: its speculative copy lands first
        if (a.fused && L == 0 && split == 0)             // an empty sequence gets zeros
            for (int i = tid; i < H * DH; i += C::THREADS) a.out[(size_t)b * H * DH + i] = 0.f;
        if (tid == PRODUCER * 32 && spec && !mbar_wait(full0, 0, limit)) raise_error(a.err, kErrTimeout);
        return;
    }
    // the last split runs to the end of the sequence (it may hold up to 5/4 of a split)
    const int t1 = max(t0, split == a.n_split - 1 ? L : min(t0 + a.tps, L));
    const int n_tiles = (t1 - t0 + TT - 1) / TT;

    if (warp == ISSUER) tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t qop = smem_u32(smem + C::OFF_Q);

    if (warp == PRODUCER) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int issued = spec ? 1 : 0;
            for (int t = spec ? 1 : 0; t < n_tiles; ++t) {
                const int s = t & 1;
                if (t >= 2 && !wait_or_abort(empty0 + 8 * s, ((t >> 1) - 1) & 1, limit, flags, a.err)) break;
                if (flags[0]) break;
                issued = t + 1;
                if (hooks.skip_tile == t && split == hooks.skip_split && b == 0) continue;
                issue_tile(t, min(TT, t1 - t0 - t * TT), full0 + 8 * s);
            }
            // every copy issued for this CTA lands before it exits
            for (int t = max(0, issued - 2); t < issued; ++t) {
                if (hooks.skip_tile == t && split == hooks.skip_split && b == 0) continue;
                if (!mbar_wait(full0 + 8 * (t & 1), (t >> 1) & 1, limit)) raise_error(a.err, kErrTimeout);
            }
        }
        __syncwarp();
    } else if (warp == ISSUER) {
        // ------------------------------------------------------------ MMA issuer
        tmem_relinquish();
        asm volatile("bar.sync 2, %0;" ::"n"((SW + 1) * 32));   // query operand written
        if (lane == 0) {
            auto issue_scores = [&](int t) {
                const int s = t & 1;
                tc_fence_after();
                const uint32_t kst = smem_u32(smem + (size_t)s * C::STAGE_BYTES);
#pragma unroll
                for (int r = 0; r < R; ++r)
#pragma unroll
                    for (int ks = 0; ks < D2 / 16; ++ks)
                        umma_bf16(tmem + C::TMEM_S + s * R * SN + r * SN,
                                  desc_plain(kst + (uint32_t)(C::A_K + r * D2 + ks * 16) * 16, 128, C::GP),
                                  desc_plain(qop + ks * 256, 128, C::Q_SBO), IDESC_S, ks > 0);
                umma_commit(sfull0 + 8 * s);
            };
            int next_s = 0;                                  // next tile whose score product is issued
            bool ok = true;
            for (int t = 0; t < n_tiles && ok; ++t) {
                const int s = t & 1;
                // issue the scores of tiles up to t + 1 as they land; the values of tile t once
                // its P' is written (its score buffer is then free for tile t + 2)
                const uint64_t w0 = globaltimer();
                for (uint32_t it = 1;; ++it) {
                    if (next_s <= t + 1 && next_s < n_tiles &&
                        mbar_try_wait(full0 + 8 * (next_s & 1), (next_s >> 1) & 1)) {
                        issue_scores(next_s++);
                        continue;
                    }
                    if (next_s > t && mbar_try_wait(pfull0 + 8 * s, (t >> 1) & 1)) break;
                    if ((it & 15) == 0) {
                        if (flags[0]) { ok = false; break; }
                        if (globaltimer() - w0 > limit) {
                            raise_error(a.err, kErrTimeout);
                            flags[0] = 1;
                            ok = false;
                            break;
                        }
                    }
                }
                if (!ok) break;
                tc_fence_after();
                const int n_valid = min(TT, t1 - t0 - t * TT);
                const uint32_t vst = smem_u32(smem + (size_t)s * C::STAGE_BYTES + C::KT_BYTES);
                const uint32_t pst = smem_u32(smem + C::OFF_P + (size_t)s * C::P_BYTES);
                for (int j = 0; j < (n_valid + 15) / 16; ++j)
                    umma_bf16(tmem + C::TMEM_O + s * ON,
                              desc_plain(vst + (uint32_t)(2 * j) * C::GPV + C::A_V * 16, C::GPV, 128),
                              desc_plain(pst + j * 256, 128, C::P_SBO), IDESC_O, j > 0);
                umma_commit(ofull0 + 8 * s);
                umma_commit(empty0 + 8 * s);
            }
            umma_commit(done_bar);
            if (!mbar_wait(done_bar, 0, limit)) raise_error(a.err, kErrTimeout);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax and O
        const int q4 = warp & 3, hb = warp >> 2;
        const int tok = 32 * q4 + lane;                      // this thread's token (score lane)
        const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
        float2 *cs = reinterpret_cast<float2 *>(smem + C::OFF_CS);
        float *xm = reinterpret_cast<float *>(smem + C::OFF_XM);
        float *lp = reinterpret_cast<float *>(smem + C::OFF_LP);
        float *ob = reinterpret_cast<float *>(smem + C::OFF_OB);

        // rotated, scaled query: I_{d1} (x) R^(2)(q_pos) on the pairs (2m, 2m+1), split into
        // bf16 hi and lo rows n = (head block, part, head % 8) of a K-major operand
        if (rotate && tid < D2 / 2) {
            float cth, sth;
            rope_cs_fast(qpos, rope.theta[tid], cth, sth);
            cs[tid] = make_float2(cth, sth);
        }
        asm volatile("bar.sync 1, %0;" ::"n"(SW * 32));
#pragma unroll
        for (int k = 0; k < QPT; ++k) {
            const int pr = tid + k * SW * 32;
            const int h = pr / (D2 / 2), d = 2 * (pr % (D2 / 2));
            float2 x = __bfloat1622float2(qv[k]);
            if (rotate) {
                const float2 w = cs[d >> 1];
                x = make_float2(x.x * w.x - x.y * w.y, x.x * w.y + x.y * w.x);
            }
            uint32_t hi, lo;
            split_bf16(x.x * a.qscale, x.y * a.qscale, hi, lo);
#pragma unroll
            for (int hl = 0; hl < 2; ++hl) {
                const int n = (h >> 3) * 16 + hl * 8 + (h & 7);
                *reinterpret_cast<uint32_t *>(smem + C::OFF_Q + (n >> 3) * C::Q_SBO + (d >> 3) * 128 + (n & 7) * 16 +
                                              (d & 7) * 2) = hl ? lo : hi;
            }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        asm volatile("bar.sync 2, %0;" ::"n"((SW + 1) * 32));

        float mrun[8], lrun[8], o[8], apend[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            mrun[j] = -INFINITY;
            lrun[j] = 0.f;
            o[j] = 0.f;
            apend[j] = 0.f;
        }
        bool failed = false;
        // add tile tp's value product (rows of this thread's lane, heads of its block)
        auto accumulate = [&](int tp, const float (&al)[8]) {
            const int s2 = tp & 1;
            if (!failed) failed = !wait_or_abort(ofull0 + 8 * s2, (tp >> 1) & 1, limit, flags, a.err);
            if (failed) return;
            tc_fence_after();
            float ov[16];
            tmem_ld16(tmem + lane_off + C::TMEM_O + s2 * ON + (q4 >> 1) * SN + hb * 16, ov);
#pragma unroll
            for (int j = 0; j < 8; ++j) o[j] = fmaf(o[j], al[j], ov[j] + ov[8 + j]);
        };

        for (int t = 0; t < n_tiles; ++t) {
            const int s = t & 1;
            const uint32_t ph = (t >> 1) & 1;
            const int n_valid = min(TT, t1 - t0 - t * TT);
            const bool valid = tok < n_valid;
            const unsigned char *krow = smem + (size_t)s * C::STAGE_BYTES + (tok >> 3) * C::GP + (tok & 7) * 2;
            unsigned char *vrow = smem + (size_t)s * C::STAGE_BYTES + C::KT_BYTES + (tok >> 3) * C::GPV + (tok & 7) * 2;
            if (!failed) failed = !wait_or_abort(full0 + 8 * s, ph, limit, flags, a.err);
            if (!failed) failed = !wait_or_abort(sfull0 + 8 * s, ph, limit, flags, a.err);
            float sc[8];
            if (!failed) {
                tc_fence_after();
                float u[R][16];
#pragma unroll
                for (int r = 0; r < R; ++r) tmem_ld16(tmem + lane_off + C::TMEM_S + s * R * SN + r * SN + hb * 16, u[r]);
#pragma unroll
                for (int j = 0; j < 8; ++j) sc[j] = 0.f;
#pragma unroll
                for (int r = 0; r < R; ++r)
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        sc[j] = fmaf(lds_bf16(krow + (r * H + hb * 8 + j) * 16), u[r][j] + u[r][8 + j], sc[j]);
                float mx[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (!valid) sc[j] = -INFINITY;
                    mx[j] = warp_max(sc[j]);
                }
                if (lane == 0) {
                    float4 *dst = reinterpret_cast<float4 *>(xm + (s * 4 + q4) * H + hb * 8);
                    dst[0] = make_float4(mx[0], mx[1], mx[2], mx[3]);
                    dst[1] = make_float4(mx[4], mx[5], mx[6], mx[7]);
                }
            }
            if (softmax_bar_or<SW * 32>(failed)) {
                failed = true;
                break;
            }
            // the tile's maximum per head over the four lane quarters; weights and P'
            float p[8], alpha[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float tm = xm[(s * 4) * H + hb * 8 + j];
#pragma unroll
                for (int qq = 1; qq < 4; ++qq) tm = fmaxf(tm, xm[(s * 4 + qq) * H + hb * 8 + j]);
                const float mn = fmaxf(mrun[j], tm);
                alpha[j] = exp2f(mrun[j] - mn);
                p[j] = valid ? exp2f(sc[j] - mn) : 0.f;
                lrun[j] = fmaf(lrun[j], alpha[j], p[j]);
                mrun[j] = mn;
            }
            unsigned char *prow = smem + C::OFF_P + (size_t)s * C::P_BYTES + tok * 16;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const float x0 = valid ? p[2 * jj] * lds_bf16(vrow + (r * H + hb * 8 + 2 * jj) * 16) : 0.f;
                    const float x1 = valid ? p[2 * jj + 1] * lds_bf16(vrow + (r * H + hb * 8 + 2 * jj + 1) * 16) : 0.f;
                    split_bf16(x0, x1, hi[jj], lo[jj]);
                }
                const int nb = r * (SN / 8) + hb * 2;
                *reinterpret_cast<uint4 *>(prow + nb * C::P_SBO) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4 *>(prow + (nb + 1) * C::P_SBO) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
            if (!valid) {
                // a slot past the split's end: zero its value factors (the copy may not have
                // covered it), so the value product adds exactly 0 for it
                for (int k = hb * (R * D2 / C::HB); k < (hb + 1) * (R * D2 / C::HB); ++k)
                    *reinterpret_cast<unsigned short *>(vrow + (C::A_V + k) * 16) = 0;
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(pfull0 + 8 * s);
            if (t > 0) accumulate(t - 1, apend);
#pragma unroll
            for (int j = 0; j < 8; ++j) apend[j] = alpha[j];
        }
        if (!failed && n_tiles > 0) accumulate(n_tiles - 1, apend);
        tc_fence_before();

        // denominators: sum over this warp's 32 tokens; O: add the rank-1 rows to the rank-0 rows
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) lrun[j] += __shfl_xor_sync(0xffffffffu, lrun[j], off);
        if (lane == 0) {
            float4 *dst = reinterpret_cast<float4 *>(lp + q4 * H + hb * 8);
            dst[0] = make_float4(lrun[0], lrun[1], lrun[2], lrun[3]);
            dst[1] = make_float4(lrun[4], lrun[5], lrun[6], lrun[7]);
        }
        const int dim = (q4 & 1) * 32 + lane;
        if (q4 >= 2) {
#pragma unroll
            for (int j = 0; j < 8; ++j) ob[(hb * 8 + j) * DH + dim] = o[j];
        }
        const bool ok = !softmax_bar_or<SW * 32>(failed || flags[0]);
        if (ok) {
            float *po = a.part_o + ((size_t)(b * a.n_split + split) * H) * DH;
            float *pml = a.part_ml + ((size_t)(b * a.n_split + split) * H) * 2;
            if (q4 < 2) {
#pragma unroll
                for (int j = 0; j < 8; ++j) po[(hb * 8 + j) * DH + dim] = o[j] + ob[(hb * 8 + j) * DH + dim];
            }
            if (q4 == 0 && lane < 8) {
                float m = 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    if (j == lane) m = mrun[j];
                const int h = hb * 8 + lane;
                const float l = (lp[h] + lp[H + h]) + (lp[2 * H + h] + lp[3 * H + h]);
                *reinterpret_cast<float2 *>(pml + 2 * h) = make_float2(m, l);
            }
            if (a.fused) {
                // the last CTA of this sequence merges every split into out[b]
                asm volatile("bar.sync 1, %0;" ::"n"(SW * 32));
                const int n_b = min(a.n_split, (L + a.tps - 1) / a.tps);   // splits holding tokens of b
                if (tid == 0) {
                    // acq_rel at gpu scope: releases the CTA's partial (ordered before this
                    // thread by the barrier above) and, for the last arrival, acquires the others'
                    int old;
                    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;"
                                 : "=r"(old)
                                 : "l"(a.counters + b)
                                 : "memory");
                    flags[1] = (old == n_b - 1) ? 1 : 0;
                }
                asm volatile("bar.sync 1, %0;" ::"n"(SW * 32));
                if (flags[1]) {
                    merge_split_partials<H, DH>(a.part_o, a.part_ml, a.n_split, n_b, b, a.out_scale, a.out, tid,
                                                SW * 32);
                    if (tid == 0) a.counters[b] = 0;                         // ready for the next call
                }
            }
        }
    }

    // every role is done with tensor memory (the issuer waited for its last MMA)
    __syncthreads();
    if (warp == ISSUER) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace

bool tc_decode_supported(const Dims &d) {
    return d.h1 == TcTpaH16D64R2::H && d.h2 == 1 && d.d1 == 1 && d.d2 == TcTpaH16D64R2::D2 &&
           d.rk == TcTpaH16D64R2::R && d.rv == TcTpaH16D64R2::R && !d.shared;
}

size_t tc_decode_smem() { return TcTpaH16D64R2::smem_bytes(); }

cudaError_t launch_decode_tc(const DecodeArgs &args, int batch, const DecodePlan &p, const RopeTable &rope,
                             const DecodeTestHooks &hooks, cudaStream_t st) {
    using C = TcTpaH16D64R2;
    if (args.cluster || args.qf || p.tile != C::TT) return cudaErrorInvalidValue;
    const size_t smem = C::smem_bytes();
    cudaError_t e = ensure_dynamic_smem<decode_tc_kernel<C>>(smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3((unsigned)p.n_split, (unsigned)batch);
    lc.blockDim = dim3(C::THREADS);
    lc.dynamicSmemBytes = smem;
    lc.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    return cudaLaunchKernelEx(&lc, decode_tc_kernel<C>, args, rope, hooks);
}

}  // namespace kpa
