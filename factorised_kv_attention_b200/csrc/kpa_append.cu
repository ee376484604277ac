// kpa_append.cu -- the append step: merged factor projection on the tcgen05 tensor
// cores, factor RoPE and the cache write in its epilogue, then the query assembly.
//
// "Kronecker Product Attention", eq 5 with the ranks merged: every output column of
// F = X W^T is one factor element of one token, the columns ordered
// [A^Q | B^Q | A^K | B^K | A^V | B^V] (rank-major inside each part).  The GEMM
// epilogue applies R_theta^(2)(pos) to the B^Q and B^K pairs (Theorem 2.4: the
// rotation of the reconstruction is the rotation of B alone), writes the key and
// value factors to their cache slots in bf16, and keeps the query factors in fp32
// for the assembly Q = (1/R_Q) sum_r A^Q_r (x) B~^Q_r (eq 2), done by a second kernel.
//
// GEMM: 128 x BN output tiles (BN <= 256, a multiple of 16), K in steps of 64.  Warp 0
// issues TMA loads of X and W tiles (128-byte swizzle) into a STAGES-deep ring; one
// thread of warp 1 issues tcgen05.mma (kind::f16, bf16 x bf16 -> fp32) into one of two
// TMEM accumulators and commits each stage back to the producer; warps 2..9 read the
// accumulator rows from TMEM (one row = one token per thread; two warps per TMEM lane
// quarter, each taking half of a tile's 32-column passes) and run the epilogue.
#include <cudaTypedefs.h>

#include <mutex>

#include "kpa_internal.cuh"
#include "kpa_sm100.cuh"

namespace kpa {

struct AppendArgs {
    int M, N, K;                 // tokens, projected factor columns, d_model
    int BN, n_kblocks, stages;
    int n_tok, cap;
    const int32_t *start_pos;
    int h1, h2, d1, d2, rq, rk, rv;
    int eq, ek, ev;              // elements per query / key / value record
    int d2m1;                    // d2 - 1 when d2 is a power of two (pair index by mask), else -1
    int shared;                  // one B for keys and values: columns [A^Q|B^Q|A^K|A^V|B], B unrotated
    __nv_bfloat16 *kc, *vc;
    float *qf;                   // [eq][M] query factors (B^Q rotated), or null
    int *err;
    unsigned long long wait_limit_ns;
};

namespace {

using namespace sm100;

constexpr int BM = 128, BK = 64;
constexpr int kThreads = 320;                 // producer, MMA, 8 epilogue warps (2 per TMEM lane quarter)
constexpr int kStageCols = 32;                // epilogue staging: columns per pass per column half
constexpr uint32_t kTmemCols = 512;              // two accumulators of 256 columns

__device__ __forceinline__ void store_cache(__nv_bfloat16 *plane, int b, int cap, int E, int s, int e,
                                            float v) {
    plane[(((int64_t)b * (cap / kGroup) + s / kGroup) * E + e) * kGroup + (s % kGroup)] =
        __float2bfloat16_rn(v);
}

// Rotate the projected pair (n, n+1) when it is a B^Q or B^K pair (cs(j) = (cos, sin)
// of pair j of the token's position); A factors and V pass unchanged.
// RoPE pair index j of projected column n (an even column): the pair (n, n+1) is pair j
// of a B^Q or B^K row, or -1 when the column is not rotated (A factors, values, and a
// B shared by keys and values, which the cache keeps unrotated).
__device__ __forceinline__ int rope_pair_of(const AppendArgs &a, int n) {
    const int qa = a.rq * a.h1 * a.d1, ka = a.rk * a.h1 * a.d1;
    int r = -1;                                    // offset inside a B row
    if (n < a.eq) {
        if (n >= qa) r = n - qa;
    } else if (!a.shared && n < a.eq + a.ek) {
        if (n - a.eq >= ka) r = n - a.eq - ka;
    }
    return r < 0 ? -1 : (a.d2m1 >= 0 ? (r & a.d2m1) : r % a.d2) >> 1;
}

template <class CS>
__device__ __forceinline__ void rotate_pair(const AppendArgs &a, int n, float &x0, float &x1, CS cs) {
    const int j = rope_pair_of(a, n);
    if (j >= 0) {
        const float2 w = cs(j);
        const float y0 = x0 * w.x - x1 * w.y, y1 = x0 * w.y + x1 * w.x;
        x0 = y0;
        x1 = y1;
    }
}

// Cache record of projected column n >= eq: true for the key record, with e its element.
// Columns [A^K | B^K | A^V | B^V]; with a shared B, [A^K | A^V | B] and B belongs to the
// key record after A^K.
__device__ __forceinline__ bool key_column(const AppendArgs &a, int n, int &e) {
    const int k = n - a.eq;
    if (!a.shared) {
        if (k < a.ek) { e = k; return true; }
        e = k - a.ek;
        return false;
    }
    const int ka = a.rk * a.h1 * a.d1;
    if (k < ka) { e = k; return true; }            // A^K
    if (k < 2 * ka) { e = k - ka; return false; }  // A^V
    e = k - ka;                                    // B, after A^K in the key record
    return true;
}

// One pair of projected columns (n, n+1) of token m: rotate it when it is a B^Q or B^K
// pair (cs(j) = (cos, sin) of pair j of the token's position), then keep query
// factors in fp32 and write key / value factors to the token's cache slot in bf16.
template <class CS>
__device__ __forceinline__ void emit_pair(const AppendArgs &a, int m, int b, int s, bool slot_ok, int n,
                                          float x0, float x1, CS cs) {
    rotate_pair(a, n, x0, x1, cs);
    if (n < a.eq) {                                        // query factors
        if (a.qf) {
            a.qf[(size_t)n * a.M + m] = x0;
            a.qf[(size_t)(n + 1) * a.M + m] = x1;
        }
    } else if (slot_ok) {                                  // key or value factors (a pair never
        int e;                                             // straddles two records: even columns)
        if (key_column(a, n, e)) {
            store_cache(a.kc, b, a.cap, a.ek, s, e, x0);
            store_cache(a.kc, b, a.cap, a.ek, s, e + 1, x1);
        } else {
            store_cache(a.vc, b, a.cap, a.ev, s, e, x0);
            store_cache(a.vc, b, a.cap, a.ev, s, e + 1, x1);
        }
    }
}

// Tile t of the persistent schedule -> (128-row block, first column, width).  The
// tiles every CTA gets the same number of come first; the remaining tiles are split
// into column halves of 128 and BN - 128 (both valid MMA widths), so that no CTA ends
// a whole tile after the others.
struct TileCols {
    int tm, n0, nw;
};
__device__ __forceinline__ TileCols tile_cols(int t, int n_tn, int BN, int n_even, bool split) {
    if (!split || t < n_even) return {t / n_tn, (t % n_tn) * BN, BN};
    const int u = t - n_even, f = n_even + (u >> 1), h = u & 1;
    return {f / n_tn, (f % n_tn) * BN + h * 128, h ? BN - 128 : 128};
}

__global__ void __launch_bounds__(kThreads, 1)
append_gemm_kernel(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmw,
                   AppendArgs a, RopeTable rope) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int S = a.stages, BN = a.BN;
    const uint32_t a_bytes = BM * BK * 2, b_bytes = (uint32_t)BN * BK * 2;
    unsigned char *a_st = smem;                                   // S x 16 KB
    unsigned char *b_st = a_st + (size_t)S * a_bytes;             // S x BN*128 B
    float *stg = reinterpret_cast<float *>(b_st + (size_t)S * b_bytes);   // [2 parts][kStageCols][BM]
    uint64_t *bars = reinterpret_cast<uint64_t *>(stg + 2 * kStageCols * BM);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * S + 5);
    volatile int *flags = reinterpret_cast<volatile int *>(tmem_slot + 1);    // abort, epilogue abort
    float2 *cs_all = reinterpret_cast<float2 *>(reinterpret_cast<unsigned char *>(bars) + 512);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t full0 = smem_u32(bars), empty0 = full0 + 8 * S, accf0 = full0 + 16 * S;
    const uint32_t acce0 = accf0 + 16, drain = acce0 + 16;
    const int n_tn = (a.N + BN - 1) / BN, whole = n_tn * ((a.M + BM - 1) / BM);
    const int n_even = (whole / (int)gridDim.x) * (int)gridDim.x;
    const bool split = BN > 128 && (BN - 128) % 16 == 0 && whole > n_even && 2 * (whole - n_even) <= (int)gridDim.x;
    const int n_tiles = split ? n_even + 2 * (whole - n_even) : whole;

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(accf0 + 8 * i, 1);
            mbar_init(acce0 + 8 * i, 8);                          // the 8 epilogue warps
        }
        mbar_init(drain, 1);
        flags[0] = flags[1] = 0;
        mbar_fence_init();
        tma_prefetch_desc(&tmx);
        tma_prefetch_desc(&tmw);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint64_t limit = a.wait_limit_ns;
    // bounded wait that gives up when the time runs out or another role has given up
    auto wait = [&](uint32_t b, uint32_t parity) -> bool {
        if (mbar_try_wait(b, parity)) return true;
        const uint64_t t0 = globaltimer();
        for (uint32_t it = 1;; ++it) {
            if (mbar_try_wait(b, parity)) return true;
            if ((it & 15) == 0) {
                if (flags[0]) return false;
                if (globaltimer() - t0 > limit) {
                    flags[0] = 1;
                    raise_error(a.err, kErrTimeout);
                    return false;
                }
            }
        }
    };

    if (warp == 0) {
        // ---- producer: TMA tiles of X and W for every k-block of every tile of this CTA;
        // the stage ring runs on across tile boundaries
        if (lane == 0) {
            int g = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
                const TileCols tc = tile_cols(tile, n_tn, BN, n_even, split);
                for (int kb = 0; kb < a.n_kblocks; ++kb, ++g) {
                    const int s = g % S;
                    if (g >= S && !wait(empty0 + 8 * s, ((g / S) - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(full0 + 8 * s, a_bytes + b_bytes);
                    tma_load_2d(smem_u32(a_st + (size_t)s * a_bytes), &tmx, kb * BK, tc.tm * BM, full0 + 8 * s);
                    tma_load_2d(smem_u32(b_st + (size_t)s * b_bytes), &tmw, kb * BK, tc.n0, full0 + 8 * s);
                }
            }
            // every copy issued lands before the CTA exits (normally already consumed)
            for (int k = max(0, g - S); k < g; ++k) (void)mbar_wait(full0 + 8 * (k % S), (k / S) & 1, limit);
        }
    } else if (warp == 1) {
        // ---- MMA issuer: accumulator i&1 of this CTA's i-th tile, once the epilogue has
        // drained it (tile i-2)
        if (lane == 0) {
            int g = 0, i = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++i) {
                const int buf = i & 1;
                const uint32_t idesc = umma_idesc_bf16_f32(BM, tile_cols(tile, n_tn, BN, n_even, split).nw);
                if (i >= 2 && !wait(acce0 + 8 * buf, ((i >> 1) - 1) & 1)) break;
                tc_fence_after();
                for (int kb = 0; kb < a.n_kblocks; ++kb, ++g) {
                    const int s = g % S;
                    if (!wait(full0 + 8 * s, (g / S) & 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = umma_desc_k_sw128(smem_u32(a_st + (size_t)s * a_bytes));
                    const uint64_t bd = umma_desc_k_sw128(smem_u32(b_st + (size_t)s * b_bytes));
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)     // K = 16 per instruction: 32 B along the row
                        umma_bf16(tmem + buf * 256, ad + 2 * k, bd + 2 * k, idesc, kb > 0 || k > 0);
                    umma_commit(empty0 + 8 * s);          // stage free once these MMAs finish
                }
                if (ok) umma_commit(accf0 + 8 * buf);
            }
            // nothing issued here may still run when tensor memory is released
            umma_commit(drain);
            (void)mbar_wait(drain, 0, limit);
        }
    } else {
        // ---- epilogue: thread = accumulator row = token; warps 2..5 take the first
        // half of each tile's 16-column chunks, warps 6..9 the rest
        const int quarter = warp & 3, part = (warp - 2) >> 2;
        const int row = quarter * 32 + lane;
        const int half = a.d2 / 2;
        float2 *cs = cs_all + (size_t)row * half;
        float *mystg = stg + part * kStageCols * BM;
        const int tp = (warp - 2) * 32 + lane - part * 128;           // 0..127 inside the part
        int i = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++i) {
            const TileCols tc = tile_cols(tile, n_tn, BN, n_even, split);
            const int tm = tc.tm, buf = i & 1;
            const int nch = tc.nw / 16, ch_lo = part ? (nch + 1) / 2 : 0, ch_hi = part ? nch : (nch + 1) / 2;
            const uint32_t acc = tmem + buf * 256 + ((uint32_t)(quarter * 32) << 16);
            asm volatile("bar.sync 2, 256;" ::: "memory");           // the previous tile is done with cs
            const int m = tm * BM + row;
            const bool live = m < a.M;
            int b = 0, s = 0;
            bool slot_ok = false;
            if (live) {
                b = m / a.n_tok;
                s = a.start_pos[b] + (m - b * a.n_tok);
                slot_ok = s >= 0 && s < a.cap;
                if (!slot_ok && part == 0) raise_error(a.err, kErrDeviceCheck);
                for (int j = part; j < half; j += 2) {             // the row's two threads split the angles
                    float c, sn;
                    rope_cs((double)s, rope.theta[j], c, sn);
                    cs[j] = make_float2(c, sn);
                }
            }
            // all 8 warps agree on whether the accumulator arrived before going on
            const bool got = __all_sync(0xffffffffu, wait(accf0 + 8 * buf, (i >> 1) & 1));
            if (!got && lane == 0) flags[1] = 1;
            asm volatile("bar.sync 2, 256;" ::: "memory");           // angles in, verdicts in
            if (flags[1]) break;
            tc_fence_after();
            // Fast path: the tile's 128 rows are consecutive slots of one sequence starting
            // on a cache group.  Rotated values are staged transposed, 32 columns at a time,
            // and leave as 16-byte pieces: float4 runs of query-factor columns, whole 8-token
            // cache groups.
            const int m0 = tm * BM;
            const int b0 = m0 / a.n_tok;
            const int s0 = a.start_pos[b0] + (m0 - b0 * a.n_tok);
            const bool fast = m0 + BM <= a.M && (m0 + BM - 1) / a.n_tok == b0 && s0 >= 0 && s0 % kGroup == 0 &&
                              s0 + BM <= a.cap && a.M % 4 == 0;
            if (fast) {
                for (int c0 = ch_lo; c0 < ch_hi; c0 += kStageCols / 16) {
                    const int cn = min(kStageCols / 16, ch_hi - c0);   // 16-column chunks in this pass
                    for (int cc = 0; cc < cn; ++cc) {
                        float v[16];
                        tmem_ld16(acc + (c0 + cc) * 16, v);             // warp-collective
                        const int n0 = tc.n0 + (c0 + cc) * 16;
#pragma unroll
                        for (int j = 0; j < 16; j += 2) {
                            if (n0 + j >= a.N) break;
                            float x0 = v[j], x1 = v[j + 1];
                            rotate_pair(a, n0 + j, x0, x1, [&](int k) { return cs[k]; });
                            mystg[(cc * 16 + j) * BM + row] = x0;
                            mystg[(cc * 16 + j + 1) * BM + row] = x1;
                        }
                    }
                    if (c0 + cn >= ch_hi) {                             // last read of the accumulator
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(acce0 + 8 * buf);
                    }
                    asm volatile("bar.sync %0, 128;" ::"r"(3 + part) : "memory");   // the part's chunk is staged
                    const int nb = tc.n0 + c0 * 16, ne = min(nb + cn * 16, a.N);
                    const int qe = min(ne, a.eq);
                    if (a.qf)
                        for (int it = tp; it < max(0, qe - nb) * (BM / 4); it += 128) {
                            const int lc = it / (BM / 4), i4 = it % (BM / 4);
                            const float4 x = reinterpret_cast<const float4 *>(mystg + (size_t)lc * BM)[i4];
                            *reinterpret_cast<float4 *>(a.qf + (size_t)(nb + lc) * a.M + m0 + 4 * i4) = x;
                        }
                    const int kb0 = max(nb, a.eq);
                    for (int it = tp; it < max(0, ne - kb0) * (BM / kGroup); it += 128) {
                        const int lc = kb0 - nb + it / (BM / kGroup), gq = it % (BM / kGroup);
                        const int n = nb + lc;
                        int e;
                        const bool is_k = key_column(a, n, e);
                        __nv_bfloat16 *plane = is_k ? a.kc : a.vc;
                        const int E = is_k ? a.ek : a.ev;
                        const float4 lo = reinterpret_cast<const float4 *>(mystg + (size_t)lc * BM + gq * kGroup)[0];
                        const float4 hi = reinterpret_cast<const float4 *>(mystg + (size_t)lc * BM + gq * kGroup)[1];
                        uint4 u;
                        __nv_bfloat162 *pu = reinterpret_cast<__nv_bfloat162 *>(&u);
                        pu[0] = __floats2bfloat162_rn(lo.x, lo.y);
                        pu[1] = __floats2bfloat162_rn(lo.z, lo.w);
                        pu[2] = __floats2bfloat162_rn(hi.x, hi.y);
                        pu[3] = __floats2bfloat162_rn(hi.z, hi.w);
                        *reinterpret_cast<uint4 *>(
                            plane + (((int64_t)b0 * (a.cap / kGroup) + s0 / kGroup + gq) * E + e) * kGroup) = u;
                    }
                    asm volatile("bar.sync %0, 128;" ::"r"(3 + part) : "memory");   // staging free again
                }
            } else {
                for (int ch = ch_lo; ch < ch_hi; ++ch) {
                    float v[16];
                    tmem_ld16(acc + ch * 16, v);                        // warp-collective
                    if (!live) continue;
                    const int n0 = tc.n0 + ch * 16;
#pragma unroll
                    for (int j = 0; j < 16; j += 2) {
                        if (n0 + j >= a.N) break;
                        emit_pair(a, m, b, s, slot_ok, n0 + j, v[j], v[j + 1], [&](int k) { return cs[k]; });
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acce0 + 8 * buf);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// The projection for a handful of tokens (a decode step): a matrix-vector product
// that streams W once.  One CTA per pair of W rows (n, n+1), so a rotated pair is
// formed in one place; its 8 warps split K, each lane holding 8 consecutive k of
// both rows and of every token (X stays in L2), then the partial sums are reduced
// with shuffles and through shared memory.  Thread m runs the epilogue of token m.
constexpr int kSmallMaxM = 16, kSmallWarps = 8;   // up to 16 tokens; MAXM = 8 or 16 below

template <int MAXM>
__global__ void __launch_bounds__(kSmallWarps * 32, MAXM == 8 ? 3 : 2)
append_small_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ w, AppendArgs a,
                    RopeTable rope) {
    __shared__ float red[kSmallWarps][2][MAXM];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = 2 * blockIdx.x;
    // the epilogue's own inputs (the token's start slot, the pair's RoPE frequency) are
    // requested now, with the operand loads, instead of after the reduction
    const int jn = rope_pair_of(a, n);
    const int sp = tid < a.M ? a.start_pos[tid / a.n_tok] : 0;
    const double th = tid < a.M && jn >= 0 ? rope.theta[jn] : 0.0;
    float acc0[MAXM], acc1[MAXM];
#pragma unroll
    for (int m = 0; m < MAXM; ++m) acc0[m] = acc1[m] = 0.f;
    const int k8n = a.K / 8;
    const uint4 *w0 = reinterpret_cast<const uint4 *>(w + (size_t)n * a.K);
    const uint4 *w1 = reinterpret_cast<const uint4 *>(w + (size_t)(n + 1) * a.K);
    const uint4 *xv = reinterpret_cast<const uint4 *>(x);
    for (int k8 = tid; k8 < k8n; k8 += kSmallWarps * 32) {
        const uint4 ua = __ldg(w0 + k8), ub = __ldg(w1 + k8);
        const __nv_bfloat162 *pa = reinterpret_cast<const __nv_bfloat162 *>(&ua);
        const __nv_bfloat162 *pb = reinterpret_cast<const __nv_bfloat162 *>(&ub);
        float fa[8], fb[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 ta = __bfloat1622float2(pa[i]), tb = __bfloat1622float2(pb[i]);
            fa[2 * i] = ta.x;
            fa[2 * i + 1] = ta.y;
            fb[2 * i] = tb.x;
            fb[2 * i + 1] = tb.y;
        }
        // every token's x chunk is requested before the first is used (one round trip)
        uint4 ux[MAXM];
#pragma unroll
        for (int m = 0; m < MAXM; ++m)
            ux[m] = m < a.M ? __ldg(xv + (size_t)m * k8n + k8) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int m = 0; m < MAXM; ++m) {
            if (m >= a.M) break;
            const __nv_bfloat162 *px = reinterpret_cast<const __nv_bfloat162 *>(&ux[m]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 tx = __bfloat1622float2(px[i]);
                acc0[m] = fmaf(fa[2 * i], tx.x, fmaf(fa[2 * i + 1], tx.y, acc0[m]));
                acc1[m] = fmaf(fb[2 * i], tx.x, fmaf(fb[2 * i + 1], tx.y, acc1[m]));
            }
        }
    }
#pragma unroll
    for (int m = 0; m < MAXM; ++m) {
        if (m >= a.M) break;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            acc0[m] += __shfl_xor_sync(0xffffffffu, acc0[m], off);
            acc1[m] += __shfl_xor_sync(0xffffffffu, acc1[m], off);
        }
        if (lane == 0) {
            red[warp][0][m] = acc0[m];
            red[warp][1][m] = acc1[m];
        }
    }
    __syncthreads();
    if (tid >= a.M) return;
    const int m = tid;
    float x0 = 0.f, x1 = 0.f;
#pragma unroll
    for (int i = 0; i < kSmallWarps; ++i) {
        x0 += red[i][0][m];
        x1 += red[i][1][m];
    }
    const int b = m / a.n_tok, s = sp + (m - b * a.n_tok);
    const bool slot_ok = s >= 0 && s < a.cap;
    if (!slot_ok && n == 0) raise_error(a.err, kErrDeviceCheck);
    emit_pair(a, m, b, s, slot_ok, n, x0, x1, [&](int) {     // the pair is jn
        float c, sn;
        rope_cs((double)s, th, c, sn);
        return make_float2(c, sn);
    });
}

// Query assembly for a handful of tokens: one thread per 16-byte chunk of q_out,
// (token, head, j1, 8 features of j2).
__global__ void __launch_bounds__(128)
q_assemble_small_kernel(const float *__restrict__ qf, int M, int h1, int h2, int d1, int d2, int rq,
                        __nv_bfloat16 *__restrict__ q_out) {
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    const int per_head = d1 * (d2 / 8), h = h1 * h2;
    if (idx >= M * h * per_head) return;
    const int m = idx / (h * per_head), rem = idx % (h * per_head);
    const int head = rem / per_head, j1 = (rem % per_head) / (d2 / 8), j2 = (rem % (d2 / 8)) * 8;
    const int i1 = head / h2, i2 = head % h2, qa = rq * h1 * d1;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    // ranks in groups of 4 with every load of a group issued before its arithmetic
    for (int r0 = 0; r0 < rq; r0 += 4) {
        float av[4], bv[4][8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int r = r0 + k < rq ? r0 + k : rq - 1;
            av[k] = r0 + k < rq ? __ldg(qf + (size_t)((r * h1 + i1) * d1 + j1) * M + m) : 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u) bv[k][u] = __ldg(qf + (size_t)(qa + (r * h2 + i2) * d2 + j2 + u) * M + m);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k)
#pragma unroll
            for (int u = 0; u < 8; ++u) acc[u] += av[k] * bv[k][u];
    }
    const float inv = 1.0f / (float)rq;
    uint4 o;
    uint32_t *po = reinterpret_cast<uint32_t *>(&o);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        __nv_bfloat162 hb = __floats2bfloat162_rn(acc[2 * k] * inv, acc[2 * k + 1] * inv);
        po[k] = *reinterpret_cast<uint32_t *>(&hb);
    }
    *reinterpret_cast<uint4 *>(q_out + ((size_t)m * h + head) * d1 * d2 + j1 * d2 + j2) = o;
}

// Query assembly q = (1/R_Q) sum_r A^Q_r (x) B^Q_r for the queries of the chunk.
// A CTA takes kQaTokens consecutive tokens.  Their factor columns are first staged in
// shared memory as token rows [t][e]; the loads run along the token axis of the
// [column][token] buffer, so they are coalesced.  Then each thread takes one
// (token, head, 8-feature slice of d2), keeps B^Q_r[i2, slice] (R_Q x 8) in registers,
// and walks j1, writing one 16-byte piece per j1.  A warp's 32 pieces at one j1 fill
// whole 32-byte sectors of 16 head rows of q_out.
constexpr int kQaTokens = 16;
constexpr int kQaThreads = 256;
constexpr int kQaBatch = 16;

__host__ __device__ inline int qa_ld(int eq) { return (eq + 3) / 4 * 4 + 4; }   // shared-memory row stride (floats)

template <int RQ>
__global__ void __launch_bounds__(kQaThreads)
q_assemble_kernel(const float *__restrict__ qf, int M, int h1, int h2, int d1, int d2,
                  __nv_bfloat16 *__restrict__ q_out) {
    extern __shared__ float4 qa_smem[];
    float *s = reinterpret_cast<float *>(qa_smem);
    const int qa = RQ * h1 * d1, eq = qa + RQ * h2 * d2, ld = qa_ld(eq);
    const int m0 = blockIdx.x * kQaTokens;
    const int nt = min(kQaTokens, M - m0);
    // Staging: every load of a batch is issued before the first shared-memory store,
    // so a thread has up to kQaBatch loads in flight instead of one.
    if ((M & 3) == 0) {
        // four tokens per 16-byte load (the column starts e*M + m0 are 16-byte aligned)
        const int total = eq * (kQaTokens / 4);
        for (int base = 0; base < total; base += kQaBatch * kQaThreads) {
            float4 v[kQaBatch];
#pragma unroll
            for (int k = 0; k < kQaBatch; ++k) {
                const int idx = base + k * kQaThreads + threadIdx.x;
                const int e = idx / (kQaTokens / 4), t = (idx % (kQaTokens / 4)) * 4;
                v[k] = idx < total && t < nt
                           ? __ldg(reinterpret_cast<const float4 *>(qf + (size_t)e * M + m0 + t))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int k = 0; k < kQaBatch; ++k) {
                const int idx = base + k * kQaThreads + threadIdx.x;
                const int e = idx / (kQaTokens / 4), t = (idx % (kQaTokens / 4)) * 4;
                if (idx < total) {
                    s[t * ld + e] = v[k].x;
                    s[(t + 1) * ld + e] = v[k].y;
                    s[(t + 2) * ld + e] = v[k].z;
                    s[(t + 3) * ld + e] = v[k].w;
                }
            }
        }
    } else {
        const int total = eq * kQaTokens;
        for (int base = 0; base < total; base += kQaBatch * kQaThreads) {
            float v[kQaBatch];
#pragma unroll
            for (int k = 0; k < kQaBatch; ++k) {
                const int idx = base + k * kQaThreads + threadIdx.x;
                const int e = idx / kQaTokens, t = idx % kQaTokens;
                v[k] = idx < total && t < nt ? __ldg(qf + (size_t)e * M + m0 + t) : 0.f;
            }
#pragma unroll
            for (int k = 0; k < kQaBatch; ++k) {
                const int idx = base + k * kQaThreads + threadIdx.x;
                const int e = idx / kQaTokens, t = idx % kQaTokens;
                if (idx < total) s[t * ld + e] = v[k];
            }
        }
    }
    __syncthreads();
    const int h = h1 * h2, c8 = d2 / 8, per_tok = h * c8;
    const float inv = 1.0f / (float)RQ;
    for (int task = threadIdx.x; task < nt * per_tok; task += kQaThreads) {
        const int t = task / per_tok, p = task - t * per_tok;
        const int head = p / c8, c = p - head * c8;
        const int i1 = head / h2, i2 = head - i1 * h2;
        const float *st = s + t * ld;
        float B[RQ][8];
#pragma unroll
        for (int r = 0; r < RQ; ++r) {
            const float4 *b4 = reinterpret_cast<const float4 *>(st + qa + (r * h2 + i2) * d2 + c * 8);
            const float4 x = b4[0], y = b4[1];
            B[r][0] = x.x; B[r][1] = x.y; B[r][2] = x.z; B[r][3] = x.w;
            B[r][4] = y.x; B[r][5] = y.y; B[r][6] = y.z; B[r][7] = y.w;
        }
        __nv_bfloat16 *dst = q_out + ((size_t)(m0 + t) * h + head) * d1 * d2 + c * 8;
        for (int j1 = 0; j1 < d1; ++j1) {
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int r = 0; r < RQ; ++r) {
                const float a = st[(r * h1 + i1) * d1 + j1];
#pragma unroll
                for (int u = 0; u < 8; ++u) acc[u] += a * B[r][u];
            }
            uint4 o;
            uint32_t *po = reinterpret_cast<uint32_t *>(&o);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                __nv_bfloat162 hb = __floats2bfloat162_rn(acc[2 * k] * inv, acc[2 * k + 1] * inv);
                po[k] = *reinterpret_cast<uint32_t *>(&hb);
            }
            *reinterpret_cast<uint4 *>(dst + j1 * d2) = o;
        }
    }
}

template <int RQ>
cudaError_t launch_q_assemble(const float *qf, int M, const Dims &d, __nv_bfloat16 *qo, cudaStream_t st) {
    const int eq = RQ * (d.h1 * d.d1 + d.h2 * d.d2);
    const size_t smem = (size_t)kQaTokens * qa_ld(eq) * sizeof(float);
    const cudaError_t e = ensure_dynamic_smem<q_assemble_kernel<RQ>>(smem);
    if (e != cudaSuccess) return e;
    q_assemble_kernel<RQ><<<(unsigned)((M + kQaTokens - 1) / kQaTokens), kQaThreads, smem, st>>>(
        qf, M, d.h1, d.h2, d.d1, d.d2, qo);
    return cudaGetLastError();
}

// Any shape: one thread per (token, head), loops.
__global__ void __launch_bounds__(128)
q_assemble_any_kernel(const float *__restrict__ qf, int M, int h1, int h2, int d1, int d2, int rq,
                      __nv_bfloat16 *__restrict__ q_out) {
    const int m = blockIdx.x * blockDim.x + threadIdx.x;
    if (m >= M) return;
    const int head = blockIdx.y, i1 = head / h2, i2 = head % h2, qa = rq * h1 * d1;
    const float inv = 1.0f / (float)rq;
    __nv_bfloat16 *dst = q_out + ((size_t)m * h1 * h2 + head) * d1 * d2;
    for (int j1 = 0; j1 < d1; ++j1)
        for (int j2 = 0; j2 < d2; ++j2) {
            float acc = 0.f;
            for (int r = 0; r < rq; ++r)
                acc += qf[(size_t)(r * h1 * d1 + i1 * d1 + j1) * M + m] *
                       qf[(size_t)(qa + r * h2 * d2 + i2 * d2 + j2) * M + m];
            dst[j1 * d2 + j2] = __float2bfloat16_rn(acc * inv);
        }
}

// cuTensorMapEncodeTiled from the driver, found through the runtime (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D bf16 tensor [rows][cols] (cols contiguous), boxes of 64 columns x box_rows rows,
// 128-byte swizzle; elements outside the tensor read as zero.
bool make_map(CUtensorMap *map, const void *ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t append_smem_bytes(int BN, int stages, int d2) {
    return 1024 + (size_t)stages * (BM * BK * 2 + (size_t)BN * BK * 2) + (size_t)2 * kStageCols * BM * 4 + 512 +
           (size_t)BM * (d2 / 2) * 8;
}

int append_tile_n(int N) {
    const int tiles = (N + 255) / 256;
    const int per = (N + tiles - 1) / tiles;
    return ((per + 15) / 16) * 16;
}

cudaError_t launch_append(const Dims &d, int rq, int d_model, int batch, int n_tok, const void *x,
                          const void *w, const int32_t *start_pos, int cap, void *kc, void *vc,
                          void *q_out, float *qf, const RopeTable &rope, int *err,
                          unsigned long long wait_limit_ns, cudaStream_t st) {
    AppendArgs a;
    a.M = batch * n_tok;
    a.eq = rq * (d.h1 * d.d1 + d.h2 * d.d2);
    a.ek = d.ek;
    a.ev = d.ev;
    a.shared = d.shared;
    a.N = a.eq + a.ek + a.ev;
    a.d2m1 = (d.d2 & (d.d2 - 1)) == 0 ? d.d2 - 1 : -1;
    a.K = d_model;
    a.BN = append_tile_n(a.N);
    a.n_kblocks = (d_model + BK - 1) / BK;
    a.stages = 4;
    while (a.stages > 2 && append_smem_bytes(a.BN, a.stages, d.d2) > 227 * 1024) --a.stages;
    if (append_smem_bytes(a.BN, a.stages, d.d2) > 227 * 1024) return cudaErrorInvalidValue;
    a.n_tok = n_tok;
    a.cap = cap;
    a.start_pos = start_pos;
    a.h1 = d.h1; a.h2 = d.h2; a.d1 = d.d1; a.d2 = d.d2;
    a.rq = rq; a.rk = d.rk; a.rv = d.rv;
    a.kc = static_cast<__nv_bfloat16 *>(kc);
    a.vc = static_cast<__nv_bfloat16 *>(vc);
    a.qf = qf;                           // the query factors land in the workspace when there is one
    a.err = err;
    a.wait_limit_ns = wait_limit_ns;

    cudaError_t e;
    const bool small = a.M <= kSmallMaxM;
    if (small) {
        // a decode step: stream W once with a matrix-vector kernel
        if (a.M <= 8)
            append_small_kernel<8><<<(unsigned)(a.N / 2), kSmallWarps * 32, 0, st>>>(
                static_cast<const __nv_bfloat16 *>(x), static_cast<const __nv_bfloat16 *>(w), a, rope);
        else
            append_small_kernel<16><<<(unsigned)(a.N / 2), kSmallWarps * 32, 0, st>>>(
                static_cast<const __nv_bfloat16 *>(x), static_cast<const __nv_bfloat16 *>(w), a, rope);
    } else {
    CUtensorMap tmx, tmw;
    if (!make_map(&tmx, x, (uint64_t)a.M, (uint64_t)d_model, BM)) return cudaErrorInvalidValue;
    if (!make_map(&tmw, w, (uint64_t)a.N, (uint64_t)d_model, (uint32_t)a.BN)) return cudaErrorInvalidValue;
    const size_t smem = append_smem_bytes(a.BN, a.stages, d.d2);
    e = ensure_dynamic_smem<append_gemm_kernel>(smem);
    if (e != cudaSuccess) return e;
    // persistent: one CTA per SM (or per tile when there are fewer tiles)
    int sms = 148;
    {
        int dev = 0;
        if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    }
    const int tiles = ((a.N + a.BN - 1) / a.BN) * ((a.M + BM - 1) / BM);
    append_gemm_kernel<<<(unsigned)(tiles < sms ? tiles : sms), kThreads, smem, st>>>(tmx, tmw, a, rope);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess || !q_out) return e;
    __nv_bfloat16 *qo = static_cast<__nv_bfloat16 *>(q_out);
    // the staged kernel reads B^Q slices as float4 from shared memory: d2 % 8 == 0 and
    // the B^Q block starting on a 16-byte boundary (R_Q * h1 * d1 % 4 == 0)
    const bool staged = d.d2 % 8 == 0 && (rq * d.h1 * d.d1) % 4 == 0 &&
                        (size_t)kQaTokens * qa_ld(rq * (d.h1 * d.d1 + d.h2 * d.d2)) * 4 <= 96 * 1024;
    if (small && d.d2 % 8 == 0) {
        const int threads = a.M * d.h * d.d1 * (d.d2 / 8);
        q_assemble_small_kernel<<<(unsigned)((threads + 127) / 128), 128, 0, st>>>(qf, a.M, d.h1, d.h2, d.d1,
                                                                                  d.d2, rq, qo);
    } else if (staged && rq == 1) {
        return launch_q_assemble<1>(qf, a.M, d, qo, st);
    } else if (staged && rq == 2) {
        return launch_q_assemble<2>(qf, a.M, d, qo, st);
    } else if (staged && rq == 4) {
        return launch_q_assemble<4>(qf, a.M, d, qo, st);
    } else if (staged && rq == 6) {
        return launch_q_assemble<6>(qf, a.M, d, qo, st);
    } else if (staged && rq == 8) {
        return launch_q_assemble<8>(qf, a.M, d, qo, st);
    } else {
        dim3 g3((unsigned)((a.M + 127) / 128), (unsigned)d.h);
        q_assemble_any_kernel<<<g3, 128, 0, st>>>(qf, a.M, d.h1, d.h2, d.d1, d.d2, rq, qo);
    }
    return cudaGetLastError();
}

}  // namespace kpa
