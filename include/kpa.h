/*
 * kpa.h -- C ABI of libkpa: factor-space Kronecker Product Attention (KPA)
 * and its degenerate split, Tensor Product Attention (TPA), on NVIDIA B200
 * (sm_100a).
 *
 * Each cached key and value of token t is stored only as factors,
 *     K_t = (1/R_K) sum_r A^K_r(t) (x) B^K_r(t),   A_r in R^{h1 x d1},
 *     V_t = (1/R_V) sum_r A^V_r(t) (x) B^V_r(t),   B_r in R^{h2 x d2},
 * with h = h1*h2 heads and d_h = d1*d2 features per head ("Kronecker Product
 * Attention", section 2.2, eqs 2-4).  Setting h1 = h, d1 = 1, h2 = 1, d2 = d_h
 * gives TPA (same section, final paragraph).  RoPE is the Kronecker-separable
 * operator I_{d1} (x) R_theta^(2)(t) (Definition 2.3); by Theorem 2.4 it rotates
 * only the B factors, so the cache holds B^K already rotated and A^K, A^V, B^V
 * as projected (section 2.5).  Attention reads the factors directly: the cache
 * is never expanded to full K/V in device memory.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Notation.  Head (i1, i2) is flat head i1*h2 + i2 and feature (j1, j2) is
 *    flat feature j1*d2 + j2 (the block order of Definition 2.1).
 *  - Factor record.  One token's key record holds E_K = R_K*(h1*d1 + h2*d2)
 *    elements in the order [A_0 .. A_{R_K-1} | B_0 .. B_{R_K-1}], each A_r
 *    row-major h1 x d1, each B_r row-major h2 x d2; the value record likewise
 *    with R_V (E_V elements).
 *  - RoPE.  Pairs (2m, 2m+1) of each length-d2 row of B, angle
 *    phi = pos * rope_base^(-2m/d2), (x0, x1) -> (x0 cos phi - x1 sin phi,
 *    x0 sin phi + x1 cos phi).  The angle is formed in float64.
 *  - Cache layout (the planes `kcache`, `vcache`).  Slot s of sequence b holds
 *    the token at position s.  Slots are grouped by KPA_TOKEN_GROUP (8): group
 *    g = s / 8 stores its 8 records element-major, token-minor, so element e of
 *    slot s lives at element offset
 *        ((b * (capacity / 8) + s / 8) * E + e) * 8 + s % 8
 *    (E = E_K or E_V).  `capacity` must be a positive multiple of 8.  A plane
 *    is batch * capacity * E elements of the config dtype.
 *  - Memory.  Every pointer is device memory unless stated otherwise, owned by
 *    the caller, and 16-byte aligned.  The library never allocates or frees
 *    device memory and never synchronises, except kpa_read_device_error.
 *  - Streams.  `stream` is a cudaStream_t (NULL = the legacy default stream);
 *    all work is enqueued on it and the call returns without waiting.
 *  - Errors.  Bad arguments return KPA_ERR_INVALID_ARG before anything is
 *    enqueued; shapes the kernels do not cover return KPA_ERR_UNSUPPORTED; a
 *    failed launch returns KPA_ERR_CUDA (kpa_last_cuda_error gives the CUDA
 *    code).  Problems only the device can see (a slot outside the cache, a
 *    length above max_len, a bounded wait that ran out) set a per-device error
 *    word that kpa_read_device_error returns; the offending work is skipped,
 *    never performed out of bounds.
 */
#ifndef KPA_H
#define KPA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KPA_TOKEN_GROUP 8

typedef struct CUstream_st *kpa_stream; /* the same type as cudaStream_t */

typedef enum {
    KPA_OK = 0,
    KPA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, inconsistent size   */
    KPA_ERR_UNSUPPORTED = 2,  /* valid request that no kernel here covers      */
    KPA_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required    */
    KPA_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed          */
    KPA_ERR_TIMEOUT = 5,      /* device: a bounded wait ran out                */
    KPA_ERR_DEVICE_CHECK = 6  /* device: an index or length failed its check   */
} kpa_status;

typedef enum { KPA_F32 = 0, KPA_BF16 = 1 } kpa_dtype;

typedef struct {
    int32_t h1, h2;     /* heads h = h1*h2                                      */
    int32_t d1, d2;     /* features per head d_h = d1*d2; d2 even (RoPE pairs)  */
    int32_t r_q;        /* query rank (kpa_append only; 0 elsewhere)            */
    int32_t r_k, r_v;   /* key and value ranks                                  */
    int32_t d_model;    /* hidden size (kpa_append only; 0 elsewhere)           */
    double rope_base;   /* RoPE base, e.g. 10000                                */
    kpa_dtype dtype;    /* element type of caches, factors, queries, x and W    */
    int32_t shared_b;   /* 0: separate B^K and B^V.  1: one B shared by keys and
                         * values ("Tensor Product Attention Is All You Need",
                         * section 5, "TPA KV with Shared B"; B^K_r = B^V_r, so
                         * r_k == r_v).  The key record is then [A^K | B] with B
                         * stored UNROTATED (values must not see the rotation);
                         * the value record is [A^V] only (E_V = r_v h1 d1), and
                         * kpa_decode rotates B for the score at each cached
                         * token's position.  Taken by kpa_cache_bytes_per_token,
                         * kpa_append_factors, kpa_append (merged weight columns
                         * [A^Q | B^Q | A^K | A^V | B]), the decode calls and
                         * kpa_prefill (which rotates B while rebuilding K).     */
    int32_t order;      /* 0 or 2: the Kronecker form above.  3: third-order TPA
                         * ("Tensor Product Attention Is All You Need", Appendix C):
                         * the key of head h is (1/R_K) sum_r a_r[h] (b_r (x) c_r)
                         * with a_r in R^h1, b_r in R^d1, c_r in R^d2 (d_h = d1 d2,
                         * b's index the slower one); h2 must be 1, d1 even, and
                         * shared_b 0.  A record is [a_0..a_{R-1} | b_0..b_{R-1} |
                         * c_0..c_{R-1}] (E = R (h1 + d1 + d2)); RoPE acts on the b
                         * factors only, R_{d1}(pos) (x) I_{d2} with theta_m =
                         * base^(-2m/d1), so kpa_append_factors rotates the keys' b
                         * and kpa_decode rotates the query by the same block
                         * matrix.  Taken by kpa_cache_bytes_per_token,
                         * kpa_append_factors, kpa_decode_workspace_size,
                         * kpa_decode_plan, kpa_decode_kernel_kind, kpa_decode,
                         * kpa_decode_split and kpa_decode_noalloc (d1, d2 <= 16,
                         * h1 <= 32); the projection, the prefill and the
                         * query-factor decode return KPA_ERR_UNSUPPORTED.       */
} kpa_config;

/* Human-readable name of a status code (static storage). */
const char *kpa_status_string(kpa_status status);

/* CUDA error code (cudaError_t as int) behind the calling thread's most recent
 * KPA_ERR_CUDA, or 0. */
int kpa_last_cuda_error(void);

/* Bytes one token adds to the key plane and to the value plane:
 * E_K * sizeof(dtype) and E_V * sizeof(dtype), i.e. eq 10's
 * (R_K + R_V)(h1 d1 + h2 d2) numbers split by plane ("Kronecker Product
 * Attention", section 2.5; Appendix B, eq 11).  Either output may be NULL.
 * Host only; enqueues nothing. */
kpa_status kpa_cache_bytes_per_token(const kpa_config *cfg, size_t *k_bytes, size_t *v_bytes);

/* Write given factor records into the cache (section 2.5; Theorem 2.4).
 *   k_factors [batch][n_tok][E_K]  unrotated key records, config dtype
 *   v_factors [batch][n_tok][E_V]  value records, config dtype
 *   start_pos [batch] int32        token t of sequence b goes to slot
 *                                  start_pos[b] + t, at that position
 * B^K is rotated at its position; A^K, A^V, B^V are stored unchanged.  A token
 * whose slot falls outside [0, capacity) is not written and sets
 * KPA_ERR_DEVICE_CHECK.  n_tok == 0 or batch == 0 enqueues nothing. */
kpa_status kpa_append_factors(const kpa_config *cfg, int32_t batch, int32_t n_tok,
                              const void *k_factors, const void *v_factors,
                              const int32_t *start_pos, int32_t capacity,
                              void *kcache, void *vcache, kpa_stream stream);

/* Workspace kpa_decode needs for `batch` sequences of at most `max_len` slots.
 * tokens_per_split = 0 lets the library choose the split of each sequence;
 * otherwise it must be a positive multiple of 64.  Host only. */
kpa_status kpa_decode_workspace_size(const kpa_config *cfg, int32_t batch, int32_t max_len,
                                     int32_t tokens_per_split, size_t *bytes);

/* How kpa_decode will split the work for these sizes (host only): the splits
 * per sequence, the tokens in each split (the last split of a sequence runs to
 * its end: a remainder of at most a quarter of a split is not a split of its
 * own, so the last may hold up to 5/4 of one), and the kernel launches one call
 * enqueues (1 when the splits of a sequence are merged inside the decode
 * kernel, 2 when a separate combine kernel follows).  Any output pointer may be
 * NULL.  Same argument rules as kpa_decode_workspace_size. */
kpa_status kpa_decode_plan(const kpa_config *cfg, int32_t batch, int32_t max_len,
                           int32_t tokens_per_split, int32_t *n_split,
                           int32_t *tokens_per_split_out, int32_t *launches);

/* Which kernel a dense-query kpa_decode_split call with these arguments runs
 * (kpa_decode_qf takes the mma.sync kernel, or the factored score after
 * kpa_test_set_decode_engine(2)):
 *   KPA_DECODE_KERNEL_CUDA_CORES  fp32 caches or shapes without a tensor-core variant
 *   KPA_DECODE_KERNEL_MMA_SYNC    the bf16 tensor-core kernel on mma.sync
 *   KPA_DECODE_KERNEL_TCGEN05     TPA h = 16, d_h = 64, R_K = R_V = 2 after
 *                                 kpa_test_set_decode_engine(1): both products on
 *                                 tcgen05
 * Same argument checks as kpa_decode_plan. */
enum { KPA_DECODE_KERNEL_CUDA_CORES = 0, KPA_DECODE_KERNEL_MMA_SYNC = 1, KPA_DECODE_KERNEL_TCGEN05 = 2 };
kpa_status kpa_decode_kernel_kind(const kpa_config *cfg, int32_t batch, int32_t max_len,
                                  int32_t tokens_per_split, int32_t *kind);

/* Factor-space decode attention: one query row per sequence against slots
 * 0 .. seq_len[b]-1 of the cache (Proposition 2.2 evaluated with a dense
 * query, Theorem 2.4 for the positions; FlashTPA-style blocking over the cache
 * with an online log-sum-exp, split across CTAs and merged by a combine pass).
 *   q        [batch][h][d_h]  config dtype; rotated here by
 *                             I_{d1} (x) R^(2)(q_pos[b]) when q_pos != NULL,
 *                             used as given when q_pos == NULL
 *   seq_len  [batch] int32    0 <= seq_len[b] <= max_len <= capacity; a longer
 *                             length is clamped to max_len and sets
 *                             KPA_ERR_DEVICE_CHECK
 *   sm_scale softmax scale applied to q.k (usually 1/sqrt(d_h))
 *   out      [batch][h][d_h] float32; a sequence with seq_len 0 gets zeros
 *   workspace at least kpa_decode_workspace_size(cfg, batch, max_len, 0) bytes,
 *            256-byte aligned, zero-filled before its first use (cudaMemsetAsync);
 *            every call that completes without a device error leaves it ready for
 *            the next one (after an error, zero it again)
 * Results are deterministic for a given (batch, max_len). */
kpa_status kpa_decode(const kpa_config *cfg, int32_t batch, const void *q, const int32_t *q_pos,
                      const void *kcache, const void *vcache, int32_t capacity,
                      const int32_t *seq_len, int32_t max_len, float sm_scale, float *out,
                      void *workspace, size_t ws_bytes, kpa_stream stream);

/* One long sequence split across GPUs (or any set of caches that each hold a
 * contiguous range of its tokens): each part decodes its range with the query's
 * global position and also reports, per head, the log-sum-exp of its scores; an
 * exchange of (out, lse) between the parts and kpa_merge_lse give the decode of the
 * whole range.  This is the split-KV merge of the pages' decoding kernel ("Tensor
 * Product Attention Is All You Need" explainer, "FlashTPA Decoding": the cache is
 * processed in blocks with an online log-sum-exp) carried across devices.
 *
 * kpa_append_factors_pos: kpa_append_factors whose token t of sequence b goes to
 * slot start_pos[b] + t but is rotated at position start_pos[b] + t + pos_offset[b]
 * (pos_offset: device [batch] int32, required), so a cache that holds positions
 * p0 .. p0 + n - 1 of a sequence can keep them in slots 0 .. n - 1.  Other rules as
 * kpa_append_factors; KPA_ERR_UNSUPPORTED for a shared-B cache (its keys are rotated
 * in the decode at the slot's position). */
kpa_status kpa_append_factors_pos(const kpa_config *cfg, int32_t batch, int32_t n_tok, const void *k_factors,
                                  const void *v_factors, const int32_t *start_pos, const int32_t *pos_offset,
                                  int32_t capacity, void *kcache, void *vcache, kpa_stream stream);

/* kpa_decode that also writes lse [batch][h] float32 (required): the natural
 * logarithm of sum_s exp(sm_scale q . k_s) over the sequence's slots (the softmax
 * normaliser, with the key reconstruction's 1/R_K; -inf for an empty sequence).  Its
 * splits always end in the combine kernel (two launches).  The workspace is sized by
 * kpa_decode_workspace_size.  KPA_ERR_UNSUPPORTED for a shared-B cache; other rules
 * as kpa_decode. */
kpa_status kpa_decode_lse(const kpa_config *cfg, int32_t batch, const void *q, const int32_t *q_pos,
                          const void *kcache, const void *vcache, int32_t capacity, const int32_t *seq_len,
                          int32_t max_len, float sm_scale, float *out, float *lse, void *workspace, size_t ws_bytes,
                          kpa_stream stream);

/* Merge n_parts normalised partial decodes of the same queries (the log-sum-exp
 * merge): out[b][h] = sum_p exp(lse_p - LSE) out_p[b][h] with LSE = ln sum_p exp(lse_p); a part with lse = -inf (no tokens) adds
 * nothing, and a head with no tokens in any part gets zeros and LSE = -inf.
 *   outs [n_parts][batch][heads][d_h] float32, lses [n_parts][batch][heads] float32
 *   out  [batch][heads][d_h] float32, lse (nullable) [batch][heads]: LSE
 * All device pointers (4-byte aligned); d_h <= 1024, n_parts <= 4096.  Asynchronous
 * on `stream`. */
kpa_status kpa_merge_lse(int32_t batch, int32_t heads, int32_t d_h, int32_t n_parts, const float *outs,
                         const float *lses, float *out, float *lse, kpa_stream stream);

/* kpa_decode with an explicit split of each sequence into pieces of
 * tokens_per_split slots (a positive multiple of 64, or 0 for the library's
 * choice).  The workspace must be sized with the same tokens_per_split. */
kpa_status kpa_decode_split(const kpa_config *cfg, int32_t batch, const void *q,
                            const int32_t *q_pos, const void *kcache, const void *vcache,
                            int32_t capacity, const int32_t *seq_len, int32_t max_len,
                            float sm_scale, int32_t tokens_per_split, float *out,
                            void *workspace, size_t ws_bytes, kpa_stream stream);

/* kpa_decode with the query given as its factors ("Kronecker Product Attention",
 * eq 2 for Q: q = (1/R_Q) sum_r A^Q_r (x) B^Q_r); the decode kernel assembles each
 * sequence's query in float32 in its prologue, so no separate assembly runs.  (The
 * FlashTPA decoding of the "Tensor Product Attention Is All You Need" explainer also
 * takes the query in factored form; here the scores are then taken against the
 * assembled query.)
 *   q_factors  float32; element e (0 <= e < E_Q = R_Q (h1 d1 + h2 d2)) of sequence b's
 *              record [A^Q_0 .. A^Q_{R_Q-1} | B^Q_0 .. B^Q_{R_Q-1}] (A_r row-major
 *              h1 x d1, B_r row-major h2 x d2) at q_factors[e * qf_stride + b * qf_seq_stride]
 *   q_pos      [batch] int32: B^Q is rotated at q_pos[b] here; NULL when the factors
 *              are already rotated (the query factors kpa_append leaves are)
 * kpa_append keeps its query factors, B^Q rotated, at the start of its workspace as
 * float32 [E_Q][batch * n_tok]: after a one-token append pass that workspace with
 * qf_stride = batch, qf_seq_stride = 1.  Requires r_q > 0 and a shape covered by a
 * tensor-core decode variant, with E_Q at most 2048 and at most h (d_h + 8) rounded down
 * to a multiple of 256 (the kernel stages the factors in its query rows); otherwise
 * KPA_ERR_UNSUPPORTED.  Everything else -- the
 * library's choice of split, workspace, outputs, errors -- as kpa_decode. */
kpa_status kpa_decode_qf(const kpa_config *cfg, int32_t batch, const float *q_factors, int32_t qf_stride,
                         int32_t qf_seq_stride, const int32_t *q_pos, const void *kcache, const void *vcache,
                         int32_t capacity, const int32_t *seq_len, int32_t max_len, float sm_scale, float *out,
                         void *workspace, size_t ws_bytes, kpa_stream stream);

/* Causal chunked attention in factor space (prefill).  Row t of sequence b is
 * the query at position start_pos[b] + t and sees slots 0 .. start_pos[b] + t
 * (its own key included), which must already be in the cache (kpa_append or
 * kpa_append_factors).  K/V tiles are rebuilt from the factors on chip only
 * ("Kronecker Product Attention", section 2.2, eq 4; Proposition 2.2), with fp16
 * products and fp32 accumulation.
 *   q    [batch][n_tok][h][d_h]  config dtype, already rotated
 *   out  [batch][n_tok][h][d_h]  float32
 *   start_pos [batch] int32; a row whose last slot is outside the cache is
 *   skipped (zeros) and sets KPA_ERR_DEVICE_CHECK.
 *   workspace at least kpa_prefill_workspace_size bytes (may be 0).
 * Takes bf16 caches of order 2 with d_h <= 128 whose per-head factor slices fit the
 * kernel's staging (R_K (d1 + d2) + R_V (d1 + d2) up to about 600 elements);
 * KPA_ERR_UNSUPPORTED otherwise.  kpa_prefill_kernel_kind says which kernel runs. */
kpa_status kpa_prefill_workspace_size(const kpa_config *cfg, int32_t batch, int32_t n_tok,
                                      size_t *bytes);
kpa_status kpa_prefill(const kpa_config *cfg, int32_t batch, int32_t n_tok, const void *q,
                       const int32_t *start_pos, const void *kcache, const void *vcache,
                       int32_t capacity, float sm_scale, float *out, void *workspace,
                       size_t ws_bytes, kpa_stream stream);

/* Which kernel kpa_prefill and kpa_prefill_qf run for this config on the calling
 * thread:
 *   KPA_PREFILL_KERNEL_TCGEN05    d1 = 8, d2 = 16, R_K = R_V = 2 (S, P and O in tensor
 *                                 memory; two 128-row query halves per CTA)
 *   KPA_PREFILL_KERNEL_MMA_SYNC   every other split it takes (128 query rows per CTA on
 *                                 mma.sync m16n8k16), or every split after
 *                                 kpa_test_set_prefill_engine(1)
 * KPA_ERR_UNSUPPORTED where neither applies (fp32, third order, d_h > 128). */
enum { KPA_PREFILL_KERNEL_MMA_SYNC = 1, KPA_PREFILL_KERNEL_TCGEN05 = 2 };
kpa_status kpa_prefill_kernel_kind(const kpa_config *cfg, int32_t *kind);

/* kpa_prefill with the queries given as factors ("Kronecker Product Attention", eq 2
 * for Q): the kernel forms each query row (1/R_Q) sum_r A^Q_r (x) B^Q_r in fp32 and
 * rounds it once to fp16 with the score scale folded in, so no dense query is written
 * or read.  The factors must already be rotated at the rows' positions (as kpa_append
 * leaves them in its workspace).
 *   q_factors  float32; element e (0 <= e < E_Q = R_Q (h1 d1 + h2 d2)) of the record
 *              [A^Q_0 .. | B^Q_0 ..] of row t of sequence b at
 *              q_factors[e * qf_stride + b * qf_seq_stride + t * qf_tok_stride]
 *              (the append's workspace: qf_stride = batch * n_tok, qf_seq_stride =
 *              n_tok, qf_tok_stride = 1); 4-byte aligned.
 * Requires 0 < r_q <= 6 (else KPA_ERR_UNSUPPORTED; r_q <= 0 is KPA_ERR_INVALID_ARG).
 * Everything else as kpa_prefill. */
kpa_status kpa_prefill_qf(const kpa_config *cfg, int32_t batch, int32_t n_tok, const float *q_factors,
                          int64_t qf_stride, int64_t qf_seq_stride, int64_t qf_tok_stride,
                          const int32_t *start_pos, const void *kcache, const void *vcache,
                          int32_t capacity, float sm_scale, float *out, void *workspace, size_t ws_bytes,
                          kpa_stream stream);

/* Append: merged factor projection, factor RoPE and cache write ("Kronecker
 * Product Attention", eq 5 with the ranks merged; Theorem 2.4; section 2.5).
 *   x  [batch][n_tok][d_model]  bf16 hidden states
 *   w  [N][d_model]             bf16 merged weights, N = (R_Q+R_K+R_V)(h1 d1 + h2 d2),
 *                               rows ordered [A^Q | B^Q | A^K | B^K | A^V | B^V],
 *                               each part rank-major (r, then row, then column)
 *   start_pos [batch] int32     token t of sequence b is at position and slot
 *                               start_pos[b] + t
 *   q_out [batch][n_tok][h][d_h] bf16 or NULL: the assembled query
 *                               (1/R_Q) sum_r A^Q_r (x) B^Q_r rotated at its position
 *   workspace at least kpa_append_workspace_size bytes; required when q_out is
 *             given, optional (NULL) otherwise.  When given, it holds on return the
 *             query factors (B^Q rotated) as float32 [E_Q][batch * n_tok] (see
 *             kpa_decode_qf)
 * Requires dtype == KPA_BF16 and d_model a multiple of 8. */
kpa_status kpa_append_workspace_size(const kpa_config *cfg, int32_t batch, int32_t n_tok,
                                     size_t *bytes);
kpa_status kpa_append(const kpa_config *cfg, int32_t batch, int32_t n_tok, const void *x,
                      const void *w, const int32_t *start_pos, int32_t capacity,
                      void *kcache, void *vcache, void *q_out, void *workspace,
                      size_t ws_bytes, kpa_stream stream);

/* Upper bound, in bytes, of the scratch that kpa_decode_noalloc can use. */
#define KPA_DECODE_NOALLOC_MAX_BYTES (16u << 20)

/* kpa_decode for callers that cannot allocate device memory (code running
 * while a stream is captured in a mode that forbids allocation, plugins whose
 * host framework owns all device memory, serving loops that must not allocate
 * on the decode path).  The pages have no counterpart: this is a deployment
 * convenience, not part of the method.
 * Same arguments and results as kpa_decode with the library's choice of split,
 * minus the workspace: the scratch lives in a fixed array of
 * KPA_DECODE_NOALLOC_MAX_BYTES in the library's own device memory, which every
 * GPU that loads the library holds until the process exits.  A request whose
 * kpa_decode_workspace_size exceeds that bound returns KPA_ERR_WORKSPACE and
 * enqueues nothing.  The call allocates and frees nothing.  The first call on
 * each device looks up the array's device address (with that device current),
 * so make that first call before capturing a stream.  All calls on a device
 * share the array; calls whose work overlaps on the GPU race on it and must be
 * serialised by the caller. */
kpa_status kpa_decode_noalloc(const kpa_config *cfg, int32_t batch, const void *q,
                              const int32_t *q_pos, const void *kcache, const void *vcache,
                              int32_t capacity, const int32_t *seq_len, int32_t max_len,
                              float sm_scale, float *out, kpa_stream stream);

/* Testing only: make the tensor-core decode's bounded waits observable.
 * Every bounded wait on the device gives up after wait_limit_ns (default 1 s)
 * and reports KPA_ERR_TIMEOUT; with skip_tile >= 0 the CTA of split
 * `skip_split` of sequence 0 never issues the copy of its tile `skip_tile`, so
 * its consumers' wait runs out.  (-1, -1, 1000000000) restores the defaults.
 * The setting belongs to the calling host thread: it changes that thread's later
 * calls only. */
kpa_status kpa_test_set_decode_hooks(int32_t skip_tile, int32_t skip_split, uint64_t wait_limit_ns);

/* Testing and measurement: choose the decode kernel.  0 (the default) runs every
 * bf16 tensor-core decode on the mma.sync kernel.  1 runs a dense-query decode of
 * the TPA shape h = 16, d_h = 64, R_K = R_V = 2 on the tcgen05 kernel (both
 * products on tcgen05, accumulators in tensor memory; its splits merge through
 * global memory, never in a cluster); other shapes and kpa_decode_qf are
 * unaffected.  2 runs kpa_decode_qf on TPA shapes (h2 = 1, d1 = 1, d_h = 64, h <= 32,
 * R_Q R_K <= 32, R_K and R_V <= 4, bf16) with the factored score of Proposition 2.2
 * (the FlashTPA form: head-shared dots B^Q_r . B^K_r' per token, then a rank mix per
 * head) on CUDA cores, its splits merged by the combine pass; other calls are
 * unaffected.  The setting belongs to the calling host thread (other threads keep
 * their own, 0 unless they set it); returns KPA_ERR_INVALID_ARG for other values. */
kpa_status kpa_test_set_decode_engine(int32_t engine);

/* Testing and measurement: choose the prefill kernel.  0 (the default) runs the
 * tcgen05 kernel where it is instantiated and the mma.sync kernel elsewhere; 1 runs
 * the mma.sync kernel for every split it takes, so the two can be compared on the
 * same shape.  Belongs to the calling host thread; KPA_ERR_INVALID_ARG for other
 * values. */
kpa_status kpa_test_set_prefill_engine(int32_t engine);

/* Testing only: y[i] = 2^x[i] for i < n (device arrays, float32) through the
 * prefill's FMA-pipe exponential (Cody-Waite reduction to [-1/2, 1/2] and a fitted
 * degree-4 polynomial, kpa_f32x2.cuh; inputs below -126 are taken as -126), so a
 * test can compare it with CUDA's exp2f and with float64 over its whole domain.
 * KPA_ERR_INVALID_ARG for n < 0 or null arrays; asynchronous on `stream`. */
kpa_status kpa_test_exp2_poly(const float *x, float *y, int64_t n, kpa_stream stream);

/* Wait for `stream`, then return in *code the per-device error word
 * (KPA_OK, KPA_ERR_TIMEOUT or KPA_ERR_DEVICE_CHECK) of the current device and
 * clear it.  The only call that synchronises. */
kpa_status kpa_read_device_error(kpa_stream stream, int32_t *code);

#ifdef __cplusplus
}
#endif

#endif /* KPA_H */
