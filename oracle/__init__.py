"""Float64 CPU oracle for factor-space KPA / TPA attention.

TEST INFRASTRUCTURE ONLY: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA library and never imports it.

The arithmetic lives in ``kpa_oracle.c`` (plain C, float64, no BLAS); this
module only builds it with gcc, marshals numpy arrays into it, and composes the
definitions the way the pages state them:

* ``decode``  -- one query row per sequence against slots ``0 .. seq_len-1``;
* ``prefill`` -- causal rows: query ``t`` sees slots ``0 .. start + t``;
* ``append``  -- merged factor projection (KPA paper, eq 5), the split into
  query / key / value records, RoPE on the B factors of keys (Theorem 2.4) and
  the assembled, rotated query (eq 2 followed by Definition 2.3).

Third-order TPA (``decode_order3`` and its helpers) is composed from the pinned
primitives above and pinned by ``tests/pins.py::check_order3_attention``.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
except the column order of the merged projection weights
``[A^Q | B^Q | A^K | B^K | A^V | B^V]``, a convention the pages do not fix
(parity unpinned beyond self-consistency).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kpa_oracle.c")
_LIB = os.path.join(_HERE, "libkpa_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the C oracle (gcc, OpenMP, IEEE floating point, no contraction)."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    tmp = out + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-Wall", "-Wextra", "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def _bind(path: str):
    lib = ctypes.CDLL(path)
    c_int, c_double = ctypes.c_int, ctypes.c_double
    lib.oracle_kron.argtypes = [c_int, c_int, _dp, c_int, c_int, _dp, _dp]
    lib.oracle_kron_sum_row.argtypes = [c_int] * 5 + [_dp, c_int, _dp]
    lib.oracle_reconstruct.argtypes = [c_int] * 5 + [_dp, _dp]
    lib.oracle_rope_d2.argtypes = [c_int, c_double, c_double, _dp]
    lib.oracle_rope_kpa.argtypes = [c_int, c_int, c_double, c_double, _dp]
    lib.oracle_rotate_record.argtypes = [c_int] * 5 + [c_double, c_double, _dp]
    lib.oracle_project.argtypes = [c_int, c_int, c_int, _dp, _dp, _dp]
    lib.oracle_attend.argtypes = ([c_int] * 6 + [c_double] + [c_int, c_int, _dp, _i64p, _dp, _dp,
                                   c_int, _i32p, c_int, c_double, _dp, c_int, _i32p, _dp])
    lib.oracle_attend.restype = c_int
    lib.oracle_cache_numbers_per_token.argtypes = [c_int] * 6
    lib.oracle_cache_numbers_per_token.restype = ctypes.c_int64
    lib.oracle_mha_numbers_per_token.argtypes = [c_int] * 4
    lib.oracle_mha_numbers_per_token.restype = ctypes.c_int64
    lib.oracle_compression.argtypes = [c_int] * 6
    lib.oracle_compression.restype = c_double
    lib.oracle_set_threads.argtypes = [c_int]
    lib.oracle_max_threads.restype = c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(build())
        return _lib


class use_library:
    """Context manager that points this module at another build of the oracle
    (used by the tests that plant a mistake in a copy of the C source)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        _load()
        with _lock:
            self.saved = _lib
            _lib = _bind(self.path)
        return self

    def __exit__(self, *exc):
        global _lib
        with _lock:
            _lib = self.saved
        return False


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray, typ=_dp):
    return a.ctypes.data_as(typ)


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


# ---------------------------------------------------------------- primitives
def kron(A, B) -> np.ndarray:
    """Definition 2.1 (KPA paper, section 2.1)."""
    A, B = _f64(A), _f64(B)
    out = np.empty((A.shape[0] * B.shape[0], A.shape[1] * B.shape[1]))
    _load().oracle_kron(A.shape[0], A.shape[1], _ptr(A), B.shape[0], B.shape[1], _ptr(B), _ptr(out))
    return out


def reconstruct(h1, h2, d1, d2, R, rec) -> np.ndarray:
    """(1/R) sum_r A_r (x) B_r from one factor record (eqs 2-4)."""
    rec = _f64(rec).reshape(-1)
    assert rec.size == R * (h1 * d1 + h2 * d2)
    out = np.empty((h1 * h2, d1 * d2))
    _load().oracle_reconstruct(h1, h2, d1, d2, R, _ptr(rec), _ptr(out))
    return out


def kron_sum_row(h1, h2, d1, d2, R, rec, row) -> np.ndarray:
    rec = _f64(rec).reshape(-1)
    out = np.empty(d1 * d2)
    _load().oracle_kron_sum_row(h1, h2, d1, d2, R, _ptr(rec), int(row), _ptr(out))
    return out


def rope_d2(d2, base, pos, v) -> np.ndarray:
    """R_theta^(2)(pos) v (Definition 2.3); returns a new array."""
    v = _f64(v).copy()
    _load().oracle_rope_d2(d2, float(base), float(pos), _ptr(v))
    return v


def rope_kpa(d1, d2, base, pos, v) -> np.ndarray:
    """(I_{d1} (x) R_theta^(2)(pos)) v (Definition 2.3); returns a new array."""
    v = _f64(v).copy()
    _load().oracle_rope_kpa(d1, d2, float(base), float(pos), _ptr(v))
    return v


def rotate_record(h1, h2, d1, d2, R, base, pos, rec) -> np.ndarray:
    """Rotate only the B factors of one record (Theorem 2.4)."""
    rec = _f64(rec).reshape(-1).copy()
    _load().oracle_rotate_record(h1, h2, d1, d2, R, float(base), float(pos), _ptr(rec))
    return rec


def project(x, W) -> np.ndarray:
    """Merged factor projection factors = x W^T (eq 5 with the ranks merged)."""
    x, W = _f64(x), _f64(W)
    n, dm = x.shape
    N = W.shape[0]
    assert W.shape[1] == dm
    out = np.empty((n, N))
    _load().oracle_project(n, dm, N, _ptr(x), _ptr(W), _ptr(out))
    return out


def cache_numbers_per_token(h1, h2, d1, d2, r_k, r_v) -> int:
    """eq 10: (R_K + R_V)(h1 d1 + h2 d2)."""
    return int(_load().oracle_cache_numbers_per_token(h1, h2, d1, d2, r_k, r_v))


def mha_numbers_per_token(h1, h2, d1, d2) -> int:
    return int(_load().oracle_mha_numbers_per_token(h1, h2, d1, d2))


def compression(h1, h2, d1, d2, r_k, r_v) -> float:
    """eq 10 / eq 11: C_KPA = 2 h1 h2 d1 d2 / ((R_K + R_V)(h1 d1 + h2 d2))."""
    return float(_load().oracle_compression(h1, h2, d1, d2, r_k, r_v))


# ------------------------------------------------------------ attention core
def attend(shape, q, kf, vf, n_keys, *, q_pos=None, keys_rotated=False, sm_scale=None,
           heads=None, return_lse=False):
    """Softmax attention over factor-cache slots (see ``oracle_attend`` in C).

    q  [B][n_q][h][dh]; kf, vf [B][cap][E]; n_keys [B][n_q]; q_pos [B][n_q] or None.
    ``heads``: optional iterable of flat ``b*h + head`` indices; other heads come
    back as NaN.  With ``return_lse`` also the softmax normaliser of each row,
    ln sum_s exp(score_s), as [B][n_q][h] (-inf with no visible slot).
    """
    s = shape
    h, dh = s.h1 * s.h2, s.d1 * s.d2
    q = _f64(q)
    B, n_q = q.shape[0], q.shape[1]
    assert q.shape == (B, n_q, h, dh), q.shape
    kf, vf = _f64(kf), _f64(vf)
    cap = kf.shape[1]
    assert kf.shape == (B, cap, s.r_k * (s.h1 * s.d1 + s.h2 * s.d2)), kf.shape
    assert vf.shape == (B, cap, s.r_v * (s.h1 * s.d1 + s.h2 * s.d2)), vf.shape
    nk = np.ascontiguousarray(np.asarray(n_keys, dtype=np.int32).reshape(B, n_q))
    qp = None if q_pos is None else np.ascontiguousarray(np.asarray(q_pos, dtype=np.int64).reshape(B, n_q))
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(dh)
    out = np.full((B, n_q, h, dh), np.nan)
    hl = None if heads is None else np.ascontiguousarray(np.asarray(list(heads), dtype=np.int32))
    lse = np.full((B, n_q, h), np.nan) if return_lse else None
    rc = _load().oracle_attend(
        s.h1, s.h2, s.d1, s.d2, s.r_k, s.r_v, float(s.rope_base), B, n_q, _ptr(q),
        None if qp is None else _ptr(qp, _i64p), _ptr(kf), _ptr(vf), cap, _ptr(nk, _i32p),
        1 if keys_rotated else 0, float(sm_scale), _ptr(out),
        0 if hl is None else int(hl.size), None if hl is None else _ptr(hl, _i32p),
        None if lse is None else _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attend rejected its arguments")
    return (out, lse) if return_lse else out


def decode(shape, q, kf, vf, seq_len, *, q_pos=None, keys_rotated=False, sm_scale=None,
           heads=None, return_lse=False):
    """One query row per sequence: q [B][h][dh] -> out [B][h][dh] (and with
    ``return_lse`` the softmax normaliser [B][h], see ``attend``)."""
    q = _f64(q)
    B = q.shape[0]
    res = attend(shape, q[:, None], kf, vf, np.asarray(seq_len).reshape(B, 1),
                 q_pos=None if q_pos is None else np.asarray(q_pos).reshape(B, 1),
                 keys_rotated=keys_rotated, sm_scale=sm_scale, heads=heads, return_lse=return_lse)
    if return_lse:
        return res[0][:, 0], res[1][:, 0]
    return res[:, 0]


def decode_shared_b(shape, q, kf, va, seq_len, *, q_pos=None, sm_scale=None, heads=None) -> np.ndarray:
    """Decode over a cache whose keys and values share their B factors ("Tensor Product
    Attention Is All You Need", section 5, "TPA KV with Shared B": b_r^K = b_r^V, so
    R_K = R_V = R).  Key of slot t: the rotation at position t of (1/R) sum_r A^K_r (x) B_r;
    value of slot t: (1/R) sum_r A^V_r (x) B_r, with the same, unrotated, B_r.

    kf [B][cap][R(h1 d1 + h2 d2)] holds [A^K | B] (B unrotated); va [B][cap][R h1 d1] holds
    A^V.  The value record [A^V | B] is formed and the plain definition (``decode`` with
    keys rotated at their slots) does the rest.
    """
    s = shape
    R = s.r_k
    assert s.r_v == R, "a shared B needs R_K == R_V"
    kf, va = _f64(kf), _f64(va)
    a = R * s.h1 * s.d1
    assert va.shape == kf.shape[:2] + (a,), va.shape
    vf = np.concatenate([va, kf[:, :, a:]], axis=2)
    return decode(s, q, kf, vf, seq_len, q_pos=q_pos, keys_rotated=False, sm_scale=sm_scale, heads=heads)


def cache_numbers_per_token_shared_b(h1, h2, d1, d2, r) -> int:
    """Numbers cached per token with one B set for keys and values: A^K, A^V and B."""
    return 2 * r * h1 * d1 + r * h2 * d2


# ------------------------------------------------------------ third-order TPA
# "Tensor Product Attention Is All You Need", Appendix C, as the explainer page
# summarises it: a third-order factor component is a_r (x) vec(b_r (x) c_r) with
# a_r in R^h, b_r in R^{d_b}, c_r in R^{d_c}, d_h = d_b d_c, and RoPE (Theorem C.1)
# acts on the b factors only: (R_{d_b}(p) (x) I_{d_c}) vec(b (x) c) = vec(R_{d_b}(p) b (x) c).
# Here vec(b (x) c) is the Kronecker product of the two vectors (b's index the slower
# one, Definition 2.1), and R_{d_b} is Definition 2.3's rotation on a d_b-vector.
# A record of one token is [a_0..a_{R-1} | b_0..b_{R-1} | c_0..c_{R-1}]; shapes carry
# h1 = h, h2 = 1, d1 = d_b, d2 = d_c.

def order3_as_kronecker(h, d_b, d_c, R, rec) -> np.ndarray:
    """The same R components written as a Kronecker record of the split h1 = h, h2 = 1,
    d1 = d_b, d2 = d_c: A_r = a_r b_r^T (h x d_b), B_r = c_r^T (1 x d_c), so that row h of
    (1/R) sum_r A_r (x) B_r is (1/R) sum_r a_r[h] (b_r (x) c_r).
    rec [..., R(h + d_b + d_c)] -> [..., R(h d_b + d_c)]."""
    rec = _f64(rec)
    lead = rec.shape[:-1]
    assert rec.shape[-1] == R * (h + d_b + d_c), rec.shape
    a = rec[..., :R * h].reshape(lead + (R, h))
    b = rec[..., R * h:R * (h + d_b)].reshape(lead + (R, d_b))
    c = rec[..., R * (h + d_b):].reshape(lead + (R, d_c))
    A = a[..., :, :, None] * b[..., :, None, :]
    return np.concatenate([A.reshape(lead + (R * h * d_b,)), c.reshape(lead + (R * d_c,))], axis=-1)


def rotate_order3_b(h, d_b, d_c, R, base, pos, rec) -> np.ndarray:
    """One record with every b_r rotated by R_{d_b}(pos) (pairs (2m, 2m+1), theta_m =
    base^(-2m/d_b)); a and c unchanged.  Returns a new array."""
    rec = _f64(rec).reshape(-1).copy()
    for r in range(R):
        o = R * h + r * d_b
        rec[o:o + d_b] = rope_d2(d_b, base, pos, rec[o:o + d_b])
    return rec


def rope_order3_query(h, d_b, d_c, base, pos, q) -> np.ndarray:
    """(R_{d_b}(pos) (x) I_{d_c}) applied to every head row of a dense query [h][d_b d_c]."""
    q = _f64(q).reshape(h, d_b, d_c).copy()
    for i in range(h):
        for jc in range(d_c):
            q[i, :, jc] = rope_d2(d_b, base, pos, q[i, :, jc])
    return q.reshape(h, d_b * d_c)


class _KronShape:
    def __init__(self, h1, h2, d1, d2, r_k, r_v, rope_base):
        self.h1, self.h2, self.d1, self.d2 = h1, h2, d1, d2
        self.r_k, self.r_v, self.rope_base = r_k, r_v, rope_base


def decode_order3(shape, q, kf, vf, seq_len, *, q_pos=None, keys_rotated=False, sm_scale=None,
                  heads=None) -> np.ndarray:
    """Decode over a third-order TPA cache: kf, vf [B][cap][R(h + d_b + d_c)] with
    shape.h1 = h, shape.h2 = 1, shape.d1 = d_b, shape.d2 = d_c.  The key of slot t has its
    b factors rotated at t (unless ``keys_rotated``: the cache already holds them so), the
    query is rotated at q_pos by R_{d_b} (x) I_{d_c}, values are not rotated.  The records
    are then written in Kronecker form and the plain attention definition (``decode`` with
    the keys taken as rotated and the query as given) does the rest."""
    s = shape
    assert s.h2 == 1, "third-order TPA has its heads in the a factors"
    h, db, dc = s.h1, s.d1, s.d2
    q, kf, vf = _f64(q), _f64(kf), _f64(vf)
    B = q.shape[0]
    if not keys_rotated:
        kf = kf.copy()
        for b in range(B):
            for t in range(int(np.asarray(seq_len).reshape(-1)[b])):
                kf[b, t] = rotate_order3_b(h, db, dc, s.r_k, s.rope_base, t, kf[b, t])
    if q_pos is not None:
        qp = np.asarray(q_pos).reshape(-1)
        q = np.stack([rope_order3_query(h, db, dc, s.rope_base, int(qp[b]), q[b]) for b in range(B)])
    ks = _KronShape(h, 1, db, dc, s.r_k, s.r_v, s.rope_base)
    return decode(ks, q, order3_as_kronecker(h, db, dc, s.r_k, kf), order3_as_kronecker(h, db, dc, s.r_v, vf),
                  seq_len, q_pos=None, keys_rotated=True, sm_scale=sm_scale, heads=heads)


def cache_numbers_per_token_order3(h, d_b, d_c, r_k, r_v) -> int:
    """Numbers cached per token by a third-order TPA cache: (R_K + R_V)(h + d_b + d_c)."""
    return (r_k + r_v) * (h + d_b + d_c)


def prefill(shape, q, kf, vf, start_pos, *, q_pos=None, keys_rotated=False, sm_scale=None,
            heads=None) -> np.ndarray:
    """Causal rows: q [B][n][h][dh]; row t of sequence b sees slots 0..start_pos[b]+t."""
    q = _f64(q)
    B, n = q.shape[0], q.shape[1]
    start = np.asarray(start_pos, dtype=np.int64).reshape(B, 1)
    n_keys = start + np.arange(n, dtype=np.int64)[None, :] + 1
    return attend(shape, q, kf, vf, n_keys, q_pos=q_pos, keys_rotated=keys_rotated,
                  sm_scale=sm_scale, heads=heads)


# ------------------------------------------------------------------- append
def split_columns(shape):
    """Column ranges of the merged projection output, in the order
    [A^Q | B^Q | A^K | B^K | A^V | B^V] (a convention; see module docstring).  With one
    B shared by keys and values the order is [A^Q | B^Q | A^K | A^V | B] and the ranges
    are returned as (A^Q, B^Q, A^K, B, A^V, B): the key and the value take the same B."""
    s = shape
    a, b = s.h1 * s.d1, s.h2 * s.d2
    if getattr(s, "shared_b", 0):
        widths = [s.r_q * a, s.r_q * b, s.r_k * a, s.r_k * a, s.r_k * b]
        e = np.cumsum([0] + widths)
        aq, bq, ak, av, bb = [(int(e[i]), int(e[i + 1])) for i in range(5)]
        return [aq, bq, ak, bb, av, bb]
    widths = [s.r_q * a, s.r_q * b, s.r_k * a, s.r_k * b, s.r_v * a, s.r_v * b]
    edges = np.cumsum([0] + widths)
    return [(int(edges[i]), int(edges[i + 1])) for i in range(6)]


def append(shape, x, W, start_pos):
    """Oracle of the append step for x [B][n][d_model], W [N][d_model].

    Returns ``(q_rot, k_rec_rot, v_rec, k_rec)``:
      q_rot     [B][n][h][dh]  (1/R_Q) sum_r A^Q_r (x) B^Q_r, each head row
                              rotated by R_KPA(start_pos[b] + t)
      k_rec_rot [B][n][E_K]    key records with B^K rotated at the token position
      v_rec     [B][n][E_V]    value records (never rotated)
      k_rec     [B][n][E_K]    unrotated key records

    With a shared B (``shape.shared_b``) the key record is [A^K | B], v_rec is [A^V]
    alone, and the cache keeps B unrotated: k_rec_rot is then k_rec.
    """
    s = shape
    x = _f64(x)
    B, n, dm = x.shape
    h, dh = s.h1 * s.h2, s.d1 * s.d2
    fac = project(x.reshape(B * n, dm), W).reshape(B, n, -1)
    cols = split_columns(s)
    q_rec = np.concatenate([fac[..., cols[0][0]:cols[0][1]], fac[..., cols[1][0]:cols[1][1]]], axis=-1)
    k_rec = np.concatenate([fac[..., cols[2][0]:cols[2][1]], fac[..., cols[3][0]:cols[3][1]]], axis=-1)
    shared = bool(getattr(s, "shared_b", 0))
    if shared:
        v_rec = fac[..., cols[4][0]:cols[4][1]].copy()
    else:
        v_rec = np.concatenate([fac[..., cols[4][0]:cols[4][1]], fac[..., cols[5][0]:cols[5][1]]], axis=-1)
    q_rot = np.empty((B, n, h, dh))
    k_rot = np.empty_like(k_rec)
    start = np.asarray(start_pos, dtype=np.int64).reshape(B)
    for b in range(B):
        for t in range(n):
            pos = int(start[b]) + t
            Q = reconstruct(s.h1, s.h2, s.d1, s.d2, s.r_q, q_rec[b, t])
            for head in range(h):
                q_rot[b, t, head] = rope_kpa(s.d1, s.d2, s.rope_base, pos, Q[head])
            k_rot[b, t] = k_rec[b, t] if shared else \
                rotate_record(s.h1, s.h2, s.d1, s.d2, s.r_k, s.rope_base, pos, k_rec[b, t])
    return q_rot, k_rot, v_rec, k_rec
