"""Checks that pin the float64 oracle to what the pages and the mathematics fix.

Each ``check_*`` function raises ``AssertionError`` on a mismatch.  The pin
tests call them against the oracle as built; the mutation tests call them
against copies of the oracle with a planted mistake and expect at least one to
fail.  Nothing here retypes the oracle's own formula: each check compares it
with a library routine (numpy.kron, torch's scaled_dot_product_attention, a
numpy matmul), a closed form or printed value from the pages, an identity the
pages prove, or a brute-force special case.
"""
from __future__ import annotations

import cmath
import json
import math
import os

import numpy as np
import torch

import oracle
from workloads import Shape

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _close(a, b, tol, what):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    assert np.all(np.isfinite(a)) and np.all(np.isfinite(b)), f"{what}: non-finite values"
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol, f"{what}: max |diff| {err:.3e} > {tol:.1e}"


def _record(rng, s: Shape, R):
    return rng.standard_normal(R * (s.h1 * s.d1 + s.h2 * s.d2))


def _split_record(s: Shape, R, rec):
    a = rec[: R * s.h1 * s.d1].reshape(R, s.h1, s.d1)
    b = rec[R * s.h1 * s.d1:].reshape(R, s.h2, s.d2)
    return a, b


def _rot_matrix_d2(d2, base, pos):
    """R_theta^(2)(pos) as a matrix, column j = the oracle's rotation of e_j."""
    return np.stack([oracle.rope_d2(d2, base, pos, np.eye(d2)[j]) for j in range(d2)], axis=1)


SHAPES = [
    Shape(h1=2, h2=3, d1=2, d2=4, r_k=2, r_v=3, rope_base=10000.0),
    Shape(h1=4, h2=8, d1=8, d2=16, r_k=4, r_v=4, rope_base=10000.0),
    Shape(h1=16, h2=1, d1=1, d2=64, r_k=2, r_v=2, rope_base=10000.0),   # TPA split
    Shape(h1=3, h2=2, d1=4, d2=2, r_k=1, r_v=2, rope_base=500000.0),
]


# ------------------------------------------------------------- Definition 2.1
def check_kron_is_numpy_kron(seed=0):
    rng = np.random.default_rng(seed)
    for (m1, n1, m2, n2) in [(1, 1, 1, 1), (2, 3, 4, 5), (4, 8, 8, 16), (3, 1, 1, 7)]:
        A, B = rng.standard_normal((m1, n1)), rng.standard_normal((m2, n2))
        _close(oracle.kron(A, B), np.kron(A, B), 0.0, f"kron {m1}x{n1} (x) {m2}x{n2}")


def check_reconstruct_is_kron_sum(seed=1):
    """eqs (2)-(4): X = (1/R) sum_r A_r (x) B_r, against numpy.kron."""
    rng = np.random.default_rng(seed)
    for s in SHAPES:
        for R in (1, s.r_k, 3):
            rec = _record(rng, s, R)
            a, b = _split_record(s, R, rec)
            ref = sum(np.kron(a[r], b[r]) for r in range(R)) / R
            _close(oracle.reconstruct(s.h1, s.h2, s.d1, s.d2, R, rec), ref, 1e-14, f"reconstruct {s} R={R}")
            for row in (0, s.h - 1, s.h // 2):
                _close(oracle.kron_sum_row(s.h1, s.h2, s.d1, s.d2, R, rec, row), ref[row], 1e-14,
                       "kron_sum_row")


def check_tpa_split_is_outer_product(seed=2):
    """h1=h, d1=1, h2=1, d2=d_h reduces each term to a rank-one outer product
    (KPA paper section 2.2, final paragraph; TPA explainer, factorisation formula)."""
    rng = np.random.default_rng(seed)
    for h, dh, R in [(16, 64, 2), (5, 6, 3), (61, 64, 1)]:
        s = Shape(h1=h, h2=1, d1=1, d2=dh, r_k=R, r_v=R)
        rec = _record(rng, s, R)
        a = rec[: R * h].reshape(R, h)
        b = rec[R * h:].reshape(R, dh)
        ref = sum(np.outer(a[r], b[r]) for r in range(R)) / R
        _close(oracle.reconstruct(h, 1, 1, dh, R, rec), ref, 1e-14, "TPA outer product")


# ---------------------------------------------------------- Proposition 2.2
def check_prop22_factored_score(seed=3):
    """eq (6): q_(i1,i2) . k_(i1,i2) = 1/(R_Q R_K) sum_{r,r'} [A^Q_r A^K_r' row i1]
    [B^Q_r B^K_r' row i2], with q and k the reconstructed rows."""
    rng = np.random.default_rng(seed)
    for s in SHAPES:
        RQ, RK = 3, s.r_k
        qrec, krec = _record(rng, s, RQ), _record(rng, s, RK)
        Q = oracle.reconstruct(s.h1, s.h2, s.d1, s.d2, RQ, qrec)
        K = oracle.reconstruct(s.h1, s.h2, s.d1, s.d2, RK, krec)
        aq, bq = _split_record(s, RQ, qrec)
        ak, bk = _split_record(s, RK, krec)
        for i1 in range(s.h1):
            for i2 in range(s.h2):
                head = i1 * s.h2 + i2
                fact = sum(float(aq[r, i1] @ ak[rp, i1]) * float(bq[r, i2] @ bk[rp, i2])
                           for r in range(RQ) for rp in range(RK)) / (RQ * RK)
                dense = float(Q[head] @ K[head])
                assert abs(dense - fact) <= 1e-12 * max(1.0, abs(fact)), \
                    f"Prop 2.2 {s} head ({i1},{i2}): {dense} vs {fact}"


# ------------------------------------------------------------ Definition 2.3
def check_rope_golden_frequencies():
    """theta_m = base^(-2m/d2) at hand-evaluated points; pairs (2m, 2m+1)."""
    g = _golden("rope_frequencies.json")
    for case in g["cases"]:
        d2, base = case["d2"], case["base"]
        for pos in g["positions"]:
            for m, theta in case["theta"]:
                phi = pos * theta
                e0 = np.zeros(d2); e0[2 * m] = 1.0
                e1 = np.zeros(d2); e1[2 * m + 1] = 1.0
                r0 = oracle.rope_d2(d2, base, pos, e0)
                r1 = oracle.rope_d2(d2, base, pos, e1)
                want0 = np.zeros(d2); want0[2 * m] = math.cos(phi); want0[2 * m + 1] = math.sin(phi)
                want1 = np.zeros(d2); want1[2 * m] = -math.sin(phi); want1[2 * m + 1] = math.cos(phi)
                tol = 1e-12 * max(1.0, abs(phi))
                _close(r0, want0, tol, f"rope d2={d2} base={base} pos={pos} m={m} (e_2m)")
                _close(r1, want1, tol, f"rope d2={d2} base={base} pos={pos} m={m} (e_2m+1)")


def check_rope_tpa_is_textbook(seed=4):
    """With d1 = 1 the operator is ordinary RoPE on d_h features, written here as
    complex multiplication z_m * exp(i pos theta_m), theta_m = base^(-2m/d_h)
    (RoFormer form; TPA explainer, 'RoPE Compatibility' paragraph)."""
    rng = np.random.default_rng(seed)
    for dh, base in [(64, 10000.0), (8, 10000.0), (128, 500000.0)]:
        for pos in (0, 1, 7, 4096, 524288):
            v = rng.standard_normal(dh)
            got = oracle.rope_kpa(1, dh, base, pos, v)
            want = np.empty(dh)
            for m in range(dh // 2):
                z = complex(v[2 * m], v[2 * m + 1]) * cmath.exp(1j * pos * base ** (-2.0 * m / dh))
                want[2 * m], want[2 * m + 1] = z.real, z.imag
            _close(got, want, 1e-11 * max(1, pos) ** 0.5, f"textbook RoPE dh={dh} pos={pos}")


def check_rope_kpa_is_identity_kron_rotation(seed=5):
    """Definition 2.3: R_KPA = I_{d1} (x) R^(2), built with numpy.kron."""
    rng = np.random.default_rng(seed)
    for d1, d2, base in [(8, 8, 10000.0), (8, 16, 500000.0), (1, 64, 10000.0), (3, 4, 10000.0)]:
        for pos in (0, 5, 2048, 524288):
            R2 = _rot_matrix_d2(d2, base, pos)
            v = rng.standard_normal(d1 * d2)
            _close(oracle.rope_kpa(d1, d2, base, pos, v), np.kron(np.eye(d1), R2) @ v, 1e-12,
                   f"I(x)R d1={d1} d2={d2} pos={pos}")
            # a rotation: orthogonal, determinant 1
            _close(R2.T @ R2, np.eye(d2), 1e-12, "R^(2) orthogonal")


# -------------------------------------------------------------- Theorem 2.4
def check_thm24_rotating_b_equals_rotating_reconstruction(seed=6):
    """eqs (7)-(8): reconstruct(rotate only B) = (I (x) R) applied to each row."""
    rng = np.random.default_rng(seed)
    for s in SHAPES:
        for pos in (0, 1, 300, 524287):
            rec = _record(rng, s, s.r_k)
            left = oracle.reconstruct(s.h1, s.h2, s.d1, s.d2, s.r_k,
                                      oracle.rotate_record(s.h1, s.h2, s.d1, s.d2, s.r_k, s.rope_base, pos, rec))
            X = oracle.reconstruct(s.h1, s.h2, s.d1, s.d2, s.r_k, rec)
            right = np.stack([oracle.rope_kpa(s.d1, s.d2, s.rope_base, pos, X[i]) for i in range(s.h)])
            _close(left, right, 1e-12, f"Thm 2.4 {s} pos={pos}")
            # the A factors are left as they are
            _close(oracle.rotate_record(s.h1, s.h2, s.d1, s.d2, s.r_k, s.rope_base, pos, rec)[: s.r_k * s.h1 * s.d1],
                   rec[: s.r_k * s.h1 * s.d1], 0.0, "A unrotated")


def check_relative_position(seed=7):
    """eq (9) and the proof of Theorem 2.4: R(t)^T R(s) = R(s - t), so the score
    depends only on s - t; shifting both positions leaves it unchanged."""
    rng = np.random.default_rng(seed)
    for d1, d2, base in [(8, 8, 10000.0), (8, 16, 500000.0), (1, 64, 10000.0)]:
        for (t, s_, delta) in [(0, 5, 11), (256, 3, 1000), (524288, 100, 7), (2047, 2047, 524288)]:
            q, k = rng.standard_normal(d1 * d2), rng.standard_normal(d1 * d2)
            a = oracle.rope_kpa(d1, d2, base, t, q) @ oracle.rope_kpa(d1, d2, base, s_, k)
            b = oracle.rope_kpa(d1, d2, base, t + delta, q) @ oracle.rope_kpa(d1, d2, base, s_ + delta, k)
            c = q @ oracle.rope_kpa(d1, d2, base, s_ - t, k)
            tol = 1e-9 * max(1.0, np.abs(q).sum() * np.abs(k).max())
            assert abs(a - b) <= tol and abs(a - c) <= tol, f"relative position {d1}x{d2}: {a} {b} {c}"


# --------------------------------------------------- softmax attention (SDPA)
def _reference_attention(s: Shape, q, q_pos, kf, vf, n_keys, sm_scale, return_lse=False):
    """numpy.kron reconstruction, numpy.kron rotation matrices and torch's
    scaled_dot_product_attention (float64, CPU) with a boolean visibility mask.  With
    return_lse also torch.logsumexp of the masked scores Q K^T * sm_scale."""
    B, n_q = q.shape[0], q.shape[1]
    cap = kf.shape[1]
    h, dh = s.h, s.dh
    K = np.zeros((B, cap, h, dh)); V = np.zeros((B, cap, h, dh))
    for b in range(B):
        for t in range(cap):
            ak, bk = _split_record(s, s.r_k, kf[b, t])
            av, bv = _split_record(s, s.r_v, vf[b, t])
            Kt = sum(np.kron(ak[r], bk[r]) for r in range(s.r_k)) / s.r_k
            Vt = sum(np.kron(av[r], bv[r]) for r in range(s.r_v)) / s.r_v
            rot = np.kron(np.eye(s.d1), _rot_matrix_d2(s.d2, s.rope_base, t))
            K[b, t] = Kt @ rot.T
            V[b, t] = Vt
    Q = np.empty_like(q)
    for b in range(B):
        for i in range(n_q):
            rot = np.kron(np.eye(s.d1), _rot_matrix_d2(s.d2, s.rope_base, q_pos[b, i]))
            Q[b, i] = q[b, i] @ rot.T
    mask = np.arange(cap)[None, None, :] < np.asarray(n_keys)[:, :, None]        # [B][n_q][cap]
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q).permute(0, 2, 1, 3), torch.from_numpy(K).permute(0, 2, 1, 3),
        torch.from_numpy(V).permute(0, 2, 1, 3), attn_mask=torch.from_numpy(mask)[:, None],
        scale=sm_scale).permute(0, 2, 1, 3).numpy()
    if not return_lse:
        return out
    scores = np.einsum("bqhd,bkhd->bqhk", Q, K) * sm_scale
    scores = np.where(mask[:, :, None, :], scores, -np.inf)
    return out, torch.logsumexp(torch.from_numpy(scores), dim=-1).numpy()


def check_attention_matches_sdpa(seed=8):
    rng = np.random.default_rng(seed)
    for s in [SHAPES[0], SHAPES[2], SHAPES[3], Shape(h1=2, h2=2, d1=4, d2=4, r_k=2, r_v=1)]:
        B, n_q, cap = 2, 3, 9
        q = rng.standard_normal((B, n_q, s.h, s.dh))
        kf = rng.standard_normal((B, cap, s.e_k)); vf = rng.standard_normal((B, cap, s.e_v))
        q_pos = rng.integers(0, 600000, size=(B, n_q))
        n_keys = rng.integers(1, cap + 1, size=(B, n_q)).astype(np.int32)
        scale = 0.7 / math.sqrt(s.dh)
        got = oracle.attend(s, q, kf, vf, n_keys, q_pos=q_pos, sm_scale=scale)
        want = _reference_attention(s, q, q_pos, kf, vf, n_keys, scale)
        _close(got, want, 1e-11, f"attention vs SDPA {s}")


def check_attention_lse(seed=18):
    """The softmax normaliser ln sum_s exp(score_s) of each row against torch.logsumexp
    of the reference scores; one visible slot gives that slot's score; none gives -inf."""
    rng = np.random.default_rng(seed)
    for s in [SHAPES[0], SHAPES[3], Shape(h1=2, h2=2, d1=4, d2=4, r_k=2, r_v=1)]:
        B, n_q, cap = 2, 3, 9
        q = rng.standard_normal((B, n_q, s.h, s.dh))
        kf = rng.standard_normal((B, cap, s.e_k)); vf = rng.standard_normal((B, cap, s.e_v))
        q_pos = rng.integers(0, 600000, size=(B, n_q))
        n_keys = rng.integers(1, cap + 1, size=(B, n_q)).astype(np.int32)
        n_keys[0, 0] = 1
        scale = 0.7 / math.sqrt(s.dh)
        got_o, got_l = oracle.attend(s, q, kf, vf, n_keys, q_pos=q_pos, sm_scale=scale, return_lse=True)
        want_o, want_l = _reference_attention(s, q, q_pos, kf, vf, n_keys, scale, return_lse=True)
        _close(got_o, want_o, 1e-11, f"attention (with lse) vs SDPA {s}")
        _close(got_l, want_l, 1e-11, f"lse vs logsumexp {s}")
    _, l0 = oracle.attend(s, q, kf, vf, np.zeros((B, n_q), np.int32), q_pos=q_pos, return_lse=True)
    assert np.all(np.isneginf(l0)), "no visible slot: -inf"


def check_attention_closed_forms(seed=9):
    rng = np.random.default_rng(seed)
    s = SHAPES[1]
    B, cap = 3, 6
    kf = rng.standard_normal((B, cap, s.e_k)); vf = rng.standard_normal((B, cap, s.e_v))
    q = rng.standard_normal((B, s.h, s.dh)) * 5.0
    Vrows = np.stack([np.stack([oracle.reconstruct(s.h1, s.h2, s.d1, s.d2, s.r_v, vf[b, t])
                                for t in range(cap)]) for b in range(B)])        # [B][cap][h][dh]
    # one slot: out = V_0 whatever the query
    out = oracle.decode(s, q, kf, vf, [1, 1, 1], q_pos=[7, 0, 99])
    _close(out, Vrows[:, 0], 1e-13, "L=1 gives V_0")
    # zero query: uniform weights, out = mean of the visible V rows
    out = oracle.decode(s, np.zeros_like(q), kf, vf, [cap, 4, 2], q_pos=[cap, 4, 2])
    for b, L in enumerate([cap, 4, 2]):
        _close(out[b], Vrows[b, :L].mean(axis=0), 1e-13, "q=0 gives the mean")
    # identical (already rotated) keys: uniform weights
    kf_same = np.repeat(kf[:, :1], cap, axis=1)
    out = oracle.decode(s, q, kf_same, vf, [cap] * B, keys_rotated=True)
    _close(out, Vrows.mean(axis=1), 1e-12, "identical keys give the mean")
    # no visible slot: zeros
    out = oracle.decode(s, q, kf, vf, [0, 0, 0], q_pos=[0, 0, 0])
    _close(out, np.zeros_like(out), 0.0, "empty sequence")


def check_prefill_rows_are_decodes(seed=10):
    rng = np.random.default_rng(seed)
    s = SHAPES[0]
    B, n, cap = 2, 5, 12
    start = np.array([0, 4])
    kf = rng.standard_normal((B, cap, s.e_k)); vf = rng.standard_normal((B, cap, s.e_v))
    q = rng.standard_normal((B, n, s.h, s.dh))
    q_pos = start[:, None] + np.arange(n)[None, :]
    pre = oracle.prefill(s, q, kf, vf, start, q_pos=q_pos)
    for t in range(n):
        dec = oracle.decode(s, q[:, t], kf, vf, start + t + 1, q_pos=start + t)
        _close(pre[:, t], dec, 1e-14, f"prefill row {t} == decode")
    # causal brute force against SDPA with a causal mask
    want = _reference_attention(s, q, q_pos, kf, vf, start[:, None] + np.arange(n)[None, :] + 1,
                                1.0 / math.sqrt(s.dh))
    _close(pre, want, 1e-11, "causal prefill vs SDPA")


# ------------------------------------------------------------------ eq (5)
def check_projection_is_matmul(seed=11):
    rng = np.random.default_rng(seed)
    x, W = rng.standard_normal((7, 33)), rng.standard_normal((20, 33))
    _close(oracle.project(x, W), x @ W.T, 1e-12, "projection")


def check_append_scores_follow_eq9(seed=12):
    """The appended query (rotated, 1/R_Q folded) against an appended key gives the
    factored, relative-position score of eq (9)."""
    rng = np.random.default_rng(seed)
    s = Shape(h1=2, h2=3, d1=2, d2=4, r_k=2, r_v=1, r_q=3, d_model=11, rope_base=10000.0)
    B, n = 1, 4
    x = rng.standard_normal((B, n, s.d_model))
    W = rng.standard_normal((s.n_proj, s.d_model))
    start = np.array([5])
    q_rot, k_rot, v_rec, k_rec = oracle.append(s, x, W, start)
    fac = x[0] @ W.T
    cols = oracle.split_columns(s)
    for t in range(n):
        for u in range(n):
            aq = fac[t, cols[0][0]:cols[0][1]].reshape(s.r_q, s.h1, s.d1)
            bq = fac[t, cols[1][0]:cols[1][1]].reshape(s.r_q, s.h2, s.d2)
            ak = fac[u, cols[2][0]:cols[2][1]].reshape(s.r_k, s.h1, s.d1)
            bk = fac[u, cols[3][0]:cols[3][1]].reshape(s.r_k, s.h2, s.d2)
            Rrel = _rot_matrix_d2(s.d2, s.rope_base, u - t)
            Kpos = oracle.reconstruct(s.h1, s.h2, s.d1, s.d2, s.r_k, k_rot[0, u])
            for i1 in range(s.h1):
                for i2 in range(s.h2):
                    eq9 = sum(float(aq[r, i1] @ ak[rp, i1]) * float(bq[r, i2] @ Rrel @ bk[rp, i2])
                              for r in range(s.r_q) for rp in range(s.r_k)) / (s.r_q * s.r_k)
                    got = float(q_rot[0, t, i1 * s.h2 + i2] @ Kpos[i1 * s.h2 + i2])
                    assert abs(got - eq9) <= 1e-10 * max(1.0, abs(eq9)), f"eq 9 t={t} u={u}: {got} vs {eq9}"
    # values are not rotated; the unrotated key records are the raw columns
    _close(v_rec[0], np.concatenate([fac[:, cols[4][0]:cols[4][1]], fac[:, cols[5][0]:cols[5][1]]], axis=-1),
           1e-12, "value records")
    _close(k_rec[0], np.concatenate([fac[:, cols[2][0]:cols[2][1]], fac[:, cols[3][0]:cols[3][1]]], axis=-1),
           1e-12, "key records")


# ------------------------------------------------------------ eq (10)/(11)
def check_cache_sizes_golden():
    g = _golden("cache_sizes.json")
    for c in g["kpa_compression"]:
        r = oracle.compression(c["h1"], c["h2"], c["d1"], c["d2"], c["r_k"], c["r_v"])
        assert abs(r - c["ratio"]) <= c["tol"], f"{c['cite']}: {r} vs {c['ratio']}"
    for c in g["tpa_numbers_per_token"]:
        n = oracle.cache_numbers_per_token(c["h"], 1, 1, c["dh"], c["r_k"], c["r_v"])
        assert n == c["numbers"], f"{c['cite']}: {n}"
    for c in g["tpa_compression"]:
        r = oracle.compression(c["h"], 1, 1, c["dh"], c["r_k"], c["r_v"])
        assert abs(r - c["ratio"]) <= c["tol"], f"{c['cite']}: {r}"
    for c in g["mha_numbers_per_token"]:
        for (h1, h2) in [(c["h"], 1), (1, c["h"])]:
            n = oracle.mha_numbers_per_token(h1, h2, 1, c["dh"])
            assert n == c["numbers"], f"{c['cite']}: {n}"
    for c in g["tpa_sequence_bytes"]:
        n = oracle.cache_numbers_per_token(c["h"], 1, 1, c["dh"], c["r_k"], c["r_v"])
        mb = n * c["tokens"] * c["bytes_per_number"] / 1e6
        assert abs(mb - c["approx_mb"]) <= c["tol_mb"], f"{c['cite']}: {mb} MB"


def check_shared_b_attention(seed=13):
    """A shared-B cache ("Tensor Product Attention Is All You Need", section 5): the
    factors A^K, A^V and B are drawn as separate arrays, K_t and V_t are formed with
    numpy.kron from the SAME B_r, K_t is rotated with numpy.kron rotation matrices, and
    torch's scaled_dot_product_attention gives the expected output."""
    rng = np.random.default_rng(seed)
    for s in [Shape(h1=16, h2=1, d1=1, d2=8, r_k=2, r_v=2), Shape(h1=2, h2=3, d1=2, d2=4, r_k=3, r_v=3),
              Shape(h1=3, h2=2, d1=4, d2=2, r_k=1, r_v=1, rope_base=500000.0)]:
        B, cap, R = 2, 7, s.r_k
        AK = rng.standard_normal((B, cap, R, s.h1, s.d1))
        AV = rng.standard_normal((B, cap, R, s.h1, s.d1))
        Bf = rng.standard_normal((B, cap, R, s.h2, s.d2))
        q = rng.standard_normal((B, s.h, s.dh))
        q_pos = rng.integers(0, 600000, size=B)
        L = np.array([cap, 4])
        scale = 0.9 / math.sqrt(s.dh)
        kf = np.concatenate([AK.reshape(B, cap, -1), Bf.reshape(B, cap, -1)], axis=2)
        got = oracle.decode_shared_b(s, q, kf, AV.reshape(B, cap, -1), L, q_pos=q_pos, sm_scale=scale)
        K = np.zeros((B, cap, s.h, s.dh)); V = np.zeros((B, cap, s.h, s.dh))
        for b in range(B):
            for t in range(cap):
                rot = np.kron(np.eye(s.d1), _rot_matrix_d2(s.d2, s.rope_base, t))
                K[b, t] = (sum(np.kron(AK[b, t, r], Bf[b, t, r]) for r in range(R)) / R) @ rot.T
                V[b, t] = sum(np.kron(AV[b, t, r], Bf[b, t, r]) for r in range(R)) / R
        Q = np.stack([q[b] @ np.kron(np.eye(s.d1), _rot_matrix_d2(s.d2, s.rope_base, q_pos[b])).T
                      for b in range(B)])
        mask = np.arange(cap)[None, :] < L[:, None]
        want = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(Q)[:, :, None], torch.from_numpy(K).permute(0, 2, 1, 3),
            torch.from_numpy(V).permute(0, 2, 1, 3), attn_mask=torch.from_numpy(mask)[:, None, None],
            scale=scale)[:, :, 0].numpy()
        _close(got, want, 1e-11, f"shared-B attention vs SDPA {s}")
        # one B set instead of two: the unshared count minus R h2 d2
        n = oracle.cache_numbers_per_token_shared_b(s.h1, s.h2, s.d1, s.d2, R)
        assert n == oracle.cache_numbers_per_token(s.h1, s.h2, s.d1, s.d2, R, R) - R * s.h2 * s.d2


def check_order3_attention(seed=14):
    """Third-order TPA ("Tensor Product Attention Is All You Need", Appendix C, as the
    explainer summarises it): a, b and c are drawn as separate arrays; K_t and V_t are
    built with numpy.kron as (1/R) sum_r a_r (x) (b_r (x) c_r); K_t is rotated with the
    block matrix numpy.kron(R_{d_b}(t), I_{d_c}) (RoPE on b, Theorem C.1) and the query
    with numpy.kron(R_{d_b}(q_pos), I_{d_c}); torch's scaled_dot_product_attention gives
    the expected output.  With d_c = 1 the cache is a second-order TPA cache with
    B_r = c_r b_r, and the plain decode of that cache must agree."""
    rng = np.random.default_rng(seed)
    for (h, db, dc, R, base) in [(4, 4, 2, 2, 10000.0), (3, 2, 3, 1, 500000.0), (2, 6, 1, 3, 10000.0)]:
        B, cap = 2, 9
        a = rng.standard_normal((2, B, cap, R, h))
        b = rng.standard_normal((2, B, cap, R, db))
        c = rng.standard_normal((2, B, cap, R, dc))
        q = rng.standard_normal((B, h, db * dc))
        q_pos = rng.integers(0, 600000, size=B)
        L = np.array([cap, 5])
        scale = 1.1 / math.sqrt(db * dc)
        s3 = Shape(h1=h, h2=1, d1=db, d2=dc, r_k=R, r_v=R, rope_base=base, order=3)
        kf = np.concatenate([a[0].reshape(B, cap, -1), b[0].reshape(B, cap, -1), c[0].reshape(B, cap, -1)], axis=2)
        vf = np.concatenate([a[1].reshape(B, cap, -1), b[1].reshape(B, cap, -1), c[1].reshape(B, cap, -1)], axis=2)
        got = oracle.decode_order3(s3, q, kf, vf, L, q_pos=q_pos, sm_scale=scale)
        K = np.zeros((B, cap, h, db * dc)); V = np.zeros((B, cap, h, db * dc))
        for bb in range(B):
            for t in range(cap):
                rot = np.kron(_rot_matrix_d2(db, base, t), np.eye(dc))
                K[bb, t] = (sum(np.kron(a[0, bb, t, r][:, None], np.kron(b[0, bb, t, r], c[0, bb, t, r])[None, :])
                                for r in range(R)) / R) @ rot.T
                V[bb, t] = sum(np.kron(a[1, bb, t, r][:, None], np.kron(b[1, bb, t, r], c[1, bb, t, r])[None, :])
                               for r in range(R)) / R
        Q = np.stack([q[bb] @ np.kron(_rot_matrix_d2(db, base, q_pos[bb]), np.eye(dc)).T for bb in range(B)])
        mask = np.arange(cap)[None, :] < L[:, None]
        want = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(Q)[:, :, None], torch.from_numpy(K).permute(0, 2, 1, 3),
            torch.from_numpy(V).permute(0, 2, 1, 3), attn_mask=torch.from_numpy(mask)[:, None, None],
            scale=scale)[:, :, 0].numpy()
        _close(got, want, 1e-11, f"third-order attention vs SDPA {(h, db, dc, R)}")
        # the rotated cache (b rotated at each slot) read with keys_rotated gives the same
        kr = np.stack([np.stack([oracle.rotate_order3_b(h, db, dc, R, base, t, kf[bb, t]) for t in range(cap)])
                       for bb in range(B)])
        _close(oracle.decode_order3(s3, q, kr, vf, L, q_pos=q_pos, sm_scale=scale, keys_rotated=True), want,
               1e-11, "third-order, keys stored rotated")
        if dc == 1:
            s2 = Shape(h1=h, h2=1, d1=1, d2=db, r_k=R, r_v=R, rope_base=base)
            k2 = np.concatenate([a[0].reshape(B, cap, -1), (b[0] * c[0]).reshape(B, cap, -1)], axis=2)
            v2 = np.concatenate([a[1].reshape(B, cap, -1), (b[1] * c[1]).reshape(B, cap, -1)], axis=2)
            _close(got, oracle.decode(s2, q, k2, v2, L, q_pos=q_pos, sm_scale=scale), 1e-11,
                   "third-order with d_c = 1 is second-order TPA with B = c b")
        # cache size: R (h + d_b + d_c) numbers per key or value record
        assert oracle.cache_numbers_per_token_order3(h, db, dc, R, R) == kf.shape[2] + vf.shape[2]


ALL_CHECKS = [
    check_kron_is_numpy_kron, check_reconstruct_is_kron_sum, check_tpa_split_is_outer_product,
    check_prop22_factored_score, check_rope_golden_frequencies, check_rope_tpa_is_textbook,
    check_rope_kpa_is_identity_kron_rotation, check_thm24_rotating_b_equals_rotating_reconstruction,
    check_relative_position, check_attention_matches_sdpa, check_attention_lse, check_attention_closed_forms,
    check_prefill_rows_are_decodes, check_projection_is_matmul, check_append_scores_follow_eq9,
    check_cache_sizes_golden, check_shared_b_attention, check_order3_attention,
]
