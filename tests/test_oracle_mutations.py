"""Plant one mistake at a time in a copy of the C oracle and check that the pins
catch it (CPU only).  The copies are built in a temporary directory; the
oracle itself is never modified."""
import os

import pytest

import oracle
import pins

# (name, original text, planted mistake)
MUTATIONS = [
    ("rope sign", "v[2 * m + 1] = x0 * s + x1 * c;", "v[2 * m + 1] = -x0 * s + x1 * c;"),
    ("rope frequency index from 1", "-2.0 * (double)m / (double)d2", "-2.0 * (double)(m + 1) / (double)d2"),
    ("rope frequency over d_h", "oracle_rope_d2(d2, base, pos, v + (size_t)j1 * d2);",
     "oracle_rope_d2(d2, base * d1, pos, v + (size_t)j1 * d2);"),
    ("transposed head order", "const int i1 = row / h2, i2 = row % h2;",
     "const int i1 = row % h1, i2 = row / h1;"),
    ("dropped 1/R", "out[j1 * d2 + j2] = acc / (double)R;", "out[j1 * d2 + j2] = acc;"),
    ("dropped rank term", "for (int r = 0; r < R; ++r)\n                acc +=",
     "for (int r = 0; r + 1 < R; ++r)\n                acc +="),
    ("kron block order", "out[(i1 * m2 + i2) * cols + j1 * n2 + j2]", "out[(i2 * m1 + i1) * cols + j1 * n2 + j2]"),
    ("dropped softmax scale", "scores[(size_t)t * max_keys + s] = sm_scale * dot;",
     "scores[(size_t)t * max_keys + s] = dot;"),
    ("key rotated at s+1", "oracle_rope_kpa(d1, d2, rope_base, (double)s, krow);",
     "oracle_rope_kpa(d1, d2, rope_base, (double)(s + 1), krow);"),
    ("softmax range drops the last slot", "for (int s = 0; s < nk; ++s) { row[s] = exp(row[s] - mx); sum += row[s]; }",
     "for (int s = 0; s + 1 < nk; ++s) { row[s] = exp(row[s] - mx); sum += row[s]; }"),
    ("rotate A instead of B", "{\n    double *B = rec + (size_t)R * h1 * d1;", "{\n    double *B = rec;"),
    ("transposed projection", "acc += W[(size_t)n * d_model + k] * x[(size_t)t * d_model + k];",
     "acc += W[(size_t)k * n_out + n] * x[(size_t)t * d_model + k];"),
    ("cache count drops a factor", "return (int64_t)(r_k + r_v) * ((int64_t)h1 * d1 + (int64_t)h2 * d2);",
     "return (int64_t)(r_k + r_v) * ((int64_t)h1 + (int64_t)h2 * d2);"),
    ("value row from the key factors", "oracle_kron_sum_row(h1, h2, d1, d2, r_v, vf + ((size_t)b * cap + s) * ev,",
     "oracle_kron_sum_row(h1, h2, d1, d2, r_v, kf + ((size_t)b * cap + s) * ev,"),
    ("normaliser without the maximum", "if (lrow) *lrow = mx + log(sum);", "if (lrow) *lrow = log(sum);"),
]


@pytest.mark.parametrize("name,orig,bad", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(tmp_path, name, orig, bad):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "kpa_oracle.c")).read()
    assert src.count(orig) == 1, f"mutation anchor for '{name}' not unique"
    mut_src = tmp_path / "mutant.c"
    mut_src.write_text(src.replace(orig, bad))
    lib = oracle.build(force=True, src=str(mut_src), out=str(tmp_path / "libmutant.so"))
    caught = []
    with oracle.use_library(lib):
        for check in pins.ALL_CHECKS:
            try:
                check()
            except (AssertionError, ValueError) as e:
                caught.append(f"{check.__name__}: {str(e)[:80]}")
    assert caught, f"planted mistake '{name}' passed every pin"


def _prefill_without_self(shape, q, kf, vf, start_pos, **kw):
    """A causal rule with a planted mistake: row t sees slots 0 .. start+t-1."""
    q = oracle._f64(q)
    B, n = q.shape[0], q.shape[1]
    start = oracle.np.asarray(start_pos, dtype=oracle.np.int64).reshape(B, 1)
    return oracle.attend(shape, q, kf, vf, start + oracle.np.arange(n)[None, :], **kw)


def test_planted_causal_mistake_is_caught(monkeypatch):
    monkeypatch.setattr(oracle, "prefill", _prefill_without_self)
    with pytest.raises(AssertionError):
        pins.check_prefill_rows_are_decodes()


def _order3_transposed_a_b(h, d_b, d_c, R, rec):
    """A planted mistake: A_r laid out as b_r a_r^T (d_b x h) instead of a_r b_r^T."""
    rec = oracle._f64(rec)
    lead = rec.shape[:-1]
    a = rec[..., :R * h].reshape(lead + (R, h))
    b = rec[..., R * h:R * (h + d_b)].reshape(lead + (R, d_b))
    c = rec[..., R * (h + d_b):].reshape(lead + (R, d_c))
    A = b[..., :, :, None] * a[..., :, None, :]
    return oracle.np.concatenate([A.reshape(lead + (R * h * d_b,)), c.reshape(lead + (R * d_c,))], axis=-1)


_rotate_b = oracle.rotate_order3_b
_rope_q3 = oracle.rope_order3_query


def _order3_key_rotated_one_slot_late(h, d_b, d_c, R, base, pos, rec):
    return _rotate_b(h, d_b, d_c, R, base, pos + 1, rec)


def _order3_query_rotated_on_c(h, d_b, d_c, base, pos, q):
    """A planted mistake: the query's rotation acts on the c index instead of b."""
    q = oracle._f64(q).reshape(h, d_b, d_c).copy()
    if d_c % 2:
        return _rope_q3(h, d_b, d_c, base, pos + 1, q.reshape(h, -1))
    for i in range(h):
        for jb in range(d_b):
            q[i, jb, :] = oracle.rope_d2(d_c, base, pos, q[i, jb, :])
    return q.reshape(h, d_b * d_c)


@pytest.mark.parametrize("attr,bad", [("order3_as_kronecker", _order3_transposed_a_b),
                                      ("rotate_order3_b", _order3_key_rotated_one_slot_late),
                                      ("rope_order3_query", _order3_query_rotated_on_c)],
                         ids=["a and b transposed", "key rotated one slot late", "query rotated on c"])
def test_planted_order3_mistake_is_caught(monkeypatch, attr, bad):
    monkeypatch.setattr(oracle, attr, bad)
    with pytest.raises((AssertionError, ValueError)):
        pins.check_order3_attention()
