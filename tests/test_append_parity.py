"""kpa_append (merged projection on tcgen05, factor RoPE, cache write, query
assembly) against the float64 oracle (GPU).

The oracle takes the same bf16 x and W upcast exactly to float64.  The GPU rounds
at the two documented storage points (the cache write and q_out), so each stored
value must match the oracle within half a bf16 ulp plus the fp32 accumulation error
of the projection."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import kpa, natural, planes
from workloads import APPEND_PREFILL, append_inputs, to_f64

pytestmark = pytest.mark.gpu


def _close_bf16(got, want, what):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    scale = np.abs(want).max()
    bad = np.abs(got - want) > 2.0 ** -8 * np.abs(want) + 1e-5 * max(scale, 1.0)
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} values off, worst "
                           f"{np.abs(got - want).max():.3e}")


def _run_append(lib, w, inp, start, n_tok=None):
    s = w.shape
    n_tok = w.n_tok if n_tok is None else n_tok
    cfg = lib.make_config(s, "bf16")
    kc, vc = planes(s, w.batch, w.capacity, "bf16")
    ws = torch.zeros(max(lib.kpa_append_workspace_size(cfg, w.batch, n_tok), 256), dtype=torch.uint8,
                     device="cuda")
    q_out = torch.full((w.batch, n_tok, s.h, s.dh), float("nan"), dtype=torch.bfloat16, device="cuda")
    lib.kpa_append(cfg, w.batch, n_tok, inp["x"].cuda().contiguous(), inp["W"].cuda().contiguous(),
                   start.cuda(), w.capacity, kc, vc, q_out, ws)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    return cfg, kc, vc, q_out


SMALL = APPEND_PREFILL.replace(batch=2, n_tok=300, capacity=512, seed=3)
SMALL_SHAPE = SMALL.shape.__class__(h1=4, h2=4, d1=8, d2=16, r_k=2, r_v=2, r_q=6, d_model=256,
                                    rope_base=10000.0)


def test_append_small_against_oracle():
    w = SMALL.replace(shape=SMALL_SHAPE)
    s = w.shape
    inp = append_inputs(w)
    start = torch.tensor([0, 77], dtype=torch.int32)
    lib = kpa()
    _, kc, vc, q_out = _run_append(lib, w, inp, start)
    q_rot, k_rot, v_rec, _ = oracle.append(s, to_f64(inp["x"]), to_f64(inp["W"]), start.numpy())
    kn = to_f64(natural(kc.cpu(), w.batch, w.capacity, s.e_k))
    vn = to_f64(natural(vc.cpu(), w.batch, w.capacity, s.e_v))
    for b in range(w.batch):
        st = int(start[b])
        _close_bf16(kn[b, st:st + w.n_tok], k_rot[b], f"key cache b={b}")
        _close_bf16(vn[b, st:st + w.n_tok], v_rec[b], f"value cache b={b}")
        assert np.all(kn[b, :st] == 0) and np.all(kn[b, st + w.n_tok:] == 0), "wrote outside its slots"
    _close_bf16(to_f64(q_out.cpu()), q_rot, "assembled query")


# Query assembly at other shapes: TPA-like (d1 = 1) with R_Q = 4, R_Q = 1 and 8 (the
# staged kernel's other instantiations), R_Q = 3 (no instantiation: the generic
# kernel), and a B^Q block that starts off a 16-byte boundary (R_Q*h1*d1 = 6).
OTHER_SHAPES = {
    "tpa_rq4": dict(h1=8, h2=1, d1=1, d2=64, r_k=2, r_v=2, r_q=4),
    "kpa_rq1": dict(h1=2, h2=4, d1=4, d2=16, r_k=1, r_v=1, r_q=1),
    "kpa_rq8": dict(h1=4, h2=2, d1=2, d2=32, r_k=2, r_v=1, r_q=8),
    "kpa_rq3": dict(h1=2, h2=4, d1=4, d2=16, r_k=2, r_v=2, r_q=3),
    "unaligned": dict(h1=3, h2=2, d1=1, d2=16, r_k=2, r_v=2, r_q=2),
}


@pytest.mark.parametrize("name", list(OTHER_SHAPES))
def test_append_query_assembly_other_shapes(name):
    s = SMALL_SHAPE.__class__(d_model=128, rope_base=10000.0, **OTHER_SHAPES[name])
    w = SMALL.replace(shape=s, n_tok=53, capacity=128)
    inp = append_inputs(w)
    start = torch.tensor([8, 0], dtype=torch.int32)
    lib = kpa()
    _, kc, vc, q_out = _run_append(lib, w, inp, start)
    q_rot, k_rot, v_rec, _ = oracle.append(s, to_f64(inp["x"]), to_f64(inp["W"]), start.numpy())
    kn = to_f64(natural(kc.cpu(), w.batch, w.capacity, s.e_k))
    vn = to_f64(natural(vc.cpu(), w.batch, w.capacity, s.e_v))
    for b in range(w.batch):
        st = int(start[b])
        _close_bf16(kn[b, st:st + w.n_tok], k_rot[b], f"{name} key cache b={b}")
        _close_bf16(vn[b, st:st + w.n_tok], v_rec[b], f"{name} value cache b={b}")
    _close_bf16(to_f64(q_out.cpu()), q_rot, f"{name} assembled query")


def test_append_full_config_sampled_tokens():
    """Configuration 5 at full size (B=8, 2048 tokens, d_model 2048, R_Q=6): sampled
    tokens of the cache and of q_out checked one by one."""
    w = APPEND_PREFILL
    s = w.shape
    inp = append_inputs(w)
    start = inp["start_pos"]
    lib = kpa()
    _, kc, vc, q_out = _run_append(lib, w, inp, start)
    rng = np.random.default_rng(11)
    picks = [(int(b), int(t)) for b, t in zip(rng.integers(0, w.batch, 24), rng.integers(0, w.n_tok, 24))]
    picks += [(0, 0), (w.batch - 1, w.n_tok - 1), (3, 127), (3, 128)]
    kn = natural(kc, w.batch, w.capacity, s.e_k)
    vn = natural(vc, w.batch, w.capacity, s.e_v)
    W = to_f64(inp["W"])
    for b, t in picks:
        pos = int(start[b]) + t
        q_rot, k_rot, v_rec, _ = oracle.append(s, to_f64(inp["x"][b:b + 1, t:t + 1]), W, [pos])
        _close_bf16(to_f64(kn[b, pos].cpu()), k_rot[0, 0], f"key ({b},{t})")
        _close_bf16(to_f64(vn[b, pos].cpu()), v_rec[0, 0], f"value ({b},{t})")
        _close_bf16(to_f64(q_out[b, t].cpu()), q_rot[0, 0], f"query ({b},{t})")


def test_append_without_query_and_out_of_range_slot():
    w = SMALL.replace(shape=SMALL_SHAPE, batch=2, n_tok=20, capacity=64)
    s = w.shape
    inp = append_inputs(w)
    lib = kpa()
    cfg = lib.make_config(s, "bf16")
    kc, vc = planes(s, w.batch, w.capacity, "bf16")
    start = torch.tensor([0, 50], dtype=torch.int32, device="cuda")   # sequence 1 runs past 64
    lib.kpa_append(cfg, w.batch, w.n_tok, inp["x"].cuda(), inp["W"].cuda(), start, w.capacity, kc, vc,
                   None, None)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == lib.KPA_ERR_DEVICE_CHECK
    _, k_rot, _, _ = oracle.append(s, to_f64(inp["x"]), to_f64(inp["W"]), [0, 50])
    kn = to_f64(natural(kc.cpu(), w.batch, w.capacity, s.e_k))
    _close_bf16(kn[0, :20], k_rot[0], "sequence 0")
    _close_bf16(kn[1, 50:64], k_rot[1, :14], "sequence 1, slots inside the cache")


def test_append_few_tokens_against_oracle():
    """A decode-sized append (batch 3 x 5 tokens: the matrix-vector path) against the
    oracle, at start positions that are not multiples of the cache group."""
    w = SMALL.replace(shape=SMALL_SHAPE, batch=3, n_tok=5, capacity=64, seed=9)
    s = w.shape
    inp = append_inputs(w)
    start = torch.tensor([0, 13, 58], dtype=torch.int32)
    lib = kpa()
    _, kc, vc, q_out = _run_append(lib, w, inp, start)
    q_rot, k_rot, v_rec, _ = oracle.append(s, to_f64(inp["x"]), to_f64(inp["W"]), start.numpy())
    kn = to_f64(natural(kc.cpu(), w.batch, w.capacity, s.e_k))
    vn = to_f64(natural(vc.cpu(), w.batch, w.capacity, s.e_v))
    for b in range(w.batch):
        st = int(start[b])
        _close_bf16(kn[b, st:st + w.n_tok], k_rot[b], f"key cache b={b}")
        _close_bf16(vn[b, st:st + w.n_tok], v_rec[b], f"value cache b={b}")
        assert np.all(kn[b, :st] == 0) and np.all(kn[b, st + w.n_tok:] == 0), "wrote outside its slots"
    _close_bf16(to_f64(q_out.cpu()), q_rot, "assembled query")
