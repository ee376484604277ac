"""Third-order TPA (a (x) b (x) c factors, RoPE on b): kpa_append_factors and
kpa_decode against the float64 oracle on the same seeded inputs (GPU)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_close, errors, fill_cache, kpa, natural, run_decode
from workloads import TPA3_DECODE, Shape, decode_inputs, to_f64

pytestmark = pytest.mark.gpu

SMALL = {
    # the benchmark shape at reduced sizes: several tiles and splits, ragged tails
    "h16_8x8": TPA3_DECODE.replace(batch=3, capacity=1024, length=0, ragged=(1, 1024), seed=51),
    # odd c length, three ranks, another RoPE base
    "h12_4x3_r3": TPA3_DECODE.replace(
        shape=Shape(h1=12, h2=1, d1=4, d2=3, r_k=3, r_v=2, rope_base=500000.0, order=3),
        batch=2, capacity=520, length=0, ragged=(1, 520), seed=52),
    # fp32 cache, 32 heads, d_h = 16 x 16 (the largest the kernel takes)
    "f32_h32_16x16": TPA3_DECODE.replace(
        shape=Shape(h1=32, h2=1, d1=16, d2=16, r_k=1, r_v=2, rope_base=10000.0, order=3),
        dtype="f32", batch=2, capacity=200, length=0, ragged=(1, 200), seed=53, factor_std=0.8, q_std=0.1),
}


def _oracle_from_cache(w, kc, vc, inp, sm_scale=None):
    s = w.shape
    kn = to_f64(natural(kc.cpu(), w.batch, w.capacity, s.e_k))
    vn = to_f64(natural(vc.cpu(), w.batch, w.capacity, s.e_v))
    return oracle.decode_order3(s, to_f64(inp["q"]), kn, vn, inp["seq_len"].numpy(),
                                q_pos=inp["q_pos"].numpy(), keys_rotated=True, sm_scale=sm_scale)


def _oracle_unrotated(w, inp, sm_scale=None):
    return oracle.decode_order3(w.shape, to_f64(inp["q"]), to_f64(inp["kf"]), to_f64(inp["vf"]),
                                inp["seq_len"].numpy(), q_pos=inp["q_pos"].numpy(), sm_scale=sm_scale)


def _decode(w, inp, **kw):
    lib = kpa()
    cfg, kc, vc = fill_cache(lib, w, inp)
    out = run_decode(lib, w, cfg, kc, vc, inp["q"], inp["seq_len"], inp["q_pos"], **kw)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    return out.cpu().numpy(), kc, vc


@pytest.mark.parametrize("name", sorted(SMALL))
def test_order3_stage_and_end_to_end(name):
    w = SMALL[name]
    inp = decode_inputs(w)
    got, kc, vc = _decode(w, inp)
    assert_close(w.dtype, got, _oracle_from_cache(w, kc, vc, inp), f"stage {name}")
    assert_close(w.dtype, got, _oracle_unrotated(w, inp), f"end to end {name}")


def test_order3_cache_contents():
    """The keys' b factors are rotated at their slot (bf16 RNE of the float64 rotation,
    within half a bf16 ulp plus fp32 rounding); a, c and the value records bit-exact."""
    w = SMALL["h16_8x8"]
    s = w.shape
    inp = decode_inputs(w)
    lib = kpa()
    cfg = lib.make_config(s, w.dtype)
    assert lib.kpa_cache_bytes_per_token(cfg) == (s.e_k * 2, s.e_v * 2)
    assert s.e_k == s.r_k * (s.h1 + s.d1 + s.d2)
    start = torch.tensor([0, 8, 3], dtype=torch.int32)
    n_tok = 300
    kf, vf = inp["kf"][:, :n_tok].contiguous(), inp["vf"][:, :n_tok].contiguous()
    kc = torch.full((w.batch * w.capacity * s.e_k,), 7.0, dtype=torch.bfloat16, device="cuda")
    vc = torch.full((w.batch * w.capacity * s.e_v,), 7.0, dtype=torch.bfloat16, device="cuda")
    lib.kpa_append_factors(cfg, w.batch, n_tok, kf.cuda(), vf.cuda(), start.cuda(), w.capacity, kc, vc)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    kn = to_f64(natural(kc.cpu(), w.batch, w.capacity, s.e_k))
    vn = to_f64(natural(vc.cpu(), w.batch, w.capacity, s.e_v))
    a, bend = s.r_k * s.h1, s.r_k * (s.h1 + s.d1)
    for b in range(w.batch):
        st = int(start[b])
        assert np.all(kn[b, :st] == 7.0) and np.all(kn[b, st + n_tok:] == 7.0), "wrote outside"
        np.testing.assert_array_equal(vn[b, st:st + n_tok], to_f64(vf[b]))
        for t in range(0, n_tok, 29):
            want = oracle.rotate_order3_b(s.h1, s.d1, s.d2, s.r_k, s.rope_base, st + t, to_f64(kf[b, t]))
            got = kn[b, st + t]
            np.testing.assert_array_equal(got[:a], want[:a])
            np.testing.assert_array_equal(got[bend:], want[bend:])
            assert np.all(np.abs(got - want) <= 2.0 ** -8 * np.abs(want) + 1e-30), f"b={b} t={t}"


def test_order3_special_lengths_and_splits():
    """L = 0 gives zeros, L = 1 gives V_0; several split sizes agree."""
    w = TPA3_DECODE.replace(batch=6, capacity=1024, length=1024, seed=54)
    inp = decode_inputs(w)
    inp["seq_len"] = torch.tensor([0, 1, 7, 33, 129, 1024], dtype=torch.int32)
    inp["q_pos"] = inp["seq_len"].clone()
    lib = kpa()
    cfg, kc, vc = fill_cache(lib, w, inp)
    assert lib.kpa_decode_kernel_kind(cfg, w.batch, 1024) == "mma_sync"   # the d_b = d_c = 8 variant
    outs = []
    for tps in (0, 64, 256, 1024):
        out = run_decode(lib, w, cfg, kc, vc, inp["q"], inp["seq_len"], inp["q_pos"], max_len=1024,
                         tokens_per_split=tps)
        torch.cuda.synchronize()
        assert lib.kpa_read_device_error() == 0
        outs.append(out.cpu().numpy())
    got = outs[0]
    assert np.all(got[0] == 0.0)
    s = w.shape
    vn = to_f64(natural(vc.cpu(), w.batch, w.capacity, s.e_v))
    v0 = oracle.order3_as_kronecker(s.h1, s.d1, s.d2, s.r_v, vn[1, 0])
    v0 = oracle.reconstruct(s.h1, 1, s.d1, s.d2, s.r_v, v0)
    assert_close(w.dtype, got[1], v0, "L=1")
    assert_close(w.dtype, got[1:], _oracle_from_cache(w, kc, vc, inp)[1:], "tails")
    for o in outs[1:]:
        max_abs, rel = errors(o[1:], got[1:])
        assert max_abs <= 2e-5 and rel <= 1e-5, (max_abs, rel)


def test_order3_full_size_sampled_heads():
    """The benchmark configuration (B=8, L=4096) at full size, checked on a sample of
    (sequence, head) pairs that the oracle computes one by one."""
    w = TPA3_DECODE
    inp = decode_inputs(w)
    got, kc, vc = _decode(w, inp)
    s = w.shape
    rng = np.random.default_rng(5)
    flat = rng.choice(w.batch * s.h, size=12, replace=False)
    kn = to_f64(natural(kc.cpu(), w.batch, w.capacity, s.e_k))
    vn = to_f64(natural(vc.cpu(), w.batch, w.capacity, s.e_v))
    want = oracle.decode_order3(s, to_f64(inp["q"]), kn, vn, inp["seq_len"].numpy(), q_pos=inp["q_pos"].numpy(),
                                keys_rotated=True, heads=flat)
    g = got.reshape(w.batch * s.h, -1)[flat]
    wv = want.reshape(w.batch * s.h, -1)[flat]
    assert_close(w.dtype, g, wv, "full size, sampled heads")


@pytest.mark.parametrize("mode", ["peaked_q", "peaked_scale", "zero_q", "prerotated"])
def test_order3_softmax_edges(mode):
    """Logit gaps far above 10 (q x 64, exact in bf16; or sm_scale x 64), a zero query (the
    mean of the values) and a query used as given (q_pos = NULL), on the tensor-core variant
    and on the CUDA-core kernel (another shape).  Stage parity: the oracle reads the cache the
    GPU wrote, so a x64 scale does not also amplify the rounding at the cache write."""
    lib = kpa()
    for w in (SMALL["h16_8x8"], SMALL["h12_4x3_r3"]):
        inp = decode_inputs(w)
        sm_scale = 1.0 / np.sqrt(w.shape.dh)
        if mode == "peaked_q":
            inp["q"] = inp["q"] * 64
        elif mode == "peaked_scale":
            sm_scale *= 64
        elif mode == "zero_q":
            inp["q"] = torch.zeros_like(inp["q"])
        q_pos = None if mode == "prerotated" else inp["q_pos"]
        cfg, kc, vc = fill_cache(lib, w, inp)
        out = run_decode(lib, w, cfg, kc, vc, inp["q"], inp["seq_len"], q_pos, sm_scale=float(sm_scale))
        torch.cuda.synchronize()
        assert lib.kpa_read_device_error() == 0
        s = w.shape
        kn = to_f64(natural(kc.cpu(), w.batch, w.capacity, s.e_k))
        vn = to_f64(natural(vc.cpu(), w.batch, w.capacity, s.e_v))
        want = oracle.decode_order3(s, to_f64(inp["q"]), kn, vn, inp["seq_len"].numpy(),
                                    q_pos=None if q_pos is None else q_pos.numpy(), keys_rotated=True,
                                    sm_scale=sm_scale)
        assert_close(w.dtype, out.cpu().numpy(), want, f"{mode} {w.shape}")
