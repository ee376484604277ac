"""The tcgen05 TPA decode (h = 16, d_h = 64, R_K = R_V = 2) against the float64
oracle, and against the mma.sync decode on the same inputs (GPU).

`kpa_test_set_decode_engine(1)` sends this shape to the tcgen05 kernel; the
default is the mma.sync kernel.
`kpa_decode_kernel_kind` says which one a call runs."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (assert_bf16_close, errors, fill_cache, kpa, natural, oracle_decode_from_cache,
                      oracle_decode_unrotated, run_decode)
from workloads import TPA_DECODE, decode_inputs, to_f64

pytestmark = pytest.mark.gpu

CASES = {
    # several tiles per split and ragged tails (lengths 1 .. 2048)
    "ragged": TPA_DECODE.replace(batch=5, capacity=2048, length=0, ragged=(1, 2048), seed=41),
    # whole tiles only
    "whole_tiles": TPA_DECODE.replace(batch=2, capacity=1024, length=1024, seed=42),
    # the full-size batch at a short length
    "batch8": TPA_DECODE.replace(batch=8, capacity=1600, length=1543, seed=43),
}


def _run_engines(w, inp, tokens_per_split=0, sm_scale=None):
    lib = kpa()
    cfg, kc, vc = fill_cache(lib, w, inp)
    max_len = int(inp["seq_len"].max().item())
    kinds, outs = [], []
    for engine in (1, 0):
        lib.kpa_test_set_decode_engine(engine)
        try:
            kinds.append(lib.kpa_decode_kernel_kind(cfg, w.batch, max_len, tokens_per_split))
            out = run_decode(lib, w, cfg, kc, vc, inp["q"], inp["seq_len"], inp["q_pos"],
                             tokens_per_split=tokens_per_split, sm_scale=sm_scale)
            torch.cuda.synchronize()
            assert lib.kpa_read_device_error() == 0
        finally:
            lib.kpa_test_set_decode_engine(0)
        outs.append(out.cpu().numpy())
    assert kinds == ["tcgen05", "mma_sync"]
    return kinds[0], outs, kc, vc


@pytest.mark.parametrize("tps", [0, 128, 256, 320, 1024])
@pytest.mark.parametrize("name", sorted(CASES))
def test_tcgen05_decode_matches_oracle_and_mma_sync(name, tps):
    w = CASES[name]
    inp = decode_inputs(w)
    kind, (tc, ms), kc, vc = _run_engines(w, inp, tokens_per_split=tps)
    want = oracle_decode_from_cache(w, kc.cpu(), vc.cpu(), inp["q"], inp["seq_len"], inp["q_pos"])
    assert_bf16_close(tc, want, f"{kind} {name} tps={tps}")
    assert_bf16_close(ms, want, f"mma_sync {name} tps={tps}")
    # both keep the query and P' to ~2^-16 relative (bf16 hi + lo); only the order of
    # the sums differs
    max_abs, rel = errors(tc, ms)
    assert max_abs <= 2e-5 and rel <= 1e-5, f"{kind} vs mma_sync: {max_abs} {rel}"


def test_engine_selection():
    lib = kpa()
    w = TPA_DECODE
    cfg = lib.make_config(w.shape, w.dtype)
    assert lib.kpa_decode_kernel_kind(cfg, w.batch, w.length) == "mma_sync"
    lib.kpa_test_set_decode_engine(1)
    try:
        assert lib.kpa_decode_kernel_kind(cfg, w.batch, w.length) == "tcgen05"
    finally:
        lib.kpa_test_set_decode_engine(0)
    assert lib.kpa_decode_kernel_kind(cfg, w.batch, w.length) == "mma_sync"


@pytest.mark.parametrize("engine", [1, 0], ids=["tcgen05", "mma_sync"])
def test_special_lengths_under_a_fused_plan(engine):
    """L = 0 gives zeros (the kernel merges its own splits here, so no combine pass
    writes them), L = 1 gives V_0, tails at 8k + r and at tile edges."""
    w = TPA_DECODE.replace(batch=8, capacity=1024, length=1024, seed=44)
    inp = decode_inputs(w)
    inp["seq_len"] = torch.tensor([0, 1, 7, 9, 127, 128, 129, 1024], dtype=torch.int32)
    inp["q_pos"] = inp["seq_len"].clone()
    lib = kpa()
    cfg, kc, vc = fill_cache(lib, w, inp)
    lib.kpa_test_set_decode_engine(engine)
    try:
        assert lib.kpa_decode_kernel_kind(cfg, w.batch, 1024) == ("tcgen05" if engine else "mma_sync")
        assert lib.kpa_decode_plan(cfg, w.batch, 1024)[2] == 1          # one launch: fused merge
        out = run_decode(lib, w, cfg, kc, vc, inp["q"], inp["seq_len"], inp["q_pos"], max_len=1024)
        torch.cuda.synchronize()
        assert lib.kpa_read_device_error() == 0
    finally:
        lib.kpa_test_set_decode_engine(0)
    got = out.cpu().numpy()
    assert np.all(got[0] == 0.0)
    s = w.shape
    v0 = oracle.reconstruct(s.h1, s.h2, s.d1, s.d2, s.r_v, to_f64(natural(vc.cpu(), w.batch, w.capacity, s.e_v))[1, 0])
    assert_bf16_close(got[1], v0, "L=1")
    want = oracle_decode_from_cache(w, kc.cpu(), vc.cpu(), inp["q"], inp["seq_len"], inp["q_pos"])
    assert_bf16_close(got[1:], want[1:], "tails")


@pytest.mark.parametrize("mode", ["peaked_q", "zero_q", "prerotated"])
def test_tcgen05_softmax_edges(mode):
    w = CASES["ragged"]
    inp = decode_inputs(w)
    sm_scale = None
    if mode == "peaked_q":
        inp["q"] = inp["q"] * 64                     # exact in bf16: logit gaps far above 10
    elif mode == "zero_q":
        inp["q"] = torch.zeros_like(inp["q"])        # uniform weights: the mean of the values
    else:
        inp["q_pos"] = None                          # the query used as given
    kind, (tc, ms), kc, vc = _run_engines(w, inp, sm_scale=sm_scale)
    assert kind == "tcgen05"
    want = oracle_decode_from_cache(w, kc.cpu(), vc.cpu(), inp["q"], inp["seq_len"], inp["q_pos"])
    assert_bf16_close(tc, want, f"tcgen05 {mode}")
    max_abs, rel = errors(tc, ms)
    assert max_abs <= 2e-5 and rel <= 1e-5, f"tcgen05 vs mma_sync {mode}: {max_abs} {rel}"


def test_tcgen05_end_to_end_and_rerun_is_bitwise():
    w = CASES["batch8"]
    inp = decode_inputs(w)
    lib = kpa()
    cfg, kc, vc = fill_cache(lib, w, inp)
    lib.kpa_test_set_decode_engine(1)
    try:
        assert lib.kpa_decode_kernel_kind(cfg, w.batch, int(inp["seq_len"].max())) == "tcgen05"
        a = run_decode(lib, w, cfg, kc, vc, inp["q"], inp["seq_len"], inp["q_pos"]).cpu().numpy()
        b = run_decode(lib, w, cfg, kc, vc, inp["q"], inp["seq_len"], inp["q_pos"]).cpu().numpy()
        torch.cuda.synchronize()
        assert lib.kpa_read_device_error() == 0
    finally:
        lib.kpa_test_set_decode_engine(0)
    assert np.array_equal(a, b)
    assert_bf16_close(a, oracle_decode_unrotated(w, inp), "tcgen05 end to end")
