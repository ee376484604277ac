"""kpa_append_factors + kpa_decode against the float64 oracle on the same seeded
inputs (GPU).  Two levels:

* stage parity -- the oracle reads back the exact bf16 values the GPU cache
  holds (B^K already rotated, keys_rotated=True), so only the decode kernel's
  arithmetic is measured;
* end to end -- the oracle takes the unrotated records and applies RoPE to the
  reconstruction (the plain definition); the difference then also contains the
  bf16 rounding of the rotated B^K at the cache write.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (assert_bf16_close, assert_close, assert_f32_close, errors, fill_cache, kpa,
                      natural, oracle_decode_from_cache, oracle_decode_unrotated, run_decode)
from workloads import FLASHTPA_DECODE, KPA_LONG, KPA_MEDIUM, TINY_KPA, TPA_DECODE, Shape, decode_inputs, to_f64

pytestmark = pytest.mark.gpu

# Reduced cases: several tiles and splits, ragged tails, oracle in seconds.
SMALL = {
    "tpa": TPA_DECODE.replace(batch=3, capacity=1024, length=0, ragged=(1, 1024), seed=1),
    "kpa_medium": KPA_MEDIUM.replace(batch=4, capacity=1536, ragged=(1, 1536), seed=2),
    "kpa_long_base": KPA_LONG.replace(capacity=4104, length=4101, seed=3),
    "tiny_kpa_scaled": TINY_KPA.replace(factor_std=1.0 / np.sqrt(2.0), seed=4),
    "flashtpa": FLASHTPA_DECODE.replace(batch=3, capacity=1536, length=0, ragged=(1, 1536), seed=6),
    "tpa_h61": __import__("workloads").TPA_H61_DECODE.replace(batch=3, capacity=1024, length=0, ragged=(1, 1024),
                                                             seed=7),
    "kpa_odd": KPA_MEDIUM.replace(shape=KPA_MEDIUM.shape.__class__(h1=3, h2=2, d1=2, d2=6, r_k=3,
                                                                   r_v=1, rope_base=10000.0),
                                  batch=2, capacity=200, ragged=(1, 200), seed=5),
}


def _run(w, inp, **kw):
    lib = kpa()
    cfg, kc, vc = fill_cache(lib, w, inp)
    out = run_decode(lib, w, cfg, kc, vc, inp["q"], inp["seq_len"], inp["q_pos"], **kw)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    return out.cpu().numpy(), kc, vc


def test_tiny_kpa_fp32_as_specified():
    """Configuration 1 exactly: fp32, B=1, h=2x4, d_h=8x8, R=2+2, L=256, q at 256."""
    w = TINY_KPA
    inp = decode_inputs(w)
    got, _, _ = _run(w, inp)
    assert_f32_close(got, oracle_decode_unrotated(w, inp), "tiny KPA fp32")


@pytest.mark.parametrize("name", sorted(SMALL))
def test_stage_parity(name):
    w = SMALL[name]
    inp = decode_inputs(w)
    got, kc, vc = _run(w, inp)
    want = oracle_decode_from_cache(w, kc.cpu(), vc.cpu(), inp["q"], inp["seq_len"], inp["q_pos"])
    assert_close(w.dtype, got, want, f"stage {name}")


@pytest.mark.parametrize("name", sorted(SMALL))
def test_end_to_end(name):
    w = SMALL[name]
    inp = decode_inputs(w)
    got, _, _ = _run(w, inp)
    assert_close(w.dtype, got, oracle_decode_unrotated(w, inp), f"e2e {name}")


@pytest.mark.parametrize("name", ["tpa", "kpa_medium"])
@pytest.mark.parametrize("mode", ["peaked_q", "peaked_scale"])
def test_peaked_softmax(name, mode):
    """Max logit gap far above 10: q x 64 (exact in bf16) or sm_scale x 64."""
    w = SMALL[name]
    inp = decode_inputs(w)
    scale = 1.0 / np.sqrt(w.shape.dh)
    if mode == "peaked_q":
        inp["q"] = inp["q"] * 64
    else:
        scale *= 64
    got, kc, vc = _run(w, inp, sm_scale=float(scale))
    want = oracle_decode_from_cache(w, kc.cpu(), vc.cpu(), inp["q"], inp["seq_len"], inp["q_pos"],
                                    sm_scale=scale)
    assert_close(w.dtype, got, want, f"peaked {name} {mode}")


def test_special_lengths():
    """L=0 gives zeros, L=1 gives V_0 exactly (up to fp32), L=8k+r tails."""
    w = SMALL["kpa_medium"].replace(batch=6, ragged=(), length=1)
    inp = decode_inputs(w.replace(length=1536))
    inp["seq_len"] = torch.tensor([0, 1, 7, 9, 64, 1536], dtype=torch.int32)
    inp["q_pos"] = inp["seq_len"].clone()
    lib = kpa()
    cfg, kc, vc = fill_cache(lib, w, inp)
    out = run_decode(lib, w, cfg, kc, vc, inp["q"], inp["seq_len"], inp["q_pos"], max_len=1536)
    got = out.cpu().numpy()
    assert np.all(got[0] == 0.0)
    v0 = oracle.reconstruct(w.shape.h1, w.shape.h2, w.shape.d1, w.shape.d2, w.shape.r_v,
                            to_f64(natural(vc.cpu(), w.batch, w.capacity, w.shape.e_v))[1, 0])
    assert_bf16_close(got[1], v0, "L=1")
    want = oracle_decode_from_cache(w, kc.cpu(), vc.cpu(), inp["q"], inp["seq_len"], inp["q_pos"])
    assert_bf16_close(got[1:], want[1:], "ragged tails")


def test_cuda_core_kernel_short_splits():
    """The CUDA-core kernel's own plan splits short sequences down to 16 slots (the fp32
    configuration: 256 slots over 16 CTAs).  Tails around a split's end and the last
    split's absorbed remainder (up to a quarter of a split) against the oracle in fp32,
    and against a user split of 64 slots."""
    w = TINY_KPA.replace(batch=10, seed=8)
    inp = decode_inputs(w)
    inp["seq_len"] = torch.tensor([0, 1, 15, 16, 17, 20, 21, 33, 100, 256], dtype=torch.int32)
    inp["q_pos"] = inp["seq_len"].clone()
    lib = kpa()
    cfg, kc, vc = fill_cache(lib, w, inp)
    assert lib.kpa_decode_kernel_kind(cfg, w.batch, 256) == "cuda_cores"
    n_split, tps, _ = lib.kpa_decode_plan(cfg, 1, 256)
    assert (n_split, tps) == (16, 16)
    outs = []
    for split in (0, 64):
        out = run_decode(lib, w, cfg, kc, vc, inp["q"], inp["seq_len"], inp["q_pos"], max_len=256,
                         tokens_per_split=split)
        torch.cuda.synchronize()
        assert lib.kpa_read_device_error() == 0
        outs.append(out.cpu().numpy())
    assert np.all(outs[0][0] == 0.0)
    want = oracle_decode_from_cache(w, kc.cpu(), vc.cpu(), inp["q"], inp["seq_len"], inp["q_pos"])
    assert_f32_close(outs[0][1:], want[1:], "16-slot splits")
    assert_f32_close(outs[1][1:], want[1:], "64-slot splits")


def test_zero_query_gives_the_mean():
    w = SMALL["tpa"]
    inp = decode_inputs(w)
    inp["q"] = torch.zeros_like(inp["q"])
    got, kc, vc = _run(w, inp)
    want = oracle_decode_from_cache(w, kc.cpu(), vc.cpu(), inp["q"], inp["seq_len"], inp["q_pos"])
    assert_bf16_close(got, want, "q = 0")


def test_prerotated_query():
    """q_pos == NULL: the query is used as given."""
    w = SMALL["kpa_medium"]
    inp = decode_inputs(w)
    lib = kpa()
    cfg, kc, vc = fill_cache(lib, w, inp)
    out = run_decode(lib, w, cfg, kc, vc, inp["q"], inp["seq_len"], None)
    want = oracle_decode_from_cache(w, kc.cpu(), vc.cpu(), inp["q"], inp["seq_len"], None)
    assert_bf16_close(out.cpu().numpy(), want, "q_pos NULL")


@pytest.mark.parametrize("name", ["tpa", "kpa_medium"])
def test_split_invariance_and_determinism(name):
    w = SMALL[name]
    inp = decode_inputs(w)
    lib = kpa()
    cfg, kc, vc = fill_cache(lib, w, inp)
    outs = {}
    for tps in (0, 64, 128, 448, 1536):
        outs[tps] = run_decode(lib, w, cfg, kc, vc, inp["q"], inp["seq_len"], inp["q_pos"],
                               tokens_per_split=tps).cpu().numpy()
    ref = outs[0]
    # Plans differ only in summation order, except that the d1 = 8 decode rounds each
    # P' = p A^V once to fp16 (relative 2^-11) against a running maximum that depends on
    # the plan.  Those roundings are independent per term, so two plans then agree to
    # about 2^-12 of the output's norm (times a small factor from the terms' spread):
    # 1e-3 relative.  Every other path keeps an exact bf16 hi + lo pair: 1e-5.
    fp16_values = w.shape.d1 == 8 and not w.shape.shared_b and w.shape.order != 3
    rel_tol = 1e-3 if fp16_values else 1e-5
    for tps, o in outs.items():
        max_abs, rel = errors(o, ref)
        assert max_abs <= 2e-5 and rel <= rel_tol, f"split {tps}: {max_abs} {rel}"
    again = run_decode(lib, w, cfg, kc, vc, inp["q"], inp["seq_len"], inp["q_pos"]).cpu().numpy()
    assert np.array_equal(again, ref), "rerun with the same split is not bitwise equal"


def test_append_factors_cache_contents():
    """The cache holds B^K rotated at its slot (bf16 RNE of the float64 rotation,
    within half a bf16 ulp plus fp32 rounding) and everything else bit-exact."""
    w = SMALL["kpa_medium"]
    s = w.shape
    inp = decode_inputs(w)
    lib = kpa()
    start = torch.tensor([0, 8, 3, 100], dtype=torch.int32)
    n_tok = 512
    kf, vf = inp["kf"][:, :n_tok].contiguous(), inp["vf"][:, :n_tok].contiguous()
    cfg = lib.make_config(s, w.dtype)
    kc = torch.full((w.batch * w.capacity * s.e_k,), 7.0, dtype=torch.bfloat16, device="cuda")
    vc = torch.full((w.batch * w.capacity * s.e_v,), 7.0, dtype=torch.bfloat16, device="cuda")
    lib.kpa_append_factors(cfg, w.batch, n_tok, kf.cuda(), vf.cuda(), start.cuda(), w.capacity, kc, vc)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    kn = to_f64(natural(kc.cpu(), w.batch, w.capacity, s.e_k))
    vn = to_f64(natural(vc.cpu(), w.batch, w.capacity, s.e_v))
    a = s.r_k * s.h1 * s.d1
    for b in range(w.batch):
        st = int(start[b])
        assert np.all(kn[b, :st] == 7.0) and np.all(kn[b, st + n_tok:] == 7.0), "wrote outside"
        assert np.all(vn[b, :st] == 7.0) and np.all(vn[b, st + n_tok:] == 7.0), "wrote outside"
        np.testing.assert_array_equal(vn[b, st:st + n_tok], to_f64(vf[b]))
        for t in range(0, n_tok, 37):
            want = oracle.rotate_record(s.h1, s.h2, s.d1, s.d2, s.r_k, s.rope_base, st + t, to_f64(kf[b, t]))
            got = kn[b, st + t]
            np.testing.assert_array_equal(got[:a], want[:a])
            assert np.all(np.abs(got - want) <= 2.0 ** -8 * np.abs(want) + 1e-30), f"b={b} t={t}"


def test_device_checks_set_the_error_word():
    """A length above max_len is clamped and reported; an append outside the
    cache is skipped and reported.  Nothing faults."""
    w = SMALL["tpa"]
    inp = decode_inputs(w)
    lib = kpa()
    cfg, kc, vc = fill_cache(lib, w, inp)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    seq = inp["seq_len"].clone()
    max_len = int(seq.max()) - 5
    out = run_decode(lib, w, cfg, kc, vc, inp["q"], seq, inp["q_pos"], max_len=max_len)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == lib.KPA_ERR_DEVICE_CHECK
    assert lib.kpa_read_device_error() == 0          # cleared by the read
    clamped = torch.clamp(seq, max=max_len)
    want = oracle_decode_from_cache(w, kc.cpu(), vc.cpu(), inp["q"], clamped, inp["q_pos"])
    assert_bf16_close(out.cpu().numpy(), want, "clamped")
    before = kc.clone()
    bad_start = torch.tensor([w.capacity - 2, -3, 0], dtype=torch.int32, device="cuda")
    lib.kpa_append_factors(cfg, w.batch, 4, inp["kf"][:, :4].contiguous().cuda(),
                           inp["vf"][:, :4].contiguous().cuda(), bad_start, w.capacity, kc, vc)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == lib.KPA_ERR_DEVICE_CHECK
    kn_before = natural(before, w.batch, w.capacity, w.shape.e_k)
    kn_after = natural(kc, w.batch, w.capacity, w.shape.e_k)
    # in-range slots were written, nothing else changed
    assert torch.equal(kn_before[0, : w.capacity - 2], kn_after[0, : w.capacity - 2])
    assert torch.equal(kn_before[1, 1:], kn_after[1, 1:])


# --------------------------------------------------------- full-size configs
def _sample_heads(w, seq_len, n=6, seed=0):
    rng = np.random.default_rng(seed)
    L = seq_len.numpy()
    bs = sorted({int(np.argmax(L)), int(np.argmin(L))} | set(rng.integers(0, w.batch, n).tolist()))
    return sorted({b * w.shape.h + int(rng.integers(0, w.shape.h)) for b in bs} |
                  {bs[0] * w.shape.h, bs[-1] * w.shape.h + w.shape.h - 1})


@pytest.mark.parametrize("w", [TPA_DECODE, KPA_MEDIUM, KPA_LONG, FLASHTPA_DECODE], ids=lambda w: w.name.split(" (")[0])
def test_full_size_sampled_heads(w):
    """The full configurations in the launch configuration the benchmark uses,
    checked end to end on sampled (sequence, head) outputs."""
    inp = decode_inputs(w)
    got, _, _ = _run(w, inp)
    heads = _sample_heads(w, inp["seq_len"])
    want = oracle_decode_unrotated(w, inp, heads=heads)
    idx = [(f // w.shape.h, f % w.shape.h) for f in heads]
    g = np.stack([got[b, hd] for b, hd in idx])
    o = np.stack([want[b, hd] for b, hd in idx])
    assert_bf16_close(g, o, w.name)


def _qf_case(shape, batch, cap, seed):
    w = KPA_MEDIUM.replace(shape=shape, batch=batch, capacity=cap, ragged=(1, cap), seed=seed)
    inp = decode_inputs(w)
    rng = np.random.default_rng(seed + 100)
    qf = (rng.standard_normal((batch, shape.e_q)) / np.sqrt(shape.r_q)).astype(np.float32)
    return w, inp, qf


@pytest.mark.parametrize("shape", [
    Shape(h1=4, h2=4, d1=8, d2=16, r_k=2, r_v=2, r_q=6, d_model=2048, rope_base=10000.0),
    Shape(h1=16, h2=1, d1=1, d2=64, r_k=2, r_v=2, r_q=4, d_model=1024, rope_base=10000.0),
    Shape(h1=16, h2=1, d1=1, d2=128, r_k=2, r_v=2, r_q=6, d_model=2048, rope_base=10000.0),
    Shape(h1=4, h2=4, d1=8, d2=16, r_k=4, r_v=4, r_q=6, d_model=2048, rope_base=10000.0)],
    ids=["kpa_h4x4", "tpa_h16", "tpa_h16_d128", "kpa_h4x4_r4"])
def test_decode_from_query_factors(shape):
    """kpa_decode_qf: the query as factor records (record layout), rotated in the kernel at
    q_pos, against the oracle with the float64 assembly (1/R_Q) sum_r A^Q_r (x) B^Q_r."""
    w, inp, qf = _qf_case(shape, 3, 1024, 51)
    lib = kpa()
    cfg, kc, vc = fill_cache(lib, w, inp)
    L = inp["seq_len"]
    max_len = int(L.max())
    ws = torch.zeros(lib.kpa_decode_workspace_size(cfg, w.batch, max_len), dtype=torch.uint8, device="cuda")
    out = torch.full((w.batch, shape.h, shape.dh), float("nan"), dtype=torch.float32, device="cuda")
    scale = 1.0 / np.sqrt(shape.dh)
    lib.kpa_decode_qf(cfg, w.batch, torch.from_numpy(qf).cuda(), 1, shape.e_q, inp["q_pos"].cuda(), kc, vc,
                      w.capacity, L.cuda(), max_len, scale, out, ws)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    q_dense = np.stack([oracle.reconstruct(shape.h1, shape.h2, shape.d1, shape.d2, shape.r_q, qf[b].astype(np.float64))
                        for b in range(w.batch)])
    want = oracle_decode_unrotated(w, inp, q=torch.from_numpy(q_dense), sm_scale=scale)
    assert_bf16_close(out.cpu().numpy(), want, f"decode from query factors {shape}")


def test_decode_step_reads_the_appends_query_factors():
    """A one-token kpa_append (no q_out) followed by kpa_decode_qf on the append's
    workspace ([E_Q][batch] fp32, B^Q rotated): equal to the oracle's append + decode."""
    from workloads import APPEND_PREFILL, append_inputs
    w = APPEND_PREFILL.replace(batch=3, n_tok=1, capacity=512, seed=52)
    s = w.shape
    lib = kpa()
    cfg = lib.make_config(s, "bf16")
    # earlier context in the cache, then the new token at position start = 300 + b
    ctx = KPA_MEDIUM.replace(shape=s, batch=w.batch, capacity=w.capacity, ragged=(), length=w.capacity, seed=53)
    cinp = decode_inputs(ctx)
    cfg2, kc, vc = fill_cache(lib, ctx, cinp)
    inp = append_inputs(w)
    start = torch.tensor([300, 301, 302], dtype=torch.int32)
    ws = torch.zeros(max(lib.kpa_append_workspace_size(cfg, w.batch, 1), 256), dtype=torch.uint8, device="cuda")
    lib.kpa_append(cfg, w.batch, 1, inp["x"].cuda(), inp["W"].cuda(), start.cuda(), w.capacity, kc, vc, None, ws)
    L = start + 1
    wsd = torch.zeros(lib.kpa_decode_workspace_size(cfg, w.batch, int(L.max())), dtype=torch.uint8, device="cuda")
    out = torch.full((w.batch, s.h, s.dh), float("nan"), dtype=torch.float32, device="cuda")
    scale = 1.0 / np.sqrt(s.dh)
    lib.kpa_decode_qf(cfg, w.batch, ws.view(torch.float32), w.batch, 1, None, kc, vc, w.capacity, L.cuda(),
                      int(L.max()), scale, out, wsd)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    q_rot, _, _, _ = oracle.append(s, to_f64(inp["x"]), to_f64(inp["W"]), start.numpy())
    kn = to_f64(natural(kc.cpu(), w.batch, w.capacity, s.e_k))
    vn = to_f64(natural(vc.cpu(), w.batch, w.capacity, s.e_v))
    want = oracle.decode(s, q_rot[:, 0], kn, vn, L.numpy(), keys_rotated=True, sm_scale=scale)
    assert_bf16_close(out.cpu().numpy(), want, "decode step from the append's query factors")


@pytest.mark.parametrize("name", sorted(__import__("workloads").KPA_SECTION32))
def test_section32_head_splits(name):
    """The six head splits of the KPA paper's section 3.2 (d1 = d2 = 8, R = 2; h = 4x4,
    2x8, 8x2, 4x5, 2x10, 10x2) run on the tensor cores, and match the oracle end to end
    (RoPE on the reconstruction) and at stage level, on ragged lengths over several
    tiles and splits; with a peaked softmax (scale x 64) at stage level, where the
    oracle reads the cache's own bf16 values (end to end, the bf16 rounding of the
    rotated keys would be amplified 64 times)."""
    from workloads import KPA_SECTION32
    lib = kpa()
    w = KPA_SECTION32[name].replace(batch=3, capacity=1200, length=0, ragged=(1, 1200), seed=61)
    inp = decode_inputs(w)
    cfg = lib.make_config(w.shape, w.dtype)
    max_len = int(inp["seq_len"].max())
    assert lib.kpa_decode_kernel_kind(cfg, w.batch, max_len) == "mma_sync"
    got, kc, vc = _run(w, inp)
    assert_bf16_close(got, oracle_decode_unrotated(w, inp), f"e2e {name}")
    want = oracle_decode_from_cache(w, kc.cpu(), vc.cpu(), inp["q"], inp["seq_len"], inp["q_pos"])
    assert_bf16_close(got, want, f"stage {name}")
    scale = 64.0 / np.sqrt(w.shape.dh)
    got, kc, vc = _run(w, inp, sm_scale=float(scale))
    want = oracle_decode_from_cache(w, kc.cpu(), vc.cpu(), inp["q"], inp["seq_len"], inp["q_pos"],
                                    sm_scale=scale)
    assert_bf16_close(got, want, f"peaked {name}")


# The append+prefill configuration's h = 16, d_h = 128 in its TPA split and at rank 4:
# the tensor-core decode variants that take those splits' decode steps.
SPLIT_DECODES = {
    "tpa_h16_d1x128_r2": Shape(h1=16, h2=1, d1=1, d2=128, r_k=2, r_v=2),
    "kpa_h4x4_d8x16_r4": Shape(h1=4, h2=4, d1=8, d2=16, r_k=4, r_v=4),
}


@pytest.mark.parametrize("name", sorted(SPLIT_DECODES))
def test_more_split_decodes(name):
    """The TPA split of h = 16, d_h = 128 (1152-byte records, 64 tokens a stage) and the
    KPA split at rank 4 run on the tensor cores and match the oracle end to end, at stage
    level, and with a peaked softmax (scale x 64) at stage level, on ragged lengths."""
    lib = kpa()
    w = KPA_MEDIUM.replace(shape=SPLIT_DECODES[name], batch=3, capacity=1200, length=0, ragged=(1, 1200),
                           factor_std=1.0 / np.sqrt(2.0), seed=62)
    inp = decode_inputs(w)
    cfg = lib.make_config(w.shape, w.dtype)
    max_len = int(inp["seq_len"].max())
    assert lib.kpa_decode_kernel_kind(cfg, w.batch, max_len) == "mma_sync"
    got, kc, vc = _run(w, inp)
    assert_bf16_close(got, oracle_decode_unrotated(w, inp), f"e2e {name}")
    want = oracle_decode_from_cache(w, kc.cpu(), vc.cpu(), inp["q"], inp["seq_len"], inp["q_pos"])
    assert_bf16_close(got, want, f"stage {name}")
    scale = 64.0 / np.sqrt(w.shape.dh)
    got, kc, vc = _run(w, inp, sm_scale=float(scale))
    want = oracle_decode_from_cache(w, kc.cpu(), vc.cpu(), inp["q"], inp["seq_len"], inp["q_pos"],
                                    sm_scale=scale)
    assert_bf16_close(got, want, f"peaked {name}")


def test_tpa_h61_on_the_tensor_cores():
    """The TPA explainer's 773M model, h = 61, d_h = 64, R = 2 (500 numbers per token):
    61 heads padded to four 16-row tiles split over four warps of a token slice; the
    padded query rows are zero and the 61 heads' outputs match the oracle end to end,
    at stage level and with a peaked softmax, on ragged lengths over several tiles."""
    from workloads import TPA_H61_DECODE
    lib = kpa()
    w = TPA_H61_DECODE.replace(batch=3, capacity=1200, length=0, ragged=(1, 1200), seed=63)
    inp = decode_inputs(w)
    cfg = lib.make_config(w.shape, w.dtype)
    assert lib.kpa_decode_kernel_kind(cfg, w.batch, int(inp["seq_len"].max())) == "mma_sync"
    got, kc, vc = _run(w, inp)
    assert_bf16_close(got, oracle_decode_unrotated(w, inp), "e2e tpa h=61")
    want = oracle_decode_from_cache(w, kc.cpu(), vc.cpu(), inp["q"], inp["seq_len"], inp["q_pos"])
    assert_bf16_close(got, want, "stage tpa h=61")
    scale = 64.0 / np.sqrt(w.shape.dh)
    got, kc, vc = _run(w, inp, sm_scale=float(scale))
    want = oracle_decode_from_cache(w, kc.cpu(), vc.cpu(), inp["q"], inp["seq_len"], inp["q_pos"], sm_scale=scale)
    assert_bf16_close(got, want, "peaked tpa h=61")
