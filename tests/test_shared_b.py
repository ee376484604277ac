"""Decode over a cache whose keys and values share their B factors ("Tensor Product
Attention Is All You Need", section 5, "TPA KV with Shared B") against the float64
oracle (GPU).  The key plane holds [A^K | B] with B unrotated, the value plane [A^V];
the decode kernel rotates B at each cached token's slot for the score and reads the
same, unrotated B for the values."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_bf16_close, fill_cache, kpa, natural, run_decode
from workloads import TPA_SHARED_DECODE, Shape, decode_inputs, to_f64

pytestmark = pytest.mark.gpu


def _oracle(w, inp, sm_scale, q=None):
    return oracle.decode_shared_b(w.shape, to_f64(inp["q"] if q is None else q), to_f64(inp["kf"]),
                                  to_f64(inp["vf"]), inp["seq_len"].numpy(), q_pos=inp["q_pos"].numpy(),
                                  sm_scale=sm_scale)


KPA_SHARED = Shape(h1=4, h2=4, d1=8, d2=16, r_k=2, r_v=2, rope_base=10000.0, shared_b=1)

# (workload, tokens per split, score sharpening): automatic plan over ragged lengths;
# explicit 64- and 128-token splits with ragged tails; scores sharpened 40x; and a long
# cache with a large RoPE base (angles up to several thousand radians).
CASES = {
    "ragged_auto": (TPA_SHARED_DECODE.replace(batch=4, capacity=1024, length=0, ragged=(1, 1024), seed=61), 0, 1.0),
    "split64": (TPA_SHARED_DECODE.replace(batch=3, capacity=512, length=0, ragged=(100, 512), seed=62), 64, 1.0),
    "split128_sharp": (TPA_SHARED_DECODE.replace(batch=3, capacity=768, length=0, ragged=(200, 768), seed=63),
                       128, 40.0),
    "long_base5e5": (TPA_SHARED_DECODE.replace(
        shape=dataclasses.replace(TPA_SHARED_DECODE.shape, rope_base=500000.0), batch=2, capacity=8192,
        length=8192, seed=64), 0, 1.0),
    # the Kronecker split h = 4x4, d_h = 8x16 with a shared B (rotation on the d2 pairs of B)
    "kpa_ragged": (TPA_SHARED_DECODE.replace(shape=KPA_SHARED, batch=3, capacity=1024, length=0,
                                             ragged=(1, 1024), factor_std=0.5, seed=69), 0, 1.0),
    "kpa_split64_sharp": (TPA_SHARED_DECODE.replace(shape=KPA_SHARED, batch=2, capacity=512, length=0,
                                                    ragged=(70, 512), factor_std=0.5, seed=70), 64, 20.0),
}


@pytest.mark.parametrize("name", list(CASES))
def test_shared_b_decode_against_oracle(name):
    w, tps, sharp = CASES[name]
    inp = decode_inputs(w)
    lib = kpa()
    cfg, kc, vc = fill_cache(lib, w, inp)
    scale = sharp / np.sqrt(w.shape.dh)
    out = run_decode(lib, w, cfg, kc, vc, inp["q"], inp["seq_len"], inp["q_pos"], sm_scale=scale,
                     tokens_per_split=tps)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    assert_bf16_close(out.cpu().numpy(), _oracle(w, inp, scale), f"shared B {name}")


def test_shared_b_cache_holds_the_factors_unrotated():
    """kpa_append_factors with a shared B writes the records as given: B is not rotated
    (the values read it), and the value plane holds A^V only (bit-exact)."""
    w = TPA_SHARED_DECODE.replace(batch=2, capacity=64, length=0, ragged=(17, 64), seed=65)
    inp = decode_inputs(w)
    lib = kpa()
    _, kc, vc = fill_cache(lib, w, inp)
    s = w.shape
    assert vc.numel() == w.batch * w.capacity * s.r_v * s.h1 * s.d1
    kn = natural(kc.cpu(), w.batch, w.capacity, s.e_k)
    vn = natural(vc.cpu(), w.batch, w.capacity, s.e_v)
    assert torch.equal(kn, inp["kf"]) and torch.equal(vn, inp["vf"])


def test_shared_b_decode_from_query_factors():
    """kpa_decode_qf over a shared-B cache: the query assembled from factors in the kernel."""
    w = TPA_SHARED_DECODE.replace(shape=dataclasses.replace(TPA_SHARED_DECODE.shape, r_q=6), batch=3,
                                  capacity=1024, length=0, ragged=(1, 1024), seed=66)
    s = w.shape
    inp = decode_inputs(w)
    rng = np.random.default_rng(166)
    qf = (rng.standard_normal((w.batch, s.e_q)) / np.sqrt(s.r_q)).astype(np.float32)
    lib = kpa()
    cfg, kc, vc = fill_cache(lib, w, inp)
    L = inp["seq_len"]
    max_len = int(L.max())
    ws = torch.zeros(lib.kpa_decode_workspace_size(cfg, w.batch, max_len), dtype=torch.uint8, device="cuda")
    out = torch.full((w.batch, s.h, s.dh), float("nan"), dtype=torch.float32, device="cuda")
    scale = 1.0 / np.sqrt(s.dh)
    lib.kpa_decode_qf(cfg, w.batch, torch.from_numpy(qf).cuda(), 1, s.e_q, inp["q_pos"].cuda(), kc, vc,
                      w.capacity, L.cuda(), max_len, scale, out, ws)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    q_dense = np.stack([oracle.reconstruct(s.h1, s.h2, s.d1, s.d2, s.r_q, qf[b].astype(np.float64))
                        for b in range(w.batch)])
    assert_bf16_close(out.cpu().numpy(), _oracle(w, inp, scale, q=torch.from_numpy(q_dense)),
                      "shared B, query factors")


def test_shared_b_fp16_overflow_is_reported():
    """The rotated key factors enter the score product as fp16: a cached B value beyond
    its range in a visible slot is reported as KPA_ERR_DEVICE_CHECK."""
    w = TPA_SHARED_DECODE.replace(batch=2, capacity=256, length=200, seed=67)
    inp = decode_inputs(w)
    a = w.shape.r_k * w.shape.h1 * w.shape.d1
    inp["kf"][1, 37, a + 5] = 1.0e6          # a B element of a visible slot of sequence 1
    lib = kpa()
    cfg, kc, vc = fill_cache(lib, w, inp)
    lib.kpa_read_device_error()               # clear
    run_decode(lib, w, cfg, kc, vc, inp["q"], inp["seq_len"], inp["q_pos"])
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == lib.KPA_ERR_DEVICE_CHECK


def _close_bf16(got, want, what):
    """Stored bf16 values: half a bf16 ulp plus the fp32 accumulation of the projection."""
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    bad = np.abs(got - want) > 2.0 ** -8 * np.abs(want) + 1e-5 * max(np.abs(want).max(), 1.0)
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} off, worst {np.abs(got - want).max():.3e}"


@pytest.mark.parametrize("split,n_tok", [("tpa", 300), ("tpa", 5), ("kpa", 300)],
                         ids=["tpa_gemm", "tpa_few_tokens", "kpa_gemm"])
def test_shared_b_append_then_decode(split, n_tok):
    """kpa_append with a shared B (merged columns [A^Q | B^Q | A^K | A^V | B]): the key
    records hold [A^K | B] unrotated, the value records A^V, q_out is rotated; a decode
    over that cache then matches the oracle's shared-B decode of the stored records."""
    from workloads import APPEND_PREFILL, append_inputs
    base = TPA_SHARED_DECODE.shape if split == "tpa" else KPA_SHARED
    s = dataclasses.replace(base, r_q=4, d_model=256)
    w = APPEND_PREFILL.replace(shape=s, batch=2, n_tok=n_tok, capacity=512, seed=68)
    inp = append_inputs(w)
    start = torch.tensor([0, 40], dtype=torch.int32)
    lib = kpa()
    cfg = lib.make_config(s, "bf16")
    kc = torch.zeros(w.batch * w.capacity * s.e_k, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros(w.batch * w.capacity * s.e_v, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(max(lib.kpa_append_workspace_size(cfg, w.batch, n_tok), 256), dtype=torch.uint8,
                     device="cuda")
    q_out = torch.full((w.batch, n_tok, s.h, s.dh), float("nan"), dtype=torch.bfloat16, device="cuda")
    lib.kpa_append(cfg, w.batch, n_tok, inp["x"].cuda(), inp["W"].cuda(), start.cuda(), w.capacity, kc, vc,
                   q_out, ws)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    q_rot, k_store, v_rec, _ = oracle.append(s, to_f64(inp["x"]), to_f64(inp["W"]), start.numpy())
    kn = natural(kc.cpu(), w.batch, w.capacity, s.e_k)
    vn = natural(vc.cpu(), w.batch, w.capacity, s.e_v)
    for b in range(w.batch):
        st = int(start[b])
        _close_bf16(to_f64(kn[b, st:st + n_tok]), k_store[b], f"key records b={b}")
        _close_bf16(to_f64(vn[b, st:st + n_tok]), v_rec[b], f"value records b={b}")
    _close_bf16(to_f64(q_out.cpu()), q_rot, "assembled query")
    # decode of the newest token of each sequence over the slots the append wrote
    L = start + n_tok
    dw = TPA_SHARED_DECODE.replace(shape=s, batch=w.batch, capacity=w.capacity)
    q1 = q_out[:, -1].contiguous()
    scale = 1.0 / np.sqrt(s.dh)
    out = run_decode(lib, dw, cfg, kc, vc, q1.cpu(), L, None, sm_scale=scale)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    # q_out is already rotated at its position: the oracle rotates the keys at their slots and
    # takes the query as given (position 0 = identity)
    want = oracle.decode_shared_b(s, to_f64(q1.cpu()), to_f64(kn), to_f64(vn), L.numpy(),
                                  q_pos=np.zeros(w.batch, dtype=np.int64), sm_scale=scale)
    assert_bf16_close(out.cpu().numpy(), want, f"decode after shared-B append ({n_tok} tokens)")


def test_shared_b_append_then_prefill():
    """kpa_append of a chunk into a shared-B cache (h = 4x4, d_h = 8x16), then the causal
    prefill from q_out: the kernel rebuilds K with B rotated at each key's slot and V from
    the same, unrotated B.  Sampled rows against the oracle on the stored records."""
    from workloads import APPEND_PREFILL, append_inputs
    s = dataclasses.replace(KPA_SHARED, r_q=6, d_model=256)
    n_tok = 300
    w = APPEND_PREFILL.replace(shape=s, batch=2, n_tok=n_tok, capacity=512, seed=71)
    inp = append_inputs(w)
    start = torch.tensor([0, 40], dtype=torch.int32)
    lib = kpa()
    cfg = lib.make_config(s, "bf16")
    kc = torch.zeros(w.batch * w.capacity * s.e_k, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros(w.batch * w.capacity * s.e_v, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(lib.kpa_append_workspace_size(cfg, w.batch, n_tok), dtype=torch.uint8, device="cuda")
    q_out = torch.empty(w.batch, n_tok, s.h, s.dh, dtype=torch.bfloat16, device="cuda")
    lib.kpa_append(cfg, w.batch, n_tok, inp["x"].cuda(), inp["W"].cuda(), start.cuda(), w.capacity, kc, vc,
                   q_out, ws)
    scale = 1.0 / np.sqrt(s.dh)
    out = torch.full((w.batch, n_tok, s.h, s.dh), float("nan"), dtype=torch.float32, device="cuda")
    lib.kpa_prefill(cfg, w.batch, n_tok, q_out, start.cuda(), kc, vc, w.capacity, scale, out)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    kn = to_f64(natural(kc.cpu(), w.batch, w.capacity, s.e_k))
    vn = to_f64(natural(vc.cpu(), w.batch, w.capacity, s.e_v))
    qo = to_f64(q_out.cpu())
    got = out.cpu().numpy()
    rng = np.random.default_rng(7)
    rows = [(int(b), int(t)) for b, t in zip(rng.integers(0, w.batch, 10), rng.integers(0, n_tok, 10))]
    rows += [(0, 0), (1, 0), (0, 127), (1, 128), (1, n_tok - 1)]
    for b, t in rows:
        L = int(start[b]) + t + 1
        # q_out is rotated already (position 0 = identity); the oracle rotates the keys
        want = oracle.decode_shared_b(s, qo[b, t][None], kn[b][None], vn[b][None], [L],
                                      q_pos=[0], sm_scale=scale)
        assert_bf16_close(got[b, t], want[0], f"shared-B prefill row ({b},{t})")


def test_shared_b_prefill_from_query_factors():
    """A shared-B cache written by kpa_append without q_out, then kpa_prefill_qf from the
    append's workspace: K rebuilt with B rotated per key, Q assembled from the factors."""
    from workloads import APPEND_PREFILL, append_inputs
    s = dataclasses.replace(KPA_SHARED, r_q=6, d_model=256)
    n_tok = 300
    w = APPEND_PREFILL.replace(shape=s, batch=2, n_tok=n_tok, capacity=512, seed=74)
    inp = append_inputs(w)
    start = torch.tensor([0, 40], dtype=torch.int32)
    lib = kpa()
    cfg = lib.make_config(s, "bf16")
    kc = torch.zeros(w.batch * w.capacity * s.e_k, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros(w.batch * w.capacity * s.e_v, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(lib.kpa_append_workspace_size(cfg, w.batch, n_tok), dtype=torch.uint8, device="cuda")
    lib.kpa_append(cfg, w.batch, n_tok, inp["x"].cuda(), inp["W"].cuda(), start.cuda(), w.capacity, kc, vc, None, ws)
    scale = 1.0 / np.sqrt(s.dh)
    out = torch.full((w.batch, n_tok, s.h, s.dh), float("nan"), dtype=torch.float32, device="cuda")
    lib.kpa_prefill_qf(cfg, w.batch, n_tok, ws.view(torch.float32), w.batch * n_tok, n_tok, 1, start.cuda(), kc, vc,
                       w.capacity, scale, out)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    q_rot, _, _, _ = oracle.append(s, to_f64(inp["x"]), to_f64(inp["W"]), start.numpy())
    kn = to_f64(natural(kc.cpu(), w.batch, w.capacity, s.e_k))
    vn = to_f64(natural(vc.cpu(), w.batch, w.capacity, s.e_v))
    got = out.cpu().numpy()
    for b, t in [(0, 0), (0, 150), (1, 0), (1, 128), (1, n_tok - 1), (0, n_tok - 1)]:
        L = int(start[b]) + t + 1
        want = oracle.decode_shared_b(s, q_rot[b, t][None], kn[b][None], vn[b][None], [L], q_pos=[0],
                                      sm_scale=scale)
        assert_bf16_close(got[b, t], want[0], f"shared-B prefill from query factors, row ({b},{t})")
