"""kpa_decode_qf with the factored score (Proposition 2.2: head-shared dots of the
query's B factors with the keys' B factors, then a rank mix per head; the FlashTPA
form), selected by kpa_test_set_decode_engine(2), against the float64 oracle and
against the default dense-form kernel on the same inputs (GPU)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_bf16_close, errors, fill_cache, kpa, oracle_decode_from_cache, oracle_decode_unrotated
from workloads import FLASHTPA_DECODE, KPA_MEDIUM, Shape, decode_inputs, to_f64

pytestmark = pytest.mark.gpu

SHAPES = {
    # the pages' FlashTPA decoding shape: h = 32, d_h = 64, R_Q = 16, R_K = R_V = 1
    "flashtpa": Shape(h1=32, h2=1, d1=1, d2=64, r_k=1, r_v=1, r_q=16, d_model=2048, rope_base=10000.0),
    # the TPA decode shape with four query ranks
    "tpa_h16_rq4": Shape(h1=16, h2=1, d1=1, d2=64, r_k=2, r_v=2, r_q=4, d_model=1024, rope_base=10000.0),
    # odd head count and ranks
    "h12_rk3_rv1_rq5": Shape(h1=12, h2=1, d1=1, d2=64, r_k=3, r_v=1, r_q=5, d_model=512, rope_base=500000.0),
}


def _case(shape, batch, cap, seed, ragged=True):
    w = KPA_MEDIUM.replace(shape=shape, batch=batch, capacity=cap, ragged=(1, cap) if ragged else (),
                           length=0 if ragged else cap, seed=seed, factor_std=1.0 / np.sqrt(shape.r_k))
    inp = decode_inputs(w)
    rng = np.random.default_rng(seed + 100)
    qf = (rng.standard_normal((batch, shape.e_q)) / np.sqrt(shape.r_q)).astype(np.float32)
    return w, inp, qf


def _decode_qf(lib, w, cfg, kc, vc, inp, qf_dev, qf_stride, qf_seq_stride, engine, scale):
    L = inp["seq_len"]
    max_len = int(L.max())
    out = torch.full((w.batch, w.shape.h, w.shape.dh), float("nan"), dtype=torch.float32, device="cuda")
    lib.kpa_test_set_decode_engine(engine)
    try:
        # sized with the engine selected: the factored score plans its own splits
        ws = torch.zeros(max(lib.kpa_decode_workspace_size(cfg, w.batch, max_len), 256), dtype=torch.uint8,
                         device="cuda")
        lib.kpa_decode_qf(cfg, w.batch, qf_dev, qf_stride, qf_seq_stride, inp["q_pos"].cuda(), kc, vc, w.capacity,
                          L.cuda(), max_len, scale, out, ws)
        torch.cuda.synchronize()
    finally:
        lib.kpa_test_set_decode_engine(0)
    assert lib.kpa_read_device_error() == 0
    return out.cpu().numpy()


def _oracle(w, inp, qf, scale, heads=None):
    s = w.shape
    q_dense = np.stack([oracle.reconstruct(s.h1, s.h2, s.d1, s.d2, s.r_q, qf[b].astype(np.float64))
                        for b in range(w.batch)])
    return oracle_decode_unrotated(w, inp, q=torch.from_numpy(q_dense), sm_scale=scale, heads=heads)


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_factored_score_matches_oracle_and_dense_form(name):
    shape = SHAPES[name]
    w, inp, qf = _case(shape, 3, 1024, 61)
    lib = kpa()
    cfg, kc, vc = fill_cache(lib, w, inp)
    scale = 1.0 / np.sqrt(shape.dh)
    qf_dev = torch.from_numpy(qf).cuda()
    got = _decode_qf(lib, w, cfg, kc, vc, inp, qf_dev, 1, shape.e_q, 2, scale)
    want = _oracle(w, inp, qf, scale)
    assert_bf16_close(got, want, f"factored score {name}")
    if shape.h1 % 16 == 0:        # the dense form needs a tensor-core variant (h a multiple of 16)
        dense = _decode_qf(lib, w, cfg, kc, vc, inp, qf_dev, 1, shape.e_q, 0, scale)
        assert_bf16_close(dense, want, f"dense form {name}")
        max_abs, rel = errors(got, dense)
        assert max_abs <= 1e-4 and rel <= 2e-5, f"factored vs dense {name}: {max_abs} {rel}"


def test_factored_score_reads_strided_factors_and_peaked_scores():
    """The append's workspace layout ([E_Q][batch], qf_stride = batch) and a softmax with
    logit gaps far above 10 (sm_scale x 64).  Stage parity: the oracle reads the cache
    the GPU wrote, so the x64 scale does not also amplify the bf16 rounding of the
    rotated keys at the cache write (which the end-to-end comparison would count)."""
    shape = SHAPES["tpa_h16_rq4"]
    w, inp, qf = _case(shape, 4, 520, 62)
    lib = kpa()
    cfg, kc, vc = fill_cache(lib, w, inp)
    scale = 64.0 / np.sqrt(shape.dh)
    qf_t = torch.from_numpy(np.ascontiguousarray(qf.T)).cuda()             # [E_Q][batch]
    got = _decode_qf(lib, w, cfg, kc, vc, inp, qf_t, w.batch, 1, 2, scale)
    s = w.shape
    q_dense = np.stack([oracle.reconstruct(s.h1, s.h2, s.d1, s.d2, s.r_q, qf[b].astype(np.float64))
                        for b in range(w.batch)])
    want = oracle_decode_from_cache(w, kc.cpu(), vc.cpu(), torch.from_numpy(q_dense), inp["seq_len"], inp["q_pos"],
                                    sm_scale=scale)
    assert_bf16_close(got, want, "factored score, strided factors, peaked")


def test_factored_score_special_lengths():
    """L = 0 gives zeros, L = 1 gives V_0, tails at 8k + r and at tile edges."""
    shape = SHAPES["flashtpa"]
    w, inp, qf = _case(shape, 6, 1024, 63, ragged=False)
    inp["seq_len"] = torch.tensor([0, 1, 7, 33, 129, 1024], dtype=torch.int32)
    inp["q_pos"] = inp["seq_len"].clone()
    lib = kpa()
    cfg, kc, vc = fill_cache(lib, w, inp)
    scale = 1.0 / np.sqrt(shape.dh)
    got = _decode_qf(lib, w, cfg, kc, vc, inp, torch.from_numpy(qf).cuda(), 1, shape.e_q, 2, scale)
    assert np.all(got[0] == 0.0)
    want = _oracle(w, inp, qf, scale)
    assert_bf16_close(got[1:], want[1:], "factored score, special lengths")


def test_factored_score_long_sequence_sampled_heads():
    """The FlashTPA shape at 2^15 tokens (the whole split plan at a long length), checked
    on a sample of heads that the oracle computes one by one."""
    shape = SHAPES["flashtpa"]
    w, inp, qf = _case(shape, 1, 1 << 15, 64, ragged=False)
    lib = kpa()
    cfg, kc, vc = fill_cache(lib, w, inp)
    scale = 1.0 / np.sqrt(shape.dh)
    got = _decode_qf(lib, w, cfg, kc, vc, inp, torch.from_numpy(qf).cuda(), 1, shape.e_q, 2, scale)
    heads = [0, 7, 19, 31]
    want = _oracle(w, inp, qf, scale, heads=heads)
    assert_bf16_close(got[0, heads], want[0, heads], "factored score, 2^15 tokens")
