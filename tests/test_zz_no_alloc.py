"""kpa_decode_noalloc: the decode entry point for callers that cannot allocate
device memory.  It takes no workspace; the library's fixed device scratch array
stands in for it.  Checked through the C ABI against the float64 oracle and
against kpa_decode (GPU).

This file is collected last on purpose, and it needs nothing from earlier
tests: it passes alone in a fresh process and after the rest of the suite."""
import numpy as np
import pytest
import torch

from gpu_util import assert_bf16_close, fill_cache, kpa, oracle_decode_unrotated, run_decode
from workloads import KPA_MEDIUM, TPA_DECODE, decode_inputs

pytestmark = pytest.mark.gpu


def _case(lib, w):
    inp = decode_inputs(w)
    cfg, kc, vc = fill_cache(lib, w, inp)
    ref = run_decode(lib, w, cfg, kc, vc, inp["q"], inp["seq_len"], inp["q_pos"])
    dev = {k: inp[k].cuda() for k in ("q", "q_pos", "seq_len")}
    return inp, cfg, kc, vc, dev, int(inp["seq_len"].max()), ref


def _noalloc(lib, w, cfg, kc, vc, dev, max_len, like):
    out = torch.full_like(like, float("nan"))
    lib.kpa_decode_noalloc(cfg, w.batch, dev["q"], dev["q_pos"], kc, vc, w.capacity,
                           dev["seq_len"], max_len, 1.0 / float(np.sqrt(w.shape.dh)), out)
    return out


def test_noalloc_matches_oracle_and_decode_on_two_calls_in_a_row():
    lib = kpa()
    cases = [
        KPA_MEDIUM.replace(batch=4, capacity=1536, ragged=(1, 1536), seed=21),
        TPA_DECODE.replace(batch=3, capacity=2048, length=0, ragged=(1, 2048), seed=22),
    ]
    prepared = [(w, *_case(lib, w)) for w in cases]
    torch.cuda.synchronize()
    outs = []
    for w, inp, cfg, kc, vc, dev, max_len, ref in prepared:     # two calls back to back
        outs.append(_noalloc(lib, w, cfg, kc, vc, dev, max_len, ref))
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    for (w, inp, *_, ref), out in zip(prepared, outs):
        got = out.cpu().numpy()
        assert_bf16_close(got, oracle_decode_unrotated(w, inp), f"no-alloc vs oracle: {w.name}")
        assert_bf16_close(got, ref.cpu().numpy(), f"no-alloc vs kpa_decode: {w.name}")


def test_noalloc_after_a_call_that_timed_out():
    """A call whose bounded wait runs out leaves the shared scratch's split counters
    half counted; the next call must start from cleared counters all the same."""
    lib = kpa()
    # 31 splits per sequence, merged by the last CTA of each sequence through its counter
    w = TPA_DECODE.replace(batch=3, capacity=2048, length=2000, seed=23)
    inp, cfg, kc, vc, dev, max_len, ref = _case(lib, w)
    n_split, _, launches = lib.kpa_decode_plan(cfg, w.batch, max_len)
    assert n_split > 16 and launches == 1                  # the counter merge, not a cluster
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    lib.kpa_test_set_decode_hooks(0, 0, 20_000_000)        # tile 0 of split 0 never arrives
    try:
        _noalloc(lib, w, cfg, kc, vc, dev, max_len, ref)
        torch.cuda.synchronize()
        assert lib.kpa_read_device_error() == lib.KPA_ERR_TIMEOUT
    finally:
        lib.kpa_test_set_decode_hooks(-1, -1, 1_000_000_000)
    out = _noalloc(lib, w, cfg, kc, vc, dev, max_len, ref)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    assert torch.equal(out, ref)                           # same split plan: the same sums
    assert_bf16_close(out.cpu().numpy(), oracle_decode_unrotated(w, inp), "no-alloc after a timeout")


def test_noalloc_rejects_requests_above_its_scratch():
    lib = kpa()
    w = KPA_MEDIUM
    cfg = lib.make_config(w.shape, w.dtype)
    batch, max_len = 4000, 8192
    need = lib.kpa_decode_workspace_size(cfg, batch, max_len)
    assert need > lib.KPA_DECODE_NOALLOC_MAX_BYTES
    fake = 1 << 20                                         # never dereferenced: rejected first
    with pytest.raises(lib.KpaError) as e:
        lib.kpa_decode_noalloc(cfg, batch, fake, None, fake, fake, max_len, fake, max_len, 0.1, fake)
    assert e.value.status == lib.KPA_ERR_WORKSPACE
