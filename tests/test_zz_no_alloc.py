"""kpa_decode_noalloc: the decode entry point for callers that cannot allocate
device memory.  It takes no workspace; the library's fixed device scratch array
stands in for it.  Checked through the C ABI against kpa_decode (GPU).

This file is collected last on purpose, and it needs nothing from earlier
tests: it passes alone in a fresh process and after the rest of the suite."""
import numpy as np
import pytest
import torch

from gpu_util import assert_bf16_close, fill_cache, kpa, run_decode
from workloads import KPA_MEDIUM, TPA_DECODE, decode_inputs

pytestmark = pytest.mark.gpu


def _case(lib, w):
    inp = decode_inputs(w)
    cfg, kc, vc = fill_cache(lib, w, inp)
    ref = run_decode(lib, w, cfg, kc, vc, inp["q"], inp["seq_len"], inp["q_pos"])
    dev = {k: inp[k].cuda() for k in ("q", "q_pos", "seq_len")}
    return cfg, kc, vc, dev, int(inp["seq_len"].max()), ref


def test_noalloc_matches_decode_on_two_calls_in_a_row():
    lib = kpa()
    cases = [
        (KPA_MEDIUM.replace(batch=4, capacity=1536, ragged=(1, 1536), seed=21)),
        (TPA_DECODE.replace(batch=3, capacity=2048, length=0, ragged=(1, 2048), seed=22)),
    ]
    prepared = [(w, *_case(lib, w)) for w in cases]
    torch.cuda.synchronize()
    outs = []
    for w, cfg, kc, vc, dev, max_len, ref in prepared:     # two calls back to back
        out = torch.full_like(ref, float("nan"))
        lib.kpa_decode_noalloc(cfg, w.batch, dev["q"], dev["q_pos"], kc, vc, w.capacity,
                               dev["seq_len"], max_len, 1.0 / float(np.sqrt(w.shape.dh)), out)
        outs.append(out)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    for (w, *_, ref), out in zip(prepared, outs):
        assert_bf16_close(out.cpu().numpy(), ref.cpu().numpy(), f"no-alloc vs kpa_decode: {w.name}")


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
