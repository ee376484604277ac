"""Failure detection without a GPU fault (GPU): a copy that never arrives makes
the tensor-core decode's bounded mbarrier wait run out; the kernel records
KPA_ERR_TIMEOUT, drains its own copies and returns, and the context stays
usable for the next call."""
import numpy as np
import pytest
import torch

from gpu_util import fill_cache, kpa, run_decode
from workloads import KPA_LONG, TPA_DECODE, decode_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("w", [TPA_DECODE.replace(batch=2, capacity=1024, length=1000, seed=31),
                               KPA_LONG.replace(capacity=2048, length=2000, seed=32)],
                         ids=["tpa", "kpa"])
def test_wait_that_runs_out_reports_timeout(w):
    lib = kpa()
    inp = decode_inputs(w)
    cfg, kc, vc = fill_cache(lib, w, inp)
    good = run_decode(lib, w, cfg, kc, vc, inp["q"], inp["seq_len"], inp["q_pos"])
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    lib.kpa_test_set_decode_hooks(0, 0, 20_000_000)        # tile 0 of split 0 never arrives
    try:
        run_decode(lib, w, cfg, kc, vc, inp["q"], inp["seq_len"], inp["q_pos"])
        torch.cuda.synchronize()
        assert lib.kpa_read_device_error() == lib.KPA_ERR_TIMEOUT
    finally:
        lib.kpa_test_set_decode_hooks(-1, -1, 1_000_000_000)
    again = run_decode(lib, w, cfg, kc, vc, inp["q"], inp["seq_len"], inp["q_pos"])
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    assert torch.equal(again, good)
