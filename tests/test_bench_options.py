"""bench.py's options and the query-factor inputs of its kpa_decode_qf mode (CPU only).

  - the factored-score engine runs only from query factors, and the tcgen05 engine only
    from dense queries;
  - the query factor records are seeded, shaped [batch][E_Q] float32, and the query
    they assemble (the oracle's reconstruction, eq 2 for Q) has the dense query's spread.
"""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402
from workloads import FLASHTPA_DECODE, TPA_DECODE, query_factor_inputs, to_f64  # noqa: E402


def test_engine_options_follow_the_query_form():
    a = bench._args(["--workload", "flashtpa", "--query-factors", "--decode-engine", "2"])
    assert a.query_factors and a.decode_engine == 2
    assert bench._args(["--workload", "flashtpa", "--query-factors"]).decode_engine == 0
    for bad in (["--decode-engine", "2"],                                    # factored score, dense query
                ["--query-factors", "--decode-engine", "1"],                 # tcgen05 takes dense queries
                ["--query-factors", "--tokens-per-split", "128"]):           # kpa_decode_qf plans its split
        with pytest.raises(SystemExit):
            bench._args(bad)


def test_query_factor_inputs():
    w = FLASHTPA_DECODE.replace(batch=64)
    s = w.shape
    qf = query_factor_inputs(w, 3)
    assert tuple(qf.shape) == (w.batch, s.e_q) and str(qf.dtype) == "torch.float32"
    assert np.array_equal(qf.numpy(), query_factor_inputs(w, 3).numpy())
    assert not np.array_equal(qf.numpy(), query_factor_inputs(w, 4).numpy())
    q = np.stack([oracle.reconstruct(s.h1, s.h2, s.d1, s.d2, s.r_q, f) for f in to_f64(qf)])
    assert q.shape == (w.batch, s.h, s.dh)
    # 64 x 32 x 64 elements: the sample spread is within a few percent of q_std
    assert abs(q.std() / w.q_std - 1.0) < 0.05
    with pytest.raises(ValueError):
        query_factor_inputs(TPA_DECODE, 0)                                   # r_q = 0: no query factors
