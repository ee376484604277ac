"""Helpers shared by the GPU parity tests: move seeded inputs to the device, run
the library through its C ABI, read the interleaved cache back, measure errors."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from workloads import to_f64

pytestmark = pytest.mark.gpu

# Tolerances for factor-space attention against the float64 oracle: bf16 factors
# with fp32 accumulation must stay within max-abs 1e-2 and relative L2 2e-3; an
# fp32 build within max-abs 1e-5.
BF16_MAX_ABS, BF16_REL_L2 = 1e-2, 2e-3
F32_MAX_ABS = 1e-5


def kpa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import factorised_kv_attention_b200 as lib
    return lib


def torch_dtype(dtype: str):
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def planes(shape, batch, capacity, dtype, device="cuda"):
    dt = torch_dtype(dtype)
    kc = torch.zeros(batch * capacity * shape.e_k, dtype=dt, device=device)
    vc = torch.zeros(batch * capacity * shape.e_v, dtype=dt, device=device)
    return kc, vc


def natural(plane, batch, capacity, E):
    """[batch][capacity][E] view of an interleaved cache plane (group-of-8 order undone)."""
    return plane.view(batch, capacity // 8, E, 8).permute(0, 1, 3, 2).reshape(batch, capacity, E)


def fill_cache(lib, w, inp, start=None):
    """kpa_append_factors of the workload's records into fresh planes (slot = position)."""
    s = w.shape
    cfg = lib.make_config(s, w.dtype)
    kc, vc = planes(s, w.batch, w.capacity, w.dtype)
    st = torch.zeros(w.batch, dtype=torch.int32, device="cuda") if start is None else start
    lib.kpa_append_factors(cfg, w.batch, w.capacity, inp["kf"].cuda().contiguous(),
                           inp["vf"].cuda().contiguous(), st, w.capacity, kc, vc)
    return cfg, kc, vc


def run_decode(lib, w, cfg, kc, vc, q, seq_len, q_pos, *, max_len=None, sm_scale=None,
               tokens_per_split=0):
    s = w.shape
    max_len = int(seq_len.max().item()) if max_len is None else max_len
    sm_scale = 1.0 / float(np.sqrt(s.dh)) if sm_scale is None else sm_scale
    ws_bytes = lib.kpa_decode_workspace_size(cfg, w.batch, max_len, tokens_per_split)
    ws = torch.zeros(max(ws_bytes, 256), dtype=torch.uint8, device="cuda")
    out = torch.full((w.batch, s.h, s.dh), float("nan"), dtype=torch.float32, device="cuda")
    lib.kpa_decode_split(cfg, w.batch, q.cuda().contiguous(),
                         None if q_pos is None else q_pos.cuda().contiguous(), kc, vc, w.capacity,
                         seq_len.cuda().contiguous(), max_len, sm_scale, tokens_per_split, out, ws)
    return out


def errors(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape
    assert np.all(np.isfinite(got)), "non-finite GPU output"
    d = got - want
    max_abs = float(np.max(np.abs(d))) if d.size else 0.0
    nrm = float(np.linalg.norm(want))
    rel = float(np.linalg.norm(d) / nrm) if nrm > 0 else float(np.linalg.norm(d))
    return max_abs, rel


def assert_bf16_close(got, want, what=""):
    max_abs, rel = errors(got, want)
    assert max_abs <= BF16_MAX_ABS and rel <= BF16_REL_L2, \
        f"{what}: max-abs {max_abs:.3e} (<= {BF16_MAX_ABS}), rel-L2 {rel:.3e} (<= {BF16_REL_L2})"
    return max_abs, rel


def assert_f32_close(got, want, what=""):
    max_abs, rel = errors(got, want)
    assert max_abs <= F32_MAX_ABS, f"{what}: max-abs {max_abs:.3e} (<= {F32_MAX_ABS})"
    return max_abs, rel


def assert_close(dtype, got, want, what=""):
    return (assert_bf16_close if dtype == "bf16" else assert_f32_close)(got, want, what)


def oracle_decode_from_cache(w, kc, vc, q, seq_len, q_pos, heads=None, sm_scale=None):
    """The oracle fed the exact values the GPU cache holds (B^K already rotated)."""
    s = w.shape
    kn = to_f64(natural(kc, w.batch, w.capacity, s.e_k))
    vn = to_f64(natural(vc, w.batch, w.capacity, s.e_v))
    return oracle.decode(s, to_f64(q), kn, vn, seq_len.numpy(),
                         q_pos=None if q_pos is None else q_pos.numpy(), keys_rotated=True,
                         sm_scale=sm_scale, heads=heads)


def oracle_decode_unrotated(w, inp, heads=None, sm_scale=None, q=None):
    """The plain definition: unrotated factor records, RoPE on the reconstruction."""
    return oracle.decode(w.shape, to_f64(inp["q"] if q is None else q), to_f64(inp["kf"]),
                         to_f64(inp["vf"]), inp["seq_len"].numpy(), q_pos=inp["q_pos"].numpy(),
                         sm_scale=sm_scale, heads=heads)
