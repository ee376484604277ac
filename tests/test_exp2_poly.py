"""The prefill's FMA-pipe exponential 2^x (Cody-Waite reduction plus a fitted degree-4
polynomial, kpa_f32x2.cuh).  On the CPU: the committed fit script reproduces the
header's coefficients and their float32 evaluation stays within 2.7e-6 relative of
float64 2^x over [-126, 8].  On the GPU: the kernel's own outputs over that domain
against float64 2^x and against CUDA's exp2f (torch.exp2 on the device)."""
import importlib.util
import os

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
MAX_REL = 2.7e-6


def _fit_module():
    path = os.path.join(ROOT, "factorised_kv_attention_b200", "csrc", "fit_exp2_poly.py")
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _domain():
    rng = np.random.default_rng(0)
    return np.concatenate([np.linspace(-126, 8, 2_000_001), rng.uniform(-126, 8, 500_000),
                           np.arange(-126, 9, dtype=np.float64),            # integers: f = 0
                           np.arange(-126, 8, dtype=np.float64) + 0.5,       # rounding ties
                           [-1e-30, 1e-30, -0.0, 0.0]]).astype(np.float32)


def test_fit_reproduces_the_header_coefficients():
    fit = _fit_module()
    assert np.array_equal(fit.fit(), fit.header_coefficients())
    assert fit.max_rel_error(fit.header_coefficients()) <= MAX_REL


@pytest.mark.gpu
def test_kernel_exp2_against_float64_and_cuda_exp2f():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import factorised_kv_attention_b200 as lib
    x = torch.from_numpy(_domain()).cuda()
    y = torch.full_like(x, float("nan"))
    lib.kpa_test_exp2_poly(x, y)
    ref32 = torch.exp2(x)                                  # CUDA's exp2f
    torch.cuda.synchronize()
    got = y.cpu().numpy().astype(np.float64)
    xs = x.cpu().numpy().astype(np.float64)
    want = np.exp2(xs)
    rel = np.abs(got - want) / want
    assert np.all(np.isfinite(got))
    assert rel.max() <= MAX_REL, f"max relative error {rel.max():.3e} at x = {xs[np.argmax(rel)]}"
    rel32 = np.abs(got - ref32.cpu().numpy().astype(np.float64)) / want
    assert rel32.max() <= MAX_REL + 2.0 ** -23, f"against exp2f: {rel32.max():.3e}"
    # the fit script's host model of the kernel's float32 steps agrees to one ulp
    fit = _fit_module()
    host = fit.evaluate(fit.header_coefficients(), x.cpu().numpy())
    ulps = np.abs(host.view(np.int32).astype(np.int64) - y.cpu().numpy().view(np.int32).astype(np.int64))
    assert ulps.max() <= 1
    # below the clamp every input gives 2^-126 (to the polynomial's error)
    lo = torch.tensor([-126.0, -127.5, -300.0, -1e30], device="cuda")
    ylo = torch.empty_like(lo)
    lib.kpa_test_exp2_poly(lo, ylo)
    assert np.allclose(ylo.cpu().numpy(), 2.0 ** -126, rtol=MAX_REL, atol=0)
