"""The C ABI: the library loads, exports every call that include/kpa.h declares,
and rejects bad arguments before it touches a device (CPU only)."""
import ctypes
import dataclasses
import os
import re

import pytest

import factorised_kv_attention_b200 as kpa
import oracle
from workloads import APPEND_PREFILL, DECODE_CONFIGS, Shape

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(kpa_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported():
    declared = _declared_functions()
    assert len(declared) >= 12
    lib = ctypes.CDLL(kpa.LIB_PATH)
    missing = [n for n in declared if not hasattr(lib, n)]
    assert not missing, f"declared in include/ but not exported: {missing}"


def test_status_strings():
    for code in range(7):
        s = kpa.kpa_status_string(code)
        assert s.startswith("KPA_"), s
    assert "unknown" in kpa.kpa_status_string(42)


@pytest.mark.parametrize("name", sorted(DECODE_CONFIGS))
def test_cache_bytes_match_eq10(name):
    w = DECODE_CONFIGS[name]
    s = w.shape
    cfg = kpa.make_config(s, w.dtype)
    kb, vb = kpa.kpa_cache_bytes_per_token(cfg)
    elt = 2 if w.dtype == "bf16" else 4
    if s.order == 3:
        numbers = oracle.cache_numbers_per_token_order3(s.h1, s.d1, s.d2, s.r_k, s.r_v)
        assert kb * s.r_v == vb * s.r_k
    elif s.shared_b:
        numbers = oracle.cache_numbers_per_token_shared_b(s.h1, s.h2, s.d1, s.d2, s.r_k)
        assert vb == s.r_v * s.h1 * s.d1 * elt           # the value record is A^V only
    else:
        numbers = oracle.cache_numbers_per_token(s.h1, s.h2, s.d1, s.d2, s.r_k, s.r_v)
        assert kb * s.r_v == vb * s.r_k
    assert kb + vb == numbers * elt


def test_cache_bytes_of_the_configs():
    # per-token bytes of the five configurations, from eq (10)
    want = {"tiny_kpa": 768, "tpa_decode": 640, "kpa_medium": 2560, "kpa_long": 1280}
    for name, b in want.items():
        w = DECODE_CONFIGS[name]
        kb, vb = kpa.kpa_cache_bytes_per_token(kpa.make_config(w.shape, w.dtype))
        assert kb + vb == b, name
    kb, vb = kpa.kpa_cache_bytes_per_token(kpa.make_config(APPEND_PREFILL.shape, "bf16"))
    assert kb + vb == 768
    # shared B: A^K, A^V (16 each per rank) and one B (64 per rank), R = 2, bf16
    w = DECODE_CONFIGS["tpa_shared"]
    assert kpa.kpa_cache_bytes_per_token(kpa.make_config(w.shape, w.dtype)) == (320, 64)


def test_shared_b_needs_equal_ranks():
    cfg = kpa.make_config(Shape(h1=16, h2=1, d1=1, d2=64, r_k=2, r_v=1, shared_b=1), "bf16")
    with pytest.raises(kpa.KpaError) as e:
        kpa.kpa_cache_bytes_per_token(cfg)
    assert e.value.status == kpa.KPA_ERR_INVALID_ARG
    cfg = kpa.make_config(Shape(h1=16, h2=1, d1=1, d2=64, r_k=2, r_v=2), "bf16")
    cfg.shared_b = 2
    with pytest.raises(kpa.KpaError) as e:
        kpa.kpa_cache_bytes_per_token(cfg)
    assert e.value.status == kpa.KPA_ERR_INVALID_ARG


def test_prefill_kernel_kinds():
    """The tcgen05 prefill takes d1 = 8 with d2 = 16 (R = 2 or 4) or d2 = 8 (R = 2), B shared or
    not; the mma.sync prefill every other order-2 bf16 split with d_h <= 128 whose factor
    slices fit its staging, and the tcgen05 splits too after kpa_test_set_prefill_engine(1).
    d_h > 128, oversized slices and fp32 are refused before any device call."""
    def kind(**kw):
        return kpa.kpa_prefill_kernel_kind(kpa.make_config(Shape(**kw), "bf16"))

    c5 = dict(h1=4, h2=4, d1=8, d2=16, r_k=2, r_v=2)
    assert kind(**c5) == "tcgen05"
    assert kind(**c5, shared_b=1) == "tcgen05"
    for h1, h2 in ((4, 4), (2, 8), (8, 2), (4, 5), (2, 10), (10, 2)):    # section 3.2's splits
        assert kind(h1=h1, h2=h2, d1=8, d2=8, r_k=2, r_v=2) == "tcgen05", (h1, h2)
    assert kind(h1=4, h2=4, d1=8, d2=16, r_k=4, r_v=4) == "tcgen05"                  # rank 4
    for split in (dict(h1=16, h2=1, d1=1, d2=64, r_k=2, r_v=2), dict(h1=16, h2=1, d1=1, d2=64, r_k=2, r_v=2,
                                                                    shared_b=1),
                  dict(h1=4, h2=4, d1=8, d2=16, r_k=3, r_v=1), dict(h1=2, h2=8, d1=8, d2=8, r_k=4, r_v=4),
                  dict(h1=3, h2=2, d1=4, d2=6, r_k=2, r_v=2), dict(h1=8, h2=1, d1=1, d2=128, r_k=3, r_v=2)):
        assert kind(**split) == "mma_sync", split
    try:
        kpa.kpa_test_set_prefill_engine(1)
        assert kind(**c5) == "mma_sync"
    finally:
        kpa.kpa_test_set_prefill_engine(0)
    assert kind(**c5) == "tcgen05"
    with pytest.raises(kpa.KpaError) as e:
        kpa.kpa_test_set_prefill_engine(2)
    assert e.value.status == kpa.KPA_ERR_INVALID_ARG
    for bad in (dict(h1=4, h2=4, d1=16, d2=16, r_k=2, r_v=2),          # d_h = 256
                dict(h1=1, h2=1, d1=1, d2=128, r_k=8, r_v=8)):         # 2 x 1032-element slices
        cfg = kpa.make_config(Shape(**bad), "bf16")
        with pytest.raises(kpa.KpaError) as e:
            kpa.kpa_prefill_kernel_kind(cfg)
        assert e.value.status == kpa.KPA_ERR_UNSUPPORTED, bad
        with pytest.raises(kpa.KpaError) as e:
            kpa.kpa_prefill(cfg, 1, 16, A, A, A, A, 64, 0.1, A, stream=0)
        assert e.value.status == kpa.KPA_ERR_UNSUPPORTED, bad
    cfg = kpa.make_config(Shape(**c5), "f32")
    with pytest.raises(kpa.KpaError) as e:
        kpa.kpa_prefill_kernel_kind(cfg)
    assert e.value.status == kpa.KPA_ERR_UNSUPPORTED


def test_third_order_entry_points():
    """A third-order cache ([a | b | c] records, RoPE on b) is taken by the cache write
    and the decode; the projection and the prefill refuse it before any device call,
    and its own shape rules hold (h2 = 1, d1 even, no shared B)."""
    s = DECODE_CONFIGS["tpa_order3"].shape
    cfg = kpa.make_config(s, "bf16")
    assert kpa.kpa_cache_bytes_per_token(cfg) == (2 * s.r_k * (s.h1 + s.d1 + s.d2),) * 2
    with pytest.raises(kpa.KpaError) as e:
        kpa.kpa_prefill(cfg, 1, 16, A, A, A, A, 64, 0.1, A, stream=0)
    assert e.value.status == kpa.KPA_ERR_UNSUPPORTED
    cfg_q = kpa.make_config(dataclasses.replace(s, r_q=4, d_model=256), "bf16")
    with pytest.raises(kpa.KpaError) as e:
        kpa.kpa_append_workspace_size(cfg_q, 1, 16)
    assert e.value.status == kpa.KPA_ERR_UNSUPPORTED
    # d2 (= d_c) may be odd; d1 (= d_b, the rotated factor) may not
    assert kpa.kpa_cache_bytes_per_token(kpa.make_config(dataclasses.replace(s, d2=3), "bf16"))[0] > 0
    for bad in (dict(d1=7), dict(h2=2), dict(shared_b=1), dict(order=4)):
        with pytest.raises(kpa.KpaError) as e:
            kpa.kpa_cache_bytes_per_token(kpa.make_config(dataclasses.replace(s, **bad), "bf16"))
        assert e.value.status == kpa.KPA_ERR_INVALID_ARG, bad


BAD_SHAPES = [dict(h1=0), dict(d2=7), dict(r_k=0), dict(r_v=-1), dict(d1=-2)]


@pytest.mark.parametrize("bad", BAD_SHAPES, ids=str)
def test_bad_config_rejected(bad):
    base = dict(h1=4, h2=8, d1=8, d2=16, r_k=2, r_v=2)
    base.update(bad)
    cfg = kpa.make_config(Shape(**base), "bf16")
    with pytest.raises(kpa.KpaError) as e:
        kpa.kpa_cache_bytes_per_token(cfg)
    assert e.value.status == kpa.KPA_ERR_INVALID_ARG


def test_bad_dtype_and_base_rejected():
    cfg = kpa.make_config(DECODE_CONFIGS["kpa_long"].shape, "bf16")
    cfg.dtype = 7
    with pytest.raises(kpa.KpaError) as e:
        kpa.kpa_cache_bytes_per_token(cfg)
    assert e.value.status == kpa.KPA_ERR_INVALID_ARG
    cfg = kpa.make_config(DECODE_CONFIGS["kpa_long"].shape, "bf16")
    cfg.rope_base = 0.0
    with pytest.raises(kpa.KpaError):
        kpa.kpa_cache_bytes_per_token(cfg)


# Argument checks that run before any CUDA call: fake, aligned "device" addresses
# are never dereferenced because every case below is rejected first.
A = 1 << 20          # 16-byte aligned dummy address
CFG = kpa.make_config(DECODE_CONFIGS["kpa_long"].shape, "bf16")


def _decode(**over):
    args = dict(cfg=CFG, batch=2, q=A, q_pos=None, kcache=A, vcache=A, capacity=64, seq_len=A,
                max_len=64, sm_scale=0.1, out=A, workspace=A, ws_bytes=1 << 20)
    args.update(over)
    kpa.kpa_decode(args["cfg"], args["batch"], args["q"], args["q_pos"], args["kcache"],
                   args["vcache"], args["capacity"], args["seq_len"], args["max_len"],
                   args["sm_scale"], args["out"], args["workspace"], args["ws_bytes"], stream=0)


@pytest.mark.parametrize("over", [
    dict(q=None), dict(kcache=None), dict(vcache=None), dict(seq_len=None), dict(out=None),
    dict(q=A + 2), dict(kcache=A + 8), dict(out=A + 4), dict(seq_len=A + 1),
    dict(capacity=60), dict(capacity=0), dict(max_len=65), dict(max_len=-1), dict(batch=-1),
    dict(sm_scale=float("nan")), dict(sm_scale=float("inf")),
], ids=str)
def test_decode_rejects_before_launch(over):
    with pytest.raises(kpa.KpaError) as e:
        _decode(**over)
    assert e.value.status == kpa.KPA_ERR_INVALID_ARG


def test_decode_empty_batch_is_a_no_op():
    _decode(batch=0, q=None, kcache=None, vcache=None, seq_len=None, out=None, workspace=None)


@pytest.mark.parametrize("over", [
    dict(k_factors=None), dict(start_pos=None), dict(kcache=A + 2), dict(capacity=12),
    dict(n_tok=-1),
], ids=str)
def test_append_factors_rejects_before_launch(over):
    args = dict(batch=1, n_tok=4, k_factors=A, v_factors=A, start_pos=A, capacity=64, kcache=A,
                vcache=A)
    args.update(over)
    with pytest.raises(kpa.KpaError) as e:
        kpa.kpa_append_factors(CFG, args["batch"], args["n_tok"], args["k_factors"],
                               args["v_factors"], args["start_pos"], args["capacity"],
                               args["kcache"], args["vcache"], stream=0)
    assert e.value.status == kpa.KPA_ERR_INVALID_ARG


def test_package_refuses_to_load_without_the_library(tmp_path):
    """The product path has no CPU fallback: without libkpa.so the import fails."""
    import shutil
    import subprocess
    import sys
    pkg = tmp_path / "factorised_kv_attention_b200"
    pkg.mkdir()
    src = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "factorised_kv_attention_b200",
                       "__init__.py")
    shutil.copy(src, pkg / "__init__.py")
    r = subprocess.run([sys.executable, "-c", "import factorised_kv_attention_b200"], cwd=tmp_path,
                       capture_output=True, text=True)
    assert r.returncode != 0 and "ImportError" in r.stderr and "libkpa.so" in r.stderr


PCFG = kpa.make_config(APPEND_PREFILL.shape, "bf16")


def _prefill(**over):
    args = dict(batch=2, n_tok=64, q=A, start_pos=A, kcache=A, vcache=A, capacity=128, sm_scale=0.1, out=A)
    args.update(over)
    kpa.kpa_prefill(PCFG, args["batch"], args["n_tok"], args["q"], args["start_pos"], args["kcache"],
                    args["vcache"], args["capacity"], args["sm_scale"], args["out"], stream=0)


@pytest.mark.parametrize("over", [
    dict(q=None), dict(start_pos=None), dict(kcache=None), dict(vcache=None), dict(out=None),
    dict(q=A + 2), dict(kcache=A + 8), dict(vcache=A + 4), dict(out=A + 4), dict(start_pos=A + 1),
    dict(capacity=60), dict(capacity=0), dict(batch=-1), dict(n_tok=-1),
    dict(sm_scale=float("nan")), dict(sm_scale=float("inf")),
], ids=str)
def test_prefill_rejects_before_launch(over):
    with pytest.raises(kpa.KpaError) as e:
        _prefill(**over)
    assert e.value.status == kpa.KPA_ERR_INVALID_ARG


def test_prefill_empty_is_a_no_op():
    _prefill(batch=0, q=None, start_pos=None, kcache=None, vcache=None, out=None)
    _prefill(n_tok=0, q=None, start_pos=None, kcache=None, vcache=None, out=None)


@pytest.mark.parametrize("stride", [dict(qf_stride=0), dict(qf_seq_stride=-1), dict(qf_tok_stride=-1)], ids=str)
def test_prefill_qf_rejects_bad_strides(stride):
    s = dict(qf_stride=1, qf_seq_stride=4096, qf_tok_stride=2)
    s.update(stride)
    with pytest.raises(kpa.KpaError) as e:
        kpa.kpa_prefill_qf(PCFG, 2, 64, A, s["qf_stride"], s["qf_seq_stride"], s["qf_tok_stride"], A, A, A, 128,
                           0.1, A, stream=0)
    assert e.value.status == kpa.KPA_ERR_INVALID_ARG


def _append(**over):
    args = dict(batch=2, n_tok=64, x=A, w=A, start_pos=A, capacity=128, kcache=A, vcache=A, q_out=None,
                workspace=None, ws_bytes=0)
    args.update(over)
    kpa.kpa_append(PCFG, args["batch"], args["n_tok"], args["x"], args["w"], args["start_pos"], args["capacity"],
                   args["kcache"], args["vcache"], args["q_out"], args["workspace"], args["ws_bytes"], stream=0)


@pytest.mark.parametrize("over", [
    dict(x=None), dict(w=None), dict(start_pos=None), dict(kcache=None), dict(vcache=None),
    dict(x=A + 2), dict(w=A + 8), dict(kcache=A + 4), dict(start_pos=A + 2), dict(q_out=A + 4),
    dict(capacity=12), dict(capacity=0), dict(batch=-1), dict(n_tok=-1),
], ids=str)
def test_append_rejects_before_launch(over):
    with pytest.raises(kpa.KpaError) as e:
        _append(**over)
    assert e.value.status == kpa.KPA_ERR_INVALID_ARG


def test_append_workspace_checked_before_launch():
    """q_out needs the workspace kpa_append_workspace_size gives (the query factors in fp32),
    256-byte aligned; an empty call is a no-op."""
    need = kpa.kpa_append_workspace_size(PCFG, 2, 64)
    e_q = APPEND_PREFILL.shape.r_q * (APPEND_PREFILL.shape.h1 * APPEND_PREFILL.shape.d1 +
                                      APPEND_PREFILL.shape.h2 * APPEND_PREFILL.shape.d2)
    assert need >= 2 * 64 * e_q * 4 and need % 256 == 0
    for over in (dict(q_out=A), dict(q_out=A, workspace=A, ws_bytes=need - 1), dict(workspace=A, ws_bytes=0)):
        with pytest.raises(kpa.KpaError) as e:
            _append(**over)
        assert e.value.status == kpa.KPA_ERR_WORKSPACE, over
    with pytest.raises(kpa.KpaError) as e:
        _append(q_out=A, workspace=A + 16, ws_bytes=need)
    assert e.value.status == kpa.KPA_ERR_INVALID_ARG
    _append(batch=0, x=None, w=None, start_pos=None, kcache=None, vcache=None)
