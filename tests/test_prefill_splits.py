"""kpa_prefill on Kronecker splits other than the append+prefill configuration's: the
TPA split (h1 = h, d1 = 1), R = 4, uneven ranks, d2 not a multiple of 4, d1 > d2, a
shared B and queries given as factors run on the mma.sync prefill; d1 = 8 with R = 4
and the KPA paper's section 3.2 splits (d1 = d2 = 8, R = 2) run on the tcgen05 prefill.  Each against the
float64 oracle, and both kernels on the splits the tcgen05 one takes (GPU)."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_bf16_close, kpa, natural, planes
from workloads import APPEND_PREFILL, KPA_MEDIUM, Shape, append_inputs, decode_inputs, to_f64

pytestmark = pytest.mark.gpu

SPLITS = {
    "tpa_h8_d1x64_r2": Shape(h1=8, h2=1, d1=1, d2=64, r_k=2, r_v=2),
    "tpa_h8_d1x128_rk3_rv2": Shape(h1=8, h2=1, d1=1, d2=128, r_k=3, r_v=2),
    "kpa_h4x4_d8x16_r4": Shape(h1=4, h2=4, d1=8, d2=16, r_k=4, r_v=4),
    "kpa_h2x8_d8x8_r2": Shape(h1=2, h2=8, d1=8, d2=8, r_k=2, r_v=2),
    "kpa_h10x2_d8x8_r2": Shape(h1=10, h2=2, d1=8, d2=8, r_k=2, r_v=2),
    "kpa_h4x4_d8x16_rk3_rv1": Shape(h1=4, h2=4, d1=8, d2=16, r_k=3, r_v=1),
    "kpa_h3x2_d4x6_r2": Shape(h1=3, h2=2, d1=4, d2=6, r_k=2, r_v=2),
    "kpa_h4x2_d16x4_r2": Shape(h1=4, h2=2, d1=16, d2=4, r_k=2, r_v=2),
}
# the tcgen05 kernel's split
C5_SPLIT = Shape(h1=4, h2=4, d1=8, d2=16, r_k=2, r_v=2)


def _kind(s):
    """The prefill kernel a split runs on by default."""
    if s.d1 == 8 and s.r_k == s.r_v and ((s.d2 == 16 and s.r_k in (2, 4)) or (s.d2 == 8 and s.r_k == 2)):
        return "tcgen05"
    return "mma_sync"


def _cache(lib, s, batch, cap, seed, factor_std=1.0 / np.sqrt(2.0)):
    """Random factor records in every slot of a fresh cache (slot = position)."""
    w = KPA_MEDIUM.replace(shape=s, batch=batch, capacity=cap, ragged=(), length=cap,
                           factor_std=factor_std, seed=seed)
    inp = decode_inputs(w)
    cfg = lib.make_config(s, "bf16")
    kc, vc = planes(s, batch, cap, "bf16")
    zero = torch.zeros(batch, dtype=torch.int32, device="cuda")
    lib.kpa_append_factors(cfg, batch, cap, inp["kf"].cuda(), inp["vf"].cuda(), zero, cap, kc, vc)
    return cfg, kc, vc


def _query(s, batch, n_tok, seed, std=0.3):
    rng = np.random.default_rng(seed)
    return torch.from_numpy((rng.standard_normal((batch, n_tok, s.h, s.dh)) * std).astype(np.float32)).to(
        torch.bfloat16)


def _prefill(lib, cfg, batch, n_tok, q, start, kc, vc, cap, scale):
    out = torch.full((batch, n_tok, q.shape[2], q.shape[3]), float("nan"), dtype=torch.float32, device="cuda")
    lib.kpa_prefill(cfg, batch, n_tok, q.cuda().contiguous(), start.cuda(), kc, vc, cap, scale, out)
    return out


def _oracle(s, q, kc, vc, batch, cap, starts, scale):
    kn = to_f64(natural(kc.cpu(), batch, cap, s.e_k))
    vn = to_f64(natural(vc.cpu(), batch, cap, s.e_v))
    if s.shared_b:
        a = s.r_k * s.h1 * s.d1                          # value record [A^V | B], B unrotated
        vn = np.concatenate([vn, kn[:, :, a:]], axis=2)
        return oracle.prefill(s, to_f64(q), kn, vn, starts, keys_rotated=False, sm_scale=scale)
    return oracle.prefill(s, to_f64(q), kn, vn, starts, keys_rotated=True, sm_scale=scale)


# (starts, n_tok): a ragged second 128-row tile with a start off the 64-slot grid; and
# three row tiles whose first sequence starts past two key tiles.
@pytest.mark.parametrize("starts,n_tok", [([0, 37], 200), ([130, 3], 300)], ids=["ragged", "offset"])
@pytest.mark.parametrize("name", list(SPLITS))
def test_prefill_split_against_oracle(name, starts, n_tok):
    lib = kpa()
    s = SPLITS[name]
    batch = len(starts)
    cap = max(512, (max(starts) + n_tok + 7) // 8 * 8)
    cfg, kc, vc = _cache(lib, s, batch, cap, seed=51)
    assert lib.kpa_prefill_kernel_kind(cfg) == _kind(s)
    q = _query(s, batch, n_tok, seed=8)
    start = torch.tensor(starts, dtype=torch.int32)
    scale = 1.0 / np.sqrt(s.dh)
    out = _prefill(lib, cfg, batch, n_tok, q, start, kc, vc, cap, scale)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    want = _oracle(s, q, kc, vc, batch, cap, starts, scale)
    assert_bf16_close(out.cpu().numpy(), want, f"prefill {name} starts={starts} n={n_tok}")


def test_prefill_split_sharp_scores():
    """Scores sharpened 40x on the R = 4 split: row maxima move from tile to tile, so
    the running output is rescaled at nearly every key tile."""
    lib = kpa()
    s = SPLITS["kpa_h4x4_d8x16_r4"]
    starts, n_tok, cap = [0, 64], 384, 512
    batch = len(starts)
    cfg, kc, vc = _cache(lib, s, batch, cap, seed=52)
    q = _query(s, batch, n_tok, seed=9)
    start = torch.tensor(starts, dtype=torch.int32)
    scale = 40.0 / np.sqrt(s.dh)
    out = _prefill(lib, cfg, batch, n_tok, q, start, kc, vc, cap, scale)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    assert_bf16_close(out.cpu().numpy(), _oracle(s, q, kc, vc, batch, cap, starts, scale), "sharp R=4 prefill")


def test_prefill_split_shared_b():
    """A shared B on the TPA split: K rebuilt with B rotated at each slot, V from the
    same B unrotated, against the oracle's plain definition (it rotates each key)."""
    lib = kpa()
    s = Shape(h1=8, h2=1, d1=1, d2=64, r_k=2, r_v=2, shared_b=1)
    starts, n_tok, cap = [0, 45], 260, 512
    batch = len(starts)
    cfg, kc, vc = _cache(lib, s, batch, cap, seed=53)
    assert lib.kpa_prefill_kernel_kind(cfg) == "mma_sync"
    q = _query(s, batch, n_tok, seed=10)
    start = torch.tensor(starts, dtype=torch.int32)
    scale = 1.0 / np.sqrt(s.dh)
    out = _prefill(lib, cfg, batch, n_tok, q, start, kc, vc, cap, scale)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    assert_bf16_close(out.cpu().numpy(), _oracle(s, q, kc, vc, batch, cap, starts, scale), "shared-B TPA prefill")


@pytest.mark.parametrize("s", [C5_SPLIT, SPLITS["kpa_h2x8_d8x8_r2"], SPLITS["kpa_h4x4_d8x16_r4"]],
                         ids=["d8x16", "d8x8", "d8x16_r4"])
def test_prefill_mma_kernel_on_the_tcgen05_split(s):
    """The tcgen05 kernel's splits, on both kernels (kpa_test_set_prefill_engine): each
    against the oracle, so the two prefill kernels are checked on one shape."""
    lib = kpa()
    starts, n_tok, cap = [0, 77], 400, 512
    batch = len(starts)
    cfg, kc, vc = _cache(lib, s, batch, cap, seed=54)
    q = _query(s, batch, n_tok, seed=11)
    start = torch.tensor(starts, dtype=torch.int32)
    scale = 1.0 / np.sqrt(s.dh)
    want = _oracle(s, q, kc, vc, batch, cap, starts, scale)
    assert lib.kpa_prefill_kernel_kind(cfg) == "tcgen05"
    try:
        lib.kpa_test_set_prefill_engine(1)
        assert lib.kpa_prefill_kernel_kind(cfg) == "mma_sync"
        out = _prefill(lib, cfg, batch, n_tok, q, start, kc, vc, cap, scale)
    finally:
        lib.kpa_test_set_prefill_engine(0)
    ref = _prefill(lib, cfg, batch, n_tok, q, start, kc, vc, cap, scale)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    assert_bf16_close(out.cpu().numpy(), want, "mma.sync prefill on the tcgen05 split")
    assert_bf16_close(ref.cpu().numpy(), want, "tcgen05 prefill")


def test_prefill_split_rows_outside_the_cache():
    """Rows whose position is at or past the capacity come back as zeros and raise the
    device-check error; the rows before them are still computed."""
    lib = kpa()
    s = SPLITS["tpa_h8_d1x64_r2"]
    batch, cap, n_tok = 2, 256, 150
    starts = [0, 200]                                   # sequence 1: rows 56.. are past slot 255
    cfg, kc, vc = _cache(lib, s, batch, cap, seed=55)
    q = _query(s, batch, n_tok, seed=12)
    start = torch.tensor(starts, dtype=torch.int32)
    scale = 1.0 / np.sqrt(s.dh)
    out = _prefill(lib, cfg, batch, n_tok, q, start, kc, vc, cap, scale).cpu().numpy()
    assert lib.kpa_read_device_error() == 6              # KPA_ERR_DEVICE_CHECK
    assert np.all(out[1, cap - starts[1]:] == 0.0)
    want = _oracle(s, q[:, :cap - starts[1]], kc, vc, batch, cap, starts, scale)
    assert_bf16_close(out[:, :cap - starts[1]], want, "rows inside the cache")


@pytest.mark.parametrize("name", ["tpa_h8_d1x64_r2", "kpa_h4x4_d8x16_r4"])
def test_prefill_split_from_query_factors(name):
    """kpa_append without q_out leaves the rotated query factors in its workspace;
    kpa_prefill_qf forms each query row from them on the mma.sync prefill.  Every row
    against the oracle with the float64 projection's query."""
    lib = kpa()
    s = dataclasses.replace(SPLITS[name], r_q=4, d_model=256)
    starts, n_tok = [0, 40], 300
    w = APPEND_PREFILL.replace(shape=s, batch=len(starts), n_tok=n_tok, capacity=384, seed=75)
    inp = append_inputs(w)
    cfg = lib.make_config(s, "bf16")
    kc, vc = planes(s, w.batch, w.capacity, "bf16")
    start = torch.tensor(starts, dtype=torch.int32)
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
    want = oracle.prefill(s, q_rot, kn, vn, starts, keys_rotated=True, sm_scale=scale)
    assert_bf16_close(out.cpu().numpy(), want, f"prefill from query factors, {name}")


def _bf16(a):
    """Round to bf16 (nearest even) and back to float64."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).to(torch.float32).to(
        torch.bfloat16).to(torch.float64).numpy()


@pytest.mark.parametrize("name", ["tpa_h8_d1x64_r2", "kpa_h4x4_d8x16_r4", "kpa_h2x8_d8x8_r2"])
def test_append_prefill_split_against_the_plain_definition(name):
    """kpa_append of a chunk (projection, factor RoPE, cache write, q_out) and the
    prefill from q_out, every row against oracle.append then oracle.prefill on the
    unrotated key records (the oracle rotates each reconstructed key at its slot), bf16
    at the two storage points (the cache records and q_out)."""
    lib = kpa()
    s = dataclasses.replace(SPLITS[name], r_q=4, d_model=256)
    w = APPEND_PREFILL.replace(shape=s, batch=2, n_tok=320, capacity=384, seed=76)
    inp = append_inputs(w)
    cfg = lib.make_config(s, "bf16")
    kc, vc = planes(s, w.batch, w.capacity, "bf16")
    start = torch.zeros(w.batch, dtype=torch.int32, device="cuda")
    ws = torch.zeros(lib.kpa_append_workspace_size(cfg, w.batch, w.n_tok), dtype=torch.uint8, device="cuda")
    q_out = torch.empty(w.batch, w.n_tok, s.h, s.dh, dtype=torch.bfloat16, device="cuda")
    lib.kpa_append(cfg, w.batch, w.n_tok, inp["x"].cuda(), inp["W"].cuda(), start, w.capacity, kc, vc, q_out, ws)
    scale = 1.0 / np.sqrt(s.dh)
    out = torch.full((w.batch, w.n_tok, s.h, s.dh), float("nan"), dtype=torch.float32, device="cuda")
    lib.kpa_prefill(cfg, w.batch, w.n_tok, q_out, start, kc, vc, w.capacity, scale, out)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    q_rot, _, v_rec, k_rec = oracle.append(s, to_f64(inp["x"]), to_f64(inp["W"]), np.zeros(w.batch, np.int64))
    want = oracle.prefill(s, _bf16(q_rot), _bf16(k_rec), _bf16(v_rec), [0] * w.batch, keys_rotated=False,
                          sm_scale=scale)
    assert_bf16_close(out.cpu().numpy(), want, f"append + prefill {name} against the plain definition")


@pytest.mark.parametrize("name", ["tpa_h8_d1x64_r2", "c5"])
def test_prefill_fp16_overflow_is_reported(name):
    """A cached factor whose rebuilt keys leave the fp16 range (an fp16 operand of the
    products) in a visible slot makes rows non-finite, which both prefill kernels
    report as KPA_ERR_DEVICE_CHECK."""
    lib = kpa()
    s = C5_SPLIT if name == "c5" else SPLITS[name]
    starts, n_tok, cap = [0, 0], 130, 256
    batch = len(starts)
    w = KPA_MEDIUM.replace(shape=s, batch=batch, capacity=cap, ragged=(), length=cap,
                           factor_std=1.0 / np.sqrt(2.0), seed=56)
    inp = decode_inputs(w)
    inp["kf"][1, 20, s.r_k * s.h1 * s.d1 + 3] = 1.0e6      # a B^K element of a visible slot
    cfg = lib.make_config(s, "bf16")
    kc, vc = planes(s, batch, cap, "bf16")
    zero = torch.zeros(batch, dtype=torch.int32, device="cuda")
    lib.kpa_append_factors(cfg, batch, cap, inp["kf"].cuda(), inp["vf"].cuda(), zero, cap, kc, vc)
    assert lib.kpa_prefill_kernel_kind(cfg) == ("tcgen05" if name == "c5" else "mma_sync")
    lib.kpa_read_device_error()                              # clear
    q = _query(s, batch, n_tok, seed=13)
    _prefill(lib, cfg, batch, n_tok, q, torch.tensor(starts, dtype=torch.int32), kc, vc, cap, 1.0 / np.sqrt(s.dh))
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == lib.KPA_ERR_DEVICE_CHECK
