"""kpa_prefill (causal attention with K/V rebuilt on chip from the factors, tcgen05)
against the float64 oracle, and the append + prefill + decode-step chain of the
append+prefill configuration (GPU)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_bf16_close, kpa, natural, planes, run_decode
from workloads import APPEND_PREFILL, KPA_MEDIUM, Shape, append_inputs, decode_inputs, to_f64

pytestmark = pytest.mark.gpu

SHAPE = Shape(h1=4, h2=4, d1=8, d2=16, r_k=2, r_v=2, r_q=6, d_model=2048, rope_base=10000.0)


def _prefill(lib, cfg, batch, n_tok, q, start, kc, vc, cap, sm_scale):
    out = torch.full((batch, n_tok, q.shape[2], q.shape[3]), float("nan"), dtype=torch.float32, device="cuda")
    lib.kpa_prefill(cfg, batch, n_tok, q.cuda().contiguous(), start.cuda(), kc, vc, cap, sm_scale, out)
    return out


# (starts, n_tok, score sharpening): one full 256-row pair; a ragged second half; two
# rows in the second half; three pairs whose last has no second half; a start past a
# key-tile boundary over several pairs; and scores sharpened 40x so that the row
# maxima keep growing from tile to tile and the conditional rescale runs.
@pytest.mark.parametrize("starts,n_tok,sharp", [([0, 0], 256, 1.0), ([0, 37], 200, 1.0), ([5, 300], 130, 1.0),
                                               ([0, 3], 600, 1.0), ([130, 0], 520, 1.0), ([0, 64], 384, 40.0)])
def test_prefill_against_oracle(starts, n_tok, sharp):
    """Random factors in the cache (earlier context + the chunk), random rotated q."""
    lib = kpa()
    s = SHAPE
    batch = len(starts)
    cap = max(512, (max(starts) + n_tok + 7) // 8 * 8)
    w = KPA_MEDIUM.replace(shape=s, batch=batch, capacity=cap, ragged=(), length=cap,
                           factor_std=1.0 / np.sqrt(2.0), seed=41)
    inp = decode_inputs(w)
    cfg = lib.make_config(s, "bf16")
    kc, vc = planes(s, batch, cap, "bf16")
    zero = torch.zeros(batch, dtype=torch.int32, device="cuda")
    lib.kpa_append_factors(cfg, batch, cap, inp["kf"].cuda(), inp["vf"].cuda(), zero, cap, kc, vc)
    rng = np.random.default_rng(7)
    q = torch.from_numpy((rng.standard_normal((batch, n_tok, s.h, s.dh)) * 0.3).astype(np.float32)).to(torch.bfloat16)
    start = torch.tensor(starts, dtype=torch.int32)
    scale = sharp / np.sqrt(s.dh)
    out = _prefill(lib, cfg, batch, n_tok, q, start, kc, vc, cap, scale)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    kn = to_f64(natural(kc.cpu(), batch, cap, s.e_k))
    vn = to_f64(natural(vc.cpu(), batch, cap, s.e_v))
    want = oracle.prefill(s, to_f64(q), kn, vn, starts, keys_rotated=True, sm_scale=scale)
    assert_bf16_close(out.cpu().numpy(), want, f"prefill starts={starts} n={n_tok} sharp={sharp}")


def test_prefill_rescale_when_the_maximum_jumps():
    """Each query is its own key scaled up, so a row's largest score arrives in its
    last (diagonal) key tile, far above the earlier tiles: the running maximum moves
    by more than 2^8 and the accumulated output is rescaled."""
    lib = kpa()
    s = SHAPE
    starts, n_tok, cap = [0, 64], 384, 512
    batch = len(starts)
    w = KPA_MEDIUM.replace(shape=s, batch=batch, capacity=cap, ragged=(), length=cap,
                           factor_std=1.0 / np.sqrt(2.0), seed=43)
    inp = decode_inputs(w)
    cfg = lib.make_config(s, "bf16")
    kc, vc = planes(s, batch, cap, "bf16")
    zero = torch.zeros(batch, dtype=torch.int32, device="cuda")
    lib.kpa_append_factors(cfg, batch, cap, inp["kf"].cuda(), inp["vf"].cuda(), zero, cap, kc, vc)
    kn = to_f64(natural(kc.cpu(), batch, cap, s.e_k))
    vn = to_f64(natural(vc.cpu(), batch, cap, s.e_v))
    q = np.empty((batch, n_tok, s.h, s.dh))
    for b in range(batch):
        for t in range(n_tok):
            q[b, t] = 16.0 * oracle.reconstruct(s.h1, s.h2, s.d1, s.d2, s.r_k, kn[b, starts[b] + t])
    q = torch.from_numpy(q.astype(np.float32)).to(torch.bfloat16)
    scale = 1.0 / np.sqrt(s.dh)
    out = _prefill(lib, cfg, batch, n_tok, q, torch.tensor(starts, dtype=torch.int32), kc, vc, cap, scale)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    want = oracle.prefill(s, to_f64(q), kn, vn, starts, keys_rotated=True, sm_scale=scale)
    # the self-score dominates: the output is close to the row's own value
    assert_bf16_close(out.cpu().numpy(), want, "prefill, maximum jumps on the diagonal")


def test_prefill_rows_match_decode():
    """Row t of a prefill equals a decode of length start + t + 1 (both on the GPU)."""
    lib = kpa()
    s = SHAPE
    batch, cap, n_tok = 2, 512, 160
    w = KPA_MEDIUM.replace(shape=s, batch=batch, capacity=cap, ragged=(), length=cap, seed=42)
    inp = decode_inputs(w)
    cfg = lib.make_config(s, "bf16")
    kc, vc = planes(s, batch, cap, "bf16")
    zero = torch.zeros(batch, dtype=torch.int32, device="cuda")
    lib.kpa_append_factors(cfg, batch, cap, inp["kf"].cuda(), inp["vf"].cuda(), zero, cap, kc, vc)
    q = (torch.randn(batch, n_tok, s.h, s.dh, generator=torch.Generator().manual_seed(3)) * 0.3).to(torch.bfloat16)
    start = torch.tensor([0, 100], dtype=torch.int32)
    scale = 1.0 / np.sqrt(s.dh)
    pre = _prefill(lib, cfg, batch, n_tok, q, start, kc, vc, cap, scale).cpu().numpy()
    for t in (0, 1, 63, 127, 128, 159):
        L = start + t + 1
        dec = run_decode(lib, w, cfg, kc, vc, q[:, t], L, None, max_len=int(L.max()), sm_scale=scale)
        assert_bf16_close(pre[:, t], dec.cpu().numpy(), f"row {t}")


def test_append_prefill_decode_chain_full_config():
    """Configuration 5: append the 2048-token chunk (projection, RoPE, cache write),
    causal prefill from q_out, then one decode step at position 2048; sampled rows
    against the oracle fed with the GPU's bf16 q_out and cache."""
    lib = kpa()
    w = APPEND_PREFILL
    s = w.shape
    inp = append_inputs(w)
    cfg = lib.make_config(s, "bf16")
    kc, vc = planes(s, w.batch, w.capacity, "bf16")
    start = torch.zeros(w.batch, dtype=torch.int32, device="cuda")
    ws = torch.zeros(lib.kpa_append_workspace_size(cfg, w.batch, w.n_tok), dtype=torch.uint8, device="cuda")
    q_out = torch.empty(w.batch, w.n_tok, s.h, s.dh, dtype=torch.bfloat16, device="cuda")
    lib.kpa_append(cfg, w.batch, w.n_tok, inp["x"].cuda(), inp["W"].cuda(), start, w.capacity, kc, vc, q_out, ws)
    scale = 1.0 / np.sqrt(s.dh)
    out = torch.empty(w.batch, w.n_tok, s.h, s.dh, dtype=torch.float32, device="cuda")
    lib.kpa_prefill(cfg, w.batch, w.n_tok, q_out, start, kc, vc, w.capacity, scale, out)
    # decode step: append token 2048 of every sequence, attend over 2049 slots
    ws1 = torch.zeros(max(lib.kpa_append_workspace_size(cfg, w.batch, 1), 256), dtype=torch.uint8, device="cuda")
    q1 = torch.empty(w.batch, 1, s.h, s.dh, dtype=torch.bfloat16, device="cuda")
    pos = torch.full((w.batch,), w.n_tok, dtype=torch.int32, device="cuda")
    lib.kpa_append(cfg, w.batch, 1, inp["x_step"].cuda(), inp["W"].cuda(), pos, w.capacity, kc, vc, q1, ws1)
    seq = torch.full((w.batch,), w.n_tok + 1, dtype=torch.int32)
    dw = APPEND_PREFILL  # decode on the same cache
    from workloads import DecodeWorkload
    dwl = DecodeWorkload(name="c5 step", shape=s, batch=w.batch, capacity=w.capacity, dtype="bf16",
                         factor_std=0, q_std=0, length=w.n_tok + 1)
    dec = run_decode(lib, dwl, cfg, kc, vc, q1[:, 0], seq, None, sm_scale=scale)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    kn = to_f64(natural(kc.cpu(), w.batch, w.capacity, s.e_k))
    vn = to_f64(natural(vc.cpu(), w.batch, w.capacity, s.e_v))
    qo = to_f64(q_out.cpu())
    got = out.cpu().numpy()
    rng = np.random.default_rng(5)
    rows = [(int(b), int(t)) for b, t in zip(rng.integers(0, w.batch, 12), rng.integers(0, w.n_tok, 12))]
    rows += [(0, 0), (1, 127), (2, 128), (7, w.n_tok - 1)]
    for b, t in rows:
        want = oracle.decode(s, qo[b, t][None], kn[b][None], vn[b][None], [t + 1], keys_rotated=True,
                             sm_scale=scale)
        assert_bf16_close(got[b, t], want[0], f"prefill row ({b},{t})")
    want = oracle.decode(s, to_f64(q1[:, 0].cpu()), kn, vn, seq.numpy(), keys_rotated=True, sm_scale=scale)
    assert_bf16_close(dec.cpu().numpy(), want, "decode step at 2048")


@pytest.mark.parametrize("n_tok,starts", [(300, [0, 40]), (2048, [0, 0])], ids=["ragged", "chunk2048"])
def test_prefill_from_query_factors(n_tok, starts):
    """kpa_append without q_out leaves the rotated query factors in its workspace;
    kpa_prefill_qf assembles each query row from them in the kernel (fp32, one fp16
    rounding).  Sampled rows against the oracle with the float64 projection's query."""
    lib = kpa()
    s = APPEND_PREFILL.shape if n_tok == 2048 else Shape(h1=4, h2=4, d1=8, d2=16, r_k=2, r_v=2, r_q=6,
                                                          d_model=256, rope_base=10000.0)
    w = APPEND_PREFILL.replace(shape=s, batch=len(starts), n_tok=n_tok, capacity=max(512, n_tok + 64), seed=73)
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
    got = out.cpu().numpy()
    rng = np.random.default_rng(9)
    rows = [(int(b), int(t)) for b, t in zip(rng.integers(0, w.batch, 10), rng.integers(0, n_tok, 10))]
    rows += [(0, 0), (w.batch - 1, 127), (w.batch - 1, 128), (w.batch - 1, n_tok - 1)]
    for b, t in rows:
        L = int(start[b]) + t + 1
        want = oracle.decode(s, q_rot[b, t][None], kn[b][None], vn[b][None], [L], keys_rotated=True,
                             sm_scale=scale)
        assert_bf16_close(got[b, t], want[0], f"prefill from query factors, row ({b},{t})")


def _gpu_chain(lib, w, inp):
    """The append+prefill path as the library runs it: kpa_append of the chunk (q_out),
    kpa_prefill from q_out, then the decode step (kpa_append of token n_tok with its
    query factors left in the workspace, kpa_decode_qf over n_tok + 1 slots)."""
    s = w.shape
    cfg = lib.make_config(s, "bf16")
    kc, vc = planes(s, w.batch, w.capacity, "bf16")
    start = torch.zeros(w.batch, dtype=torch.int32, device="cuda")
    ws = torch.zeros(lib.kpa_append_workspace_size(cfg, w.batch, w.n_tok), dtype=torch.uint8, device="cuda")
    q_out = torch.empty(w.batch, w.n_tok, s.h, s.dh, dtype=torch.bfloat16, device="cuda")
    W = inp["W"].cuda()
    lib.kpa_append(cfg, w.batch, w.n_tok, inp["x"].cuda(), W, start, w.capacity, kc, vc, q_out, ws)
    scale = 1.0 / np.sqrt(s.dh)
    out = torch.full((w.batch, w.n_tok, s.h, s.dh), float("nan"), dtype=torch.float32, device="cuda")
    lib.kpa_prefill(cfg, w.batch, w.n_tok, q_out, start, kc, vc, w.capacity, scale, out)
    ws1 = torch.zeros(max(lib.kpa_append_workspace_size(cfg, w.batch, 1), 256), dtype=torch.uint8, device="cuda")
    pos = torch.full((w.batch,), w.n_tok, dtype=torch.int32, device="cuda")
    lib.kpa_append(cfg, w.batch, 1, inp["x_step"].cuda(), W, pos, w.capacity, kc, vc, None, ws1)
    seq = torch.full((w.batch,), w.n_tok + 1, dtype=torch.int32, device="cuda")
    wsd = torch.zeros(max(lib.kpa_decode_workspace_size(cfg, w.batch, w.n_tok + 1), 256), dtype=torch.uint8,
                      device="cuda")
    step = torch.full((w.batch, s.h, s.dh), float("nan"), dtype=torch.float32, device="cuda")
    lib.kpa_decode_qf(cfg, w.batch, ws1.view(torch.float32), w.batch, 1, None, kc, vc, w.capacity, seq,
                      w.n_tok + 1, scale, step, wsd)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    return out.cpu().numpy(), step.cpu().numpy(), scale


def _bf16(a):
    """Round to bf16 (nearest even) and back to float64."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).to(torch.float32).to(
        torch.bfloat16).to(torch.float64).numpy()


def _oracle_records(w, inp):
    """oracle.append of the chunk and of the decode step's token: the query rotated by
    the oracle on its reconstruction, and the unrotated key and value records of slots
    0 .. n_tok (the oracle rotates each key reconstruction itself when it attends).

    The configuration stores bf16 factors, so the end-to-end oracle rounds to bf16 at
    the two storage points, the cache records and the chunk's q_out (the pages fix no
    rounding points; these are where the library stores bf16); the decode step's query is assembled from fp32
    factors and is not rounded.  The library rounds a key record after rotating its B,
    the oracle before (it rotates the reconstruction): one bf16 rounding apart, which
    the oracle alone puts at 4e-4 relative on this configuration."""
    s = w.shape
    start = np.zeros(w.batch, dtype=np.int64)
    q_rot, _, v_rec, k_rec = oracle.append(s, to_f64(inp["x"]), to_f64(inp["W"]), start)
    q1, _, v1, k1 = oracle.append(s, to_f64(inp["x_step"]), to_f64(inp["W"]), start + w.n_tok)
    kf = _bf16(np.concatenate([k_rec, k1], axis=1))
    vf = _bf16(np.concatenate([v_rec, v1], axis=1))
    return _bf16(q_rot), kf, vf, q1[:, 0]


def test_append_prefill_decode_chain_against_the_plain_definition_every_row():
    """The append+prefill configuration's shape at 2 x 512 tokens, end to end: every
    prefill row and the decode step against oracle.append then oracle.prefill /
    oracle.decode on the unrotated key records (keys_rotated=False: the oracle applies
    RoPE to each reconstructed key at its slot), bf16 at the storage points."""
    lib = kpa()
    w = APPEND_PREFILL.replace(batch=2, n_tok=512, capacity=576, seed=11)
    inp = append_inputs(w)
    got, step, scale = _gpu_chain(lib, w, inp)
    q_rot, kf, vf, q1 = _oracle_records(w, inp)
    want = oracle.prefill(w.shape, q_rot, kf, vf, [0] * w.batch, keys_rotated=False, sm_scale=scale)
    assert_bf16_close(got, want, "prefill, every row, against the plain definition")
    want1 = oracle.decode(w.shape, q1, kf, vf, [w.n_tok + 1] * w.batch, keys_rotated=False, sm_scale=scale)
    assert_bf16_close(step, want1, "decode step against the plain definition")


def test_append_prefill_decode_chain_full_config_against_the_plain_definition():
    """Configuration 5 at full size, end to end: 64 sampled prefill rows (and the first
    and last rows of two sequences) and the decode step of all 8 sequences against
    oracle.append then the oracle's attention on the unrotated key records."""
    lib = kpa()
    w = APPEND_PREFILL
    s = w.shape
    inp = append_inputs(w)
    got, step, scale = _gpu_chain(lib, w, inp)
    q_rot, kf, vf, q1 = _oracle_records(w, inp)
    rng = np.random.default_rng(12)
    rows = sorted({(int(b), int(t)) for b, t in zip(rng.integers(0, w.batch, 64), rng.integers(0, w.n_tok, 64))})
    rows += [(0, 0), (0, w.n_tok - 1), (w.batch - 1, 0), (w.batch - 1, w.n_tok - 1)]
    for b, t in rows:
        want = oracle.attend(s, q_rot[b, t][None, None], kf[b][None], vf[b][None], [[t + 1]],
                             keys_rotated=False, sm_scale=scale)
        assert_bf16_close(got[b, t], want[0, 0], f"prefill row ({b},{t}) against the plain definition")
    want1 = oracle.decode(s, q1, kf, vf, [w.n_tok + 1] * w.batch, keys_rotated=False, sm_scale=scale)
    assert_bf16_close(step, want1, "decode step at 2048 against the plain definition")
