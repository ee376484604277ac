"""One sequence split into contiguous token ranges, as the ranks of a multi-GPU decode
hold it: each range in a cache of its own (slots from 0, keys rotated at their global
positions by kpa_append_factors_pos), decoded with the query's global position by
kpa_decode_lse, and the parts merged by kpa_merge_lse (the log-sum-exp merge).  On one
GPU the parts run one after the other; the result must be the decode of the whole
sequence (GPU)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_bf16_close, errors, fill_cache, kpa, oracle_decode_unrotated, planes, run_decode
from workloads import KPA_LONG, KPA_MEDIUM, TPA_DECODE, decode_inputs, to_f64

pytestmark = pytest.mark.gpu


def _parts(lib, w, inp, cuts):
    """Decode every range [cuts[i], cuts[i+1]) of each sequence on its own cache."""
    s = w.shape
    cfg = lib.make_config(s, w.dtype)
    scale = 1.0 / float(np.sqrt(s.dh))
    L = inp["seq_len"].numpy()
    outs, lses = [], []
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        n = hi - lo
        cap = max(8, (n + 7) // 8 * 8)
        kc, vc = planes(s, w.batch, cap, w.dtype)
        if n > 0:
            kf = inp["kf"][:, lo:hi].contiguous().cuda()
            vf = inp["vf"][:, lo:hi].contiguous().cuda()
            zero = torch.zeros(w.batch, dtype=torch.int32, device="cuda")
            off = torch.full((w.batch,), lo, dtype=torch.int32, device="cuda")
            lib.kpa_append_factors_pos(cfg, w.batch, n, kf, vf, zero, off, cap, kc, vc)
        seq = torch.from_numpy(np.clip(L - lo, 0, n).astype(np.int32)).cuda()      # this range of each sequence
        max_len = int(seq.max().item())
        ws = torch.zeros(max(lib.kpa_decode_workspace_size(cfg, w.batch, max_len), 256), dtype=torch.uint8,
                         device="cuda")
        out = torch.full((w.batch, s.h, s.dh), float("nan"), dtype=torch.float32, device="cuda")
        lse = torch.full((w.batch, s.h), float("nan"), dtype=torch.float32, device="cuda")
        lib.kpa_decode_lse(cfg, w.batch, inp["q"].cuda(), inp["q_pos"].cuda(), kc, vc, cap, seq, max_len, scale,
                           out, lse, ws)
        outs.append(out)
        lses.append(lse)
    outs_t, lses_t = torch.stack(outs).contiguous(), torch.stack(lses).contiguous()
    merged = torch.full_like(outs[0], float("nan"))
    merged_lse = torch.full_like(lses[0], float("nan"))
    lib.kpa_merge_lse(outs_t, lses_t, merged, merged_lse)
    torch.cuda.synchronize()
    assert lib.kpa_read_device_error() == 0
    return merged.cpu().numpy(), merged_lse.cpu().numpy(), outs_t.cpu().numpy(), lses_t.cpu().numpy()


CASES = {
    # the long-context shape at a reduced length: three ranges, the cuts off group boundaries
    "kpa_long": (KPA_LONG.replace(capacity=4104, length=4101, seed=81), [0, 1000, 2501, 4101]),
    # ragged batch: the last range is empty for the short sequences
    "kpa_medium": (KPA_MEDIUM.replace(batch=3, capacity=1536, ragged=(200, 1536), seed=82), [0, 700, 1100, 1536]),
    # TPA split, and an empty range in the middle
    "tpa": (TPA_DECODE.replace(batch=2, capacity=2048, length=2000, seed=83), [0, 900, 900, 2000]),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_split_sequence_matches_the_whole(name):
    w, cuts = CASES[name]
    lib = kpa()
    inp = decode_inputs(w)
    got, got_lse, outs, lses = _parts(lib, w, inp, cuts)
    scale = 1.0 / float(np.sqrt(w.shape.dh))
    want, want_lse = oracle.decode(w.shape, to_f64(inp["q"]), to_f64(inp["kf"]), to_f64(inp["vf"]),
                                   inp["seq_len"].numpy(), q_pos=inp["q_pos"].numpy(), sm_scale=scale,
                                   return_lse=True)
    assert_bf16_close(got, want, f"split {name}: merged output against the whole sequence")
    # the merged normaliser is the whole sequence's (natural log units)
    assert np.max(np.abs(got_lse - want_lse)) <= 1e-2, f"lse: {np.max(np.abs(got_lse - want_lse)):.3e}"
    # against the single-cache decode on the GPU: the same sums up to the split order
    cfg, kc, vc = fill_cache(lib, w, inp)
    whole = run_decode(lib, w, cfg, kc, vc, inp["q"], inp["seq_len"], inp["q_pos"]).cpu().numpy()
    max_abs, rel = errors(got, whole)
    assert max_abs <= 2e-5 and rel <= 1e-3, f"split {name} against kpa_decode: {max_abs:.2e} {rel:.2e}"
    # an empty range reports -inf and adds nothing
    L = inp["seq_len"].numpy()
    for p, (lo, hi) in enumerate(zip(cuts[:-1], cuts[1:])):
        for b in range(w.batch):
            if min(hi, L[b]) <= lo:
                assert np.all(np.isneginf(lses[p, b])), f"range {p} of sequence {b} is empty"


def test_merge_of_one_part_is_the_part():
    lib = kpa()
    g = torch.Generator().manual_seed(5)
    outs = torch.randn(1, 2, 4, 64, generator=g).cuda()
    lses = torch.randn(1, 2, 4, generator=g).cuda()
    out = torch.empty(2, 4, 64, device="cuda")
    lse = torch.empty(2, 4, device="cuda")
    lib.kpa_merge_lse(outs, lses, out, lse)
    torch.cuda.synchronize()
    assert torch.equal(out, outs[0]) and torch.equal(lse, lses[0])
