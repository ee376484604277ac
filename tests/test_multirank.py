"""The multi-rank path of bench.py on CPU: two gloo ranks, as torchrun would start
them, check the pieces that decide the reported numbers.

  - each rank draws its own batch (replicas shard the batch; no data exchange);
  - device times combine as the maximum over ranks, work as the sum over ranks;
  - the reference arm runs on rank 0 only: other ranks exit 0 without work or output;
  - a sequence split across the ranks: the ranges cover it exactly, and each rank's
    partial decode (the oracle's, over its range, with the normaliser) gathered over
    the process group and merged by the log-sum-exp rule is the whole sequence's decode.
"""
import contextlib
import io
import multiprocessing as mp
import os
import socket
import sys
import traceback

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    try:
        sys.path.insert(0, ROOT)
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                          WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
        from datetime import timedelta

        import torch.distributed as dist
        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
        import bench
        from workloads import KPA_MEDIUM, decode_inputs

        out = {}
        out["max"] = bench.max_over_ranks(1.5 + rank, world, "cpu")
        out["sum"] = bench.sum_over_ranks(100 * (rank + 1), world, "cpu")
        w = KPA_MEDIUM.replace(batch=4, capacity=2048, ragged=(16, 2048))
        lens = decode_inputs(w.replace(seed=bench.rank_seed(rank)))["seq_len"].tolist()
        gathered = [None] * world
        dist.all_gather_object(gathered, lens)
        out["lens"] = gathered
        # one sequence split across the ranks: keys stored rotated at their global positions
        import numpy as np
        import torch

        import oracle
        from workloads import KPA_LONG, to_f64
        ws = KPA_LONG.replace(capacity=304, length=300, seed=9)
        si = decode_inputs(ws)
        s = ws.shape
        kf, vf, q = to_f64(si["kf"]), to_f64(si["vf"]), to_f64(si["q"])
        kr = np.stack([[oracle.rotate_record(s.h1, s.h2, s.d1, s.d2, s.r_k, s.rope_base, t, kf[b, t])
                        for t in range(ws.capacity)] for b in range(ws.batch)])
        lo, hi = bench.split_range(300, world, rank)
        q_rot = np.stack([[oracle.rope_kpa(s.d1, s.d2, s.rope_base, 300, q[b, h]) for h in range(s.h)]
                          for b in range(ws.batch)])
        o_p, l_p = oracle.decode(s, q_rot, kr[:, lo:hi], vf[:, lo:hi], [hi - lo] * ws.batch, keys_rotated=True,
                                 return_lse=True)
        outs, lses = bench.gather_parts(torch.from_numpy(o_p), torch.from_numpy(l_p), world)
        outs, lses = outs.numpy(), lses.numpy()
        M = lses.max(axis=0)
        wgt = np.exp(lses - M)
        merged = (wgt[..., None] * outs).sum(axis=0) / wgt.sum(axis=0)[..., None]
        whole = oracle.decode(s, q, kf, vf, si["seq_len"].numpy(), q_pos=si["q_pos"].numpy())
        out["split_err"] = float(np.max(np.abs(merged - whole)))
        out["ranges"] = [bench.split_range(L, W, r) for L in (0, 1, 9, 300, 524288, 4101) for W in (1, 2, 3, 8)
                         for r in range(W)]
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            rc = bench.main(["--impl", "reference", "--steps", "1", "--warmup", "1"]) if rank != 0 else 0
        out["ref_rc"], out["ref_out"] = rc, buf.getvalue()
        dist.barrier()
        dist.destroy_process_group()
        results.put((rank, out, None))
    except Exception:
        results.put((rank, None, traceback.format_exc()))


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        rank, out, err = results.get(timeout=180)
        assert err is None, f"rank {rank} failed:\n{err}"
        got[rank] = out
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(world):
        assert got[rank]["max"] == 2.5                    # slowest rank's time on every rank
        assert got[rank]["sum"] == 300                    # both ranks' work
    lens = got[0]["lens"]
    assert lens == got[1]["lens"]
    assert lens[0] != lens[1], "replicas must draw different batches"
    assert got[1]["ref_rc"] == 0 and got[1]["ref_out"] == "", "reference arm runs on rank 0 only"
    for rank in range(world):
        assert got[rank]["split_err"] <= 1e-12, f"split-sequence merge: {got[rank]['split_err']}"
    # the ranges of a split cover [0, L) with contiguous, ordered, group-aligned pieces
    it = iter(got[0]["ranges"])
    for L in (0, 1, 9, 300, 524288, 4101):
        for W in (1, 2, 3, 8):
            ranges = [next(it) for _ in range(W)]
            assert ranges[0][0] == 0 and ranges[-1][1] == L
            for (a0, a1), (b0, b1) in zip(ranges[:-1], ranges[1:]):
                assert a1 == b0 and a0 <= a1 and (a1 % 8 == 0 or a1 == L)
