"""The multi-rank path of bench.py on CPU: two gloo ranks, as torchrun would start
them, check the pieces that decide the reported numbers.

  - each rank draws its own batch (replicas shard the batch; no data exchange);
  - device times combine as the maximum over ranks, work as the sum over ranks;
  - the reference arm runs on rank 0 only: other ranks exit 0 without work or output.
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
