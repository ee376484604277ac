"""Decode benchmark for factor-space KPA / TPA attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kpa|reference]
                    [--workload tpa_decode|tpa_shared|kpa_medium|kpa_long|tiny_kpa|flashtpa|append_prefill]
                    [--layers L]

A step is one decode pass of a model of L attention layers over one batch: per
layer, kpa_decode of one query row per sequence against that layer's own factor
cache (rotation of the query, factor-space scores, online softmax, value
accumulation, split combine).  Each layer has its own cache, so a step streams
L x (cache bytes) through HBM and the L2 (126 MB) holds none of it between uses.
The whole step is one CUDA graph.  Throughput is cached tokens attended per
second per layer, summed over ranks; each rank runs its own replica (the batch
shards with no exchange).

Printed: one JSON line (rank 0) with the metric, the roofline of the decode
kernel against the measured HBM copy bandwidth, the float64 CPU oracle timed on
a bounded sample (cpu_baseline), an end-to-end figure through the public API with
host buffers (e2e), SM clocks sampled during the timed region, and the number of
library kernel launches in the timed region.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode cached-tokens/s per layer; achieved HBM GB/s vs B200 peak (1 GPU)"
PEAKS = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC = os.path.join(ROOT, "profiles", "decode_traffic.json")
KERNEL_SOURCES = ["factorised_kv_attention_b200/csrc/kpa_decode_mma.cu",
                  "factorised_kv_attention_b200/csrc/kpa_mma_decode.cuh",
                  "factorised_kv_attention_b200/csrc/kpa_decode_fma.cu",
                  "factorised_kv_attention_b200/csrc/kpa_internal.cuh",
                  "factorised_kv_attention_b200/csrc/kpa_decode_merge.cuh",
                  "factorised_kv_attention_b200/csrc/kpa_f32x2.cuh",
                  "factorised_kv_attention_b200/csrc/kpa_sm100.cuh"]
FALLBACK_HBM_GBS = 6650.0


def _args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["kpa", "reference"], default="kpa")
    ap.add_argument("--workload", default="kpa_long",
                    help="tpa_decode | tpa_shared | tpa_order3 | kpa_medium | kpa_long | tiny_kpa | flashtpa | "
                         "tpa_h61 | tpa_h16_d1x128 | kpa_h4x4_d8x16_r4 | kpa_h{4x4,2x8,8x2,4x5,2x10,10x2}_d8x8 | "
                         "append_prefill")
    ap.add_argument("--layers", type=int, default=0,
                    help="0 = enough layer caches to exceed 4 x L2 (at least 2)")
    ap.add_argument("--decode-engine", type=int, default=0, choices=(0, 1, 2),
                    help="1: the opt-in tcgen05 decode for the TPA shape h=16, d_h=64, R=2; 2: the factored "
                         "score on CUDA cores (with --query-factors) (measurement)")
    ap.add_argument("--query-factors", action="store_true",
                    help="decode from the query's factors (kpa_decode_qf) instead of a dense query")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seq-len", type=int, default=0, help="override: fixed length (profiling)")
    ap.add_argument("--batch", type=int, default=0, help="override: batch (profiling; append_prefill too)")
    ap.add_argument("--tokens-per-split", type=int, default=0,
                    help="override the library's split of each sequence (profiling; multiple of 64)")
    ap.add_argument("--split-sequence", action="store_true",
                    help="one sequence split across the ranks: each rank holds a contiguous range of its tokens, "
                         "decodes it with kpa_decode_lse, and the parts are all-gathered and merged "
                         "(strong scaling)")
    ap.add_argument("--sweep", choices=["flashtpa"], default=None,
                    help="flashtpa: the FlashTPA decoding shape over sequence lengths 2^12..2^19 and batch "
                         "1, 2, 4, 8, 16 (one JSON line per point, then none of the other lines)")
    ap.add_argument("--prefill-split", default="kpa_h4x4_d8x16_r2",
                    choices=["kpa_h4x4_d8x16_r2", "tpa_h16_d1x128_r2", "kpa_h4x4_d8x16_r4", "kpa353m_h4x4_d8x8_r2"],
                    help="append_prefill: the Kronecker split of its h=16, d_h=128, or the KPA paper's 353M split "
                         "(d_model 1024, d_h=8x8); the tcgen05 prefill takes the d1=8, R=2 splits, the mma.sync "
                         "prefill the others")
    ap.add_argument("--prefill-engine", type=int, default=0, choices=(0, 1),
                    help="1: the mma.sync prefill on every split (measurement)")
    ap.add_argument("--settle-seconds", type=float, default=1.0,
                    help="untimed load before timing while clocks are sampled (0 for profiling)")
    a = ap.parse_args(argv)
    a.warmup = max(a.warmup, 3)
    if a.decode_engine == 1 and a.query_factors:
        ap.error("--decode-engine 1 (tcgen05) takes dense queries only")
    if a.decode_engine == 2 and not a.query_factors:
        ap.error("--decode-engine 2 (the factored score) needs --query-factors")
    if a.query_factors and a.tokens_per_split:
        ap.error("--query-factors takes the library's split (no --tokens-per-split)")
    return a


def _dist():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def rank_seed(rank: int, layer: int = 0) -> int:
    """Seed of a rank's replica inputs: every rank draws its own batch."""
    return 1000 * rank + layer


def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's value (device times are taken as the max over ranks)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int, device) -> float:
    """Work summed over ranks (each replica processes its own batch)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def split_range(length: int, world: int, rank: int):
    """The contiguous token range [lo, hi) of a sequence that rank `rank` of `world` holds:
    equal ranges of whole 8-slot groups, the last rank taking the remainder."""
    per = (length + world - 1) // world
    per = (per + 7) // 8 * 8
    lo = min(length, rank * per)
    return lo, min(length, lo + per)


def gather_parts(out, lse, world):
    """Every rank's partial decode (out [B][h][d_h], lse [B][h]) gathered in rank order:
    ([world][B][h][d_h], [world][B][h]).  The one exchange of a split sequence."""
    import torch
    if world == 1:
        return out[None], lse[None]
    import torch.distributed as dist
    outs = [torch.empty_like(out) for _ in range(world)]
    lses = [torch.empty_like(lse) for _ in range(world)]
    dist.all_gather(outs, out.contiguous())
    dist.all_gather(lses, lse.contiguous())
    return torch.stack(outs), torch.stack(lses)


def _kernel_hash():
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _hbm_peak():
    try:
        with open(PEAKS) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _traffic(kernel_hash, workload):
    """DRAM bytes per launch from the committed ncu records, when one was taken on this
    workload and on the current decode sources (else None)."""
    try:
        with open(TRAFFIC) as f:
            t = json.load(f)
    except Exception:
        return None
    for r in t.get("records", []):
        if r.get("kernel_sources_sha") == kernel_hash and r.get("workload") == workload:
            return r.get("dram_bytes_per_launch")
    return None


class ClockSampler:
    """SM clock and throttle reasons via NVML (read only), sampled every 50 ms."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle"}

    def __init__(self, device_index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            handle = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                hd = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(hd)
                u = u.decode() if isinstance(u, bytes) else u
                if uuid in u or u.endswith(uuid):
                    handle = hd
            if handle is None:
                handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nvml, self.handle = pynvml, handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report what we could not sample
            self.error = str(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nvml.nvmlDeviceGetClockInfo(self.handle, self.nvml.NVML_CLOCK_SM)
                mask = self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append(mhz)
                for bit, name in self.REASONS.items():
                    if mask & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(0.05)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


def _workload(name, a=None):
    from workloads import DECODE_CONFIGS
    w = DECODE_CONFIGS[name]
    if a is not None and a.seq_len:
        cap = (a.seq_len + 7) // 8 * 8
        w = w.replace(length=a.seq_len, ragged=(), capacity=cap,
                      name=w.name + f" [length overridden to {a.seq_len}]")
    if a is not None and a.batch:
        w = w.replace(batch=a.batch, name=w.name + f" [batch overridden to {a.batch}]")
    return w


def _config_json(w, layers, lens, world):
    cache_bytes = int(sum(lens)) * (w.shape.e_k + w.shape.e_v) * (2 if w.dtype == "bf16" else 4)
    return {"workload": w.name, "batch": w.batch, "seq_len": int(max(lens)),
            "mean_seq_len": float(np.mean(lens)), "layers": layers,
            "factor_cache_bytes_per_layer": cache_bytes,
            "l2": f"inputs larger than L2: {layers} distinct layer caches, "
                  f"{layers * cache_bytes / 1e6:.0f} MB per step per GPU",
            "parallelism": f"replicas x{world} (batch-sharded, no exchange)",
            "accumulate": "fp32"}


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def _cpu_baseline(w, inp, seconds, steps=None, q_factors=None, call_seconds=2.5, single_thread=True):
    """The float64 oracle, as it stands, on the workload's sequences.  A call decodes one
    sequence's query over its first n slots: the whole sequence when that fits in about
    call_seconds, else a prefix of it sized from a first short call (the work per slot
    is the same).  Calls run over the sequences in turn until `seconds` have passed (or
    `steps` calls); then, unless single_thread is False, the same for a share of the time
    on one core.  With q_factors ([B][E_Q]) the query is assembled from them first (eq 2
    for Q).  Returns the line's cpu_baseline object and the per-call times (all cores)."""
    import oracle
    from workloads import to_f64
    oracle.build()
    s = w.shape
    L, qp = inp["seq_len"].numpy(), inp["q_pos"].numpy()
    if q_factors is not None:
        qf64 = to_f64(q_factors)
        q_of = lambda b: oracle.reconstruct(s.h1, s.h2, s.d1, s.d2, s.r_q, qf64[b])[None]   # noqa: E731
    else:
        q_of = lambda b: to_f64(inp["q"][b:b + 1])                                        # noqa: E731
    fn = oracle.decode_order3 if s.order == 3 else oracle.decode_shared_b if s.shared_b else oracle.decode

    def call(b, n):
        q = q_of(b)
        kf, vf = to_f64(inp["kf"][b:b + 1, :n]), to_f64(inp["vf"][b:b + 1, :n])
        t0 = time.perf_counter()
        fn(s, q, kf, vf, np.array([n], dtype=np.int32), q_pos=qp[b:b + 1])
        return time.perf_counter() - t0

    def leg(budget, n_calls):
        n_probe = int(min(L.max(), 512))
        rate = n_probe / max(call(int(np.argmax(L)), n_probe), 1e-6)          # slots per second
        n_max = max(64, int(rate * call_seconds))
        done, t_total, times, n_seq, n_prefix, b = 0, 0.0, [], 0, 0, 0
        while (n_calls is None and t_total < budget) or (n_calls is not None and len(times) < n_calls):
            n = int(min(L[b], n_max))
            if n > 0:
                dt = call(b, n)
                times.append(dt)
                t_total += dt
                done += n
                n_seq += 1
                n_prefix += n < L[b]
            b = (b + 1) % w.batch
        return done / t_total, t_total, times, n_seq, n_prefix, n_max

    cores = oracle.max_threads()
    value, t_all, times, n_seq, n_prefix, n_max = leg(seconds, steps)
    what = (f"{n_seq} calls of one layer's decode (all {s.h} heads) over the workload's sequences in turn, "
            + (f"{n_prefix} of them over a prefix of at most {n_max} slots, " if n_prefix else "whole sequences, ")
            + f"float64 C oracle, OpenMP over heads, {t_all:.1f} s")
    base = {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": what,
            "cpu_model": _cpu_model(), "cpus_in_affinity": len(os.sched_getaffinity(0))}
    if single_thread:
        oracle.set_threads(1)
        try:
            v1, t1, _, n1, p1, m1 = leg(max(seconds / 2, 1.0), None if steps is None else max(1, steps // 4))
        finally:
            oracle.set_threads(cores)
        base["single_thread"] = {"value": v1, "unit": "tokens/s", "cores": 1,
                                 "sample": f"{n1} calls, {p1} over a prefix of at most {m1} slots, {t1:.1f} s"}
    return base, times


def _cpu_baseline_prefill(w, inp, seconds, steps=None, call_seconds=2.5):
    """The float64 oracle on the append+prefill workload: a call takes the first n
    prompt tokens of one sequence through oracle.append (projection, the rank-major
    split, RoPE on the B factors and on the assembled query) and oracle.prefill (each
    row over the block's slots up to its own).  n is the largest of 2048, 1024, ... 64
    whose time, scaled from a 64-token call by the prefill's n^2, fits call_seconds.
    Calls run over the sequences in turn until `seconds` pass (or `steps` calls)."""
    import oracle
    from workloads import to_f64
    oracle.build()
    s = w.shape
    x, W = to_f64(inp["x"]), to_f64(inp["W"])
    scale = 1.0 / float(np.sqrt(s.dh))

    def call(b, n):
        t0 = time.perf_counter()
        q_rot, k_rot, v_rec, _ = oracle.append(s, x[b:b + 1, :n], W, [0])
        oracle.prefill(s, q_rot, k_rot, v_rec, [0], keys_rotated=True, sm_scale=scale)
        return time.perf_counter() - t0

    t64 = max(call(0, 64), 1e-6)
    n = 64
    while n < w.n_tok and t64 * (2 * n / 64) ** 2 <= call_seconds:
        n *= 2
    n = min(n, w.n_tok)
    done, t_total, times, b = 0, 0.0, [], 0
    while (steps is None and t_total < seconds) or (steps is not None and len(times) < steps):
        dt = call(b, n)
        times.append(dt)
        t_total += dt
        done += n
        b = (b + 1) % w.batch
    return {"value": done / t_total, "unit": "tokens/s", "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"{len(times)} calls of the first {n} prompt tokens of one sequence (of {w.n_tok}): float64 "
                      f"projection, RoPE and causal prefill over the block, OpenMP over heads, {t_total:.1f} s",
            "cpu_model": _cpu_model()}, times


def run_reference(a):
    rank, world, _ = _dist()
    if rank != 0:
        return 0
    if a.workload == "append_prefill":
        from workloads import APPEND_PREFILL_SPLITS, append_inputs
        w = APPEND_PREFILL_SPLITS[a.prefill_split]
        inp = append_inputs(w)
        per_call = min(2.5, 120.0 / max(a.steps + a.warmup, 1))
        _cpu_baseline_prefill(w, inp, 0, steps=a.warmup, call_seconds=per_call)
        base, times = _cpu_baseline_prefill(w, inp, 0, steps=a.steps, call_seconds=per_call)
        line = {"impl": "reference", "metric": "append + causal prefill + decode step, tokens/s (2048-token chunks); "
                                              "TFLOP/s vs B200 bf16 peak",
                "value": base["value"], "unit": "tokens/s", "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
                "ms_per_step": 1e3 * float(np.sum(times)) / max(len(times), 1), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": w.name, "batch": w.batch, "seq_len": w.n_tok, "d_model": w.shape.d_model,
                           "sample": "one call per step: a block of prompt tokens of one sequence"},
                "cpu_baseline": base,
                "e2e": {"value": base["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0
    from workloads import decode_inputs
    w = _workload(a.workload, a)
    inp = decode_inputs(w)
    # each step one bounded call, sized so warm-up and steps take about two minutes
    per_call = min(2.5, 120.0 / max(a.steps + a.warmup, 1))
    _cpu_baseline(w, inp, 0, steps=a.warmup, call_seconds=per_call, single_thread=False)
    base, times = _cpu_baseline(w, inp, 0, steps=a.steps, call_seconds=per_call, single_thread=False)
    L = inp["seq_len"].numpy()
    value = base["value"]
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
            "ms_per_step": 1e3 * float(np.sum(times)) / max(len(times), 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": _config_json(w, 1, L, 1),
            "cpu_baseline": base,
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    line["config"]["sample"] = "one decode call of one layer per step (a whole sequence, or a prefix of it)"
    print(json.dumps(line), flush=True)
    return 0


def run_kpa(a):
    import torch
    import torch.distributed as dist

    rank, world, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=dev)

    import factorised_kv_attention_b200 as kpa
    from workloads import decode_inputs, query_factor_inputs

    w = _workload(a.workload, a)
    s = w.shape
    qf_mode = a.query_factors            # the query as its factors, through kpa_decode_qf
    if qf_mode and s.r_q <= 0:
        raise SystemExit(f"--query-factors: the {a.workload} shape has no query factors (r_q = 0)")
    elt = 2 if w.dtype == "bf16" else 4
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    first = decode_inputs(w.replace(seed=rank_seed(rank)))
    lens = first["seq_len"].numpy()
    layer_bytes = int(lens.sum()) * (s.e_k + s.e_v) * elt
    layers = a.layers or max(2, int(np.ceil(4 * l2 / max(layer_bytes, 1))))
    cfg = kpa.make_config(s, w.dtype)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    kpa.kpa_test_set_decode_engine(a.decode_engine)

    # per-layer caches, filled through kpa_append_factors (slot = position)
    kcs, vcs = [], []
    # every layer's query and output are views of one buffer each, so a step's inputs
    # and results move between host and device in one copy each way
    q_all = (torch.empty(layers, w.batch, s.e_q, dtype=torch.float32, device=dev) if qf_mode
             else torch.empty(layers, w.batch, s.h, s.dh, dtype=tdt, device=dev))
    out_all = torch.empty(layers, w.batch, s.h, s.dh, dtype=torch.float32, device=dev)
    qs = [q_all[layer] for layer in range(layers)]
    outs = [out_all[layer] for layer in range(layers)]
    start = torch.zeros(w.batch, dtype=torch.int32, device=dev)
    seq_len = first["seq_len"].to(dev)
    q_pos = first["q_pos"].to(dev)
    for layer in range(layers):
        inp = first if layer == 0 else decode_inputs(w.replace(seed=rank_seed(rank, layer)))
        kc = torch.empty(w.batch * w.capacity * s.e_k, dtype=tdt, device=dev)
        vc = torch.empty(w.batch * w.capacity * s.e_v, dtype=tdt, device=dev)
        kpa.kpa_append_factors(cfg, w.batch, w.capacity, inp["kf"].to(dev), inp["vf"].to(dev),
                               start, w.capacity, kc, vc)
        kcs.append(kc)
        vcs.append(vc)
        qs[layer].copy_((query_factor_inputs(w, rank_seed(rank, layer)) if qf_mode else inp["q"]).to(dev))
        del inp
    max_len = int(lens.max())
    tps = a.tokens_per_split
    ws_bytes = kpa.kpa_decode_workspace_size(cfg, w.batch, max_len, tps)
    ws = torch.zeros(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    sm_scale = 1.0 / float(np.sqrt(s.dh))
    torch.cuda.synchronize()

    stream = torch.cuda.Stream(device=dev)

    def decode(q_layer, layer):
        if qf_mode:   # factor records [batch][E_Q]: element stride 1, sequence stride E_Q
            kpa.kpa_decode_qf(cfg, w.batch, q_layer, 1, s.e_q, q_pos, kcs[layer], vcs[layer], w.capacity,
                              seq_len, max_len, sm_scale, outs[layer], ws, stream=stream)
        else:
            kpa.kpa_decode_split(cfg, w.batch, q_layer, q_pos, kcs[layer], vcs[layer], w.capacity,
                                 seq_len, max_len, sm_scale, tps, outs[layer], ws, stream=stream)

    def step(qsrc):
        for layer in range(layers):
            decode(qsrc[layer], layer)

    # warm up eagerly once (also sets kernel attributes), then capture the step
    with torch.cuda.stream(stream):
        step(qs)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step(qs)

    # e2e graph: every layer's query comes from pinned host memory and every output goes
    # back to it, each step.  The copies overlap the decodes on a side stream: the first
    # two layers' queries first, the others' while those run; each group of layers'
    # outputs while the next group runs, the last layers' one by one.
    q_host = q_all.cpu().pin_memory()
    out_host = torch.empty(out_all.shape, dtype=out_all.dtype).pin_memory()
    q_dev_all = torch.empty_like(q_all)
    side = torch.cuda.Stream(device=dev)
    group = 4

    def decode_layer(layer):
        decode(q_dev_all[layer], layer)

    head = min(2, layers)                         # layers whose queries go first
    graph_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_e2e, stream=stream):
        q_dev_all[:head].copy_(q_host[:head], non_blocking=True)
        side.wait_stream(stream)
        if layers > head:
            with torch.cuda.stream(side):
                q_dev_all[head:].copy_(q_host[head:], non_blocking=True)
        lo = 0
        for layer in range(layers):
            if layer == head:
                stream.wait_stream(side)          # the other layers' queries are in
            decode_layer(layer)
            # outputs in groups of `group` layers; the last two layers one by one
            if (layer + 1) % group == 0 or layer >= layers - 3:
                side.wait_stream(stream)
                with torch.cuda.stream(side):
                    out_host[lo:layer + 1].copy_(out_all[lo:layer + 1], non_blocking=True)
                lo = layer + 1
        stream.wait_stream(side)

    sampler = ClockSampler(local)

    def timed(g, steps, warmup):
        for _ in range(warmup):
            g.replay()
        stream.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        ev[0].record(stream)
        for i in range(steps):
            g.replay()
            ev[i + 1].record(stream)
        ev[-1].synchronize()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        per = np.array([ev[i].elapsed_time(ev[i + 1]) for i in range(steps)])
        dist_ms = {"median": float(np.median(per)), "p10": float(np.percentile(per, 10)),
                   "p90": float(np.percentile(per, 90)), "min": float(per.min()), "max": float(per.max())}
        return max_over_ranks(ev[0].elapsed_time(ev[-1]), world, dev) / steps, dist_ms

    with torch.cuda.stream(stream):
        # settle clocks under load (untimed) while the sampler runs
        sampler.start()
        t_end = time.time() + a.settle_seconds
        while time.time() < t_end:
            for _ in range(20):
                graph.replay()
            stream.synchronize()
        ms_step, step_dist = timed(graph, a.steps, a.warmup)
        clocks = sampler.stop()
        ms_e2e, e2e_dist = timed(graph_e2e, a.steps, a.warmup)
    code = kpa.kpa_read_device_error(stream)
    if code != 0:
        raise RuntimeError(f"device error word {code} after the timed region")

    tokens_per_layer = int(lens.sum())
    tokens_all = sum_over_ranks(tokens_per_layer, world, dev)       # every rank's own batch
    value = tokens_all * layers / (ms_step * 1e-3)
    e2e_value = tokens_all * layers / (ms_e2e * 1e-3)
    t_launch = ms_step * 1e-3 / layers            # average decode call (split + combine)
    achieved = layer_bytes / t_launch / 1e9
    peak, peak_kind = _hbm_peak()
    khash = _kernel_hash()
    traffic_workload = (a.workload if not (a.seq_len or a.batch or a.tokens_per_split or a.decode_engine
                                           or qf_mode) else None)
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": _traffic(khash, traffic_workload),
                "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json copy test)",
                "kernel": "kpa_decode (split + combine), per layer call",
                "algorithmic_bytes_per_launch": layer_bytes,
                "launch_us": t_launch * 1e6, "kernel_sources_sha": khash,
                "launch_us_per_step_percentiles": {k: v * 1e3 / layers for k, v in step_dist.items()}}
    kind = kpa.kpa_decode_kernel_kind(cfg, w.batch, max_len, tps)
    plan = kpa.kpa_decode_plan(cfg, w.batch, max_len, tps)
    if qf_mode:
        roofline["kernel"] = "kpa_decode_qf (query factors; split + combine), per layer call"
        if a.decode_engine == 2:
            # the factored score plans its own splits and always ends with the combine kernel
            kind, plan = "factored_score_cuda_cores", (None, None, 2 if max_len > 0 else 1)
    roofline["decode_kernel"] = kind
    if s.order == 3:
        roofline["algorithmic_flops_per_launch"] = tokens_per_layer * _order3_flops_per_token(s)
    if s.order == 3 and kind == "cuda_cores":
        # on the CUDA-core kernel a third-order record is too small for HBM to bound the
        # decode: its FP32 multiply-adds do (see _order3_flops_per_token)
        flops = tokens_per_layer * _order3_flops_per_token(s)
        roofline = {"bound": "alu", "achieved": flops / t_launch / 1e12, "peak": FP32_PEAK_TFLOPS,
                    "unit": "TFLOP/s", "frac": flops / t_launch / 1e12 / FP32_PEAK_TFLOPS, "traffic": None,
                    "peak_source": "148 SMs x 128 FP32 lanes x 2 flops x 1.965 GHz (nominal unit counts and "
                                   "max SM clock)",
                    "kernel": "kpa_decode on a third-order cache (split + combine), per layer call",
                    "algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": layer_bytes,
                    "hbm_frac": achieved / peak, "launch_us": t_launch * 1e6}

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16"
            if w.dtype == "bf16" else "f32", "data": "synthetic (seeded, shapes of the pages' workloads)",
            "config": dict(_config_json(w, layers, lens, world),
                           splits_per_sequence=plan[0], tokens_per_split=plan[1],
                           query="factors [batch][E_Q] float32 (kpa_decode_qf)" if qf_mode
                           else "dense [batch][h][d_h]"),
            "roofline": roofline,
            "e2e": {"value": e2e_value, "unit": "tokens/s",
                    "h2d_bytes_per_step": int(q_host.numel() * q_host.element_size()),
                    "d2h_bytes_per_step": int(out_host.numel() * out_host.element_size()),
                    "ms_per_step": ms_e2e, "ms_per_step_percentiles": e2e_dist,
                    "path": f"pinned host queries -> device, {'kpa_decode_qf' if qf_mode else 'kpa_decode'} x "
                            "layers, outputs -> pinned host, every "
                            "step, one CUDA graph; the copies overlap the decodes on a second stream (the first "
                            "two layers' queries first, then the rest; outputs in groups of 4 layers, the last "
                            "ones singly)"},
            "ms_per_step_percentiles": step_dist,
            "clocks": clocks,
            "gpu_launches": a.steps * layers * plan[2]}

    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        base, _ = _cpu_baseline(w, first, a.cpu_seconds,
                                q_factors=query_factor_inputs(w, rank_seed(rank, 0)) if qf_mode else None)
        line["cpu_baseline"] = base
    del graph, graph_e2e
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# FP32 CUDA-core peak: 148 SMs x 128 lanes x 2 flops per FMA x 1.965 GHz.
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def _order3_flops_per_token(s):
    """Multiply-adds a third-order decode needs per cached token, x 2: the score's
    bilinear form per head and key rank, h R_K (d_b d_c + d_b) + h R_K; the products
    b^V (x) c^V once per value rank, R_V d_b d_c; the value update per head and value
    rank, h R_V d_b d_c (plus h R_V for p a^V)."""
    h, db, dc = s.h1, s.d1, s.d2
    fma = h * s.r_k * (db * dc + db + 1) + s.r_v * db * dc + h * s.r_v * (db * dc + 1)
    return 2 * fma


def _bf16_peak():
    try:
        with open(PEAKS) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return 1590.0, 1400.0, "fallback"


def run_append_prefill(a):
    """The append + prefill configuration, one step = the whole path of a prompt
    chunk and the token after it:
      1. kpa_append of a 2048-token chunk per sequence (merged projection, factor
         RoPE, cache write, query assembly),
      2. the causal kpa_prefill of the chunk over the cache,
      3. the decode step: kpa_append of token 2048 of every sequence, then kpa_decode
         of its query over the 2049 cached slots.
    Each part is timed with CUDA events on its stream; the line's roofline is the
    prefill kernel's (tensor bound)."""
    import torch
    import torch.distributed as dist
    import factorised_kv_attention_b200 as kpa
    from workloads import APPEND_PREFILL_SPLITS, append_inputs

    rank, world, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    w = APPEND_PREFILL_SPLITS[a.prefill_split]
    if a.batch:
        w = w.replace(batch=a.batch, name=w.name + f" [batch overridden to {a.batch}]")
    s = w.shape
    inp = append_inputs(w.replace(seed=rank_seed(rank)))
    cfg = kpa.make_config(s, "bf16")
    kpa.kpa_test_set_prefill_engine(a.prefill_engine)
    prefill_kernel = kpa.kpa_prefill_kernel_kind(cfg)
    x, W, x1 = inp["x"].to(dev), inp["W"].to(dev), inp["x_step"].to(dev)
    kc = torch.zeros(w.batch * w.capacity * s.e_k, dtype=torch.bfloat16, device=dev)
    vc = torch.zeros(w.batch * w.capacity * s.e_v, dtype=torch.bfloat16, device=dev)
    start = torch.zeros(w.batch, dtype=torch.int32, device=dev)
    ws = torch.zeros(kpa.kpa_append_workspace_size(cfg, w.batch, w.n_tok), dtype=torch.uint8, device=dev)
    q = torch.empty(w.batch, w.n_tok, s.h, s.dh, dtype=torch.bfloat16, device=dev)
    out = torch.empty(w.batch, w.n_tok, s.h, s.dh, dtype=torch.float32, device=dev)
    # decode step: token n_tok of every sequence, attending over n_tok + 1 slots
    pos1 = torch.full((w.batch,), w.n_tok, dtype=torch.int32, device=dev)
    len1 = torch.full((w.batch,), w.n_tok + 1, dtype=torch.int32, device=dev)
    ws1 = torch.zeros(max(kpa.kpa_append_workspace_size(cfg, w.batch, 1), 256), dtype=torch.uint8, device=dev)
    qf1 = ws1.view(torch.float32)             # the append leaves the query factors here: [E_Q][batch]
    wsd = torch.zeros(max(kpa.kpa_decode_workspace_size(cfg, w.batch, w.n_tok + 1), 256), dtype=torch.uint8,
                      device=dev)
    out1 = torch.empty(w.batch, s.h, s.dh, dtype=torch.float32, device=dev)
    scale = 1.0 / float(np.sqrt(s.dh))
    stream = torch.cuda.Stream(device=dev)
    M = w.batch * w.n_tok
    proj_flop = 2.0 * M * s.n_proj * s.d_model
    pre_flop = 4.0 * s.h * s.dh * w.batch * (w.n_tok * (w.n_tok + 1) / 2)
    dec_bytes = w.batch * (w.n_tok + 1) * (s.e_k + s.e_v) * 2
    sampler = ClockSampler(local)
    _, _, dec_launches = kpa.kpa_decode_plan(cfg, w.batch, w.n_tok + 1)
    launches_per_step = 2 + 1 + 1 + dec_launches     # append (GEMM + query assembly), prefill, step

    def append():
        kpa.kpa_append(cfg, w.batch, w.n_tok, x, W, start, w.capacity, kc, vc, q, ws, stream=stream)

    def prefill():
        kpa.kpa_prefill(cfg, w.batch, w.n_tok, q, start, kc, vc, w.capacity, scale, out, stream=stream)

    # the decode step reads the one-token append's query factors where a tensor-core decode
    # variant takes this split (kpa_decode_qf), else the append's dense rotated query
    step_qf = kpa.kpa_decode_kernel_kind(cfg, w.batch, w.n_tok + 1) == "mma_sync"
    q1 = torch.empty(w.batch, 1, s.h, s.dh, dtype=torch.bfloat16, device=dev)

    def decode_step():
        # one-token append (matrix-vector projection, RoPE, cache write; query factors into
        # its workspace), then decode straight from those query factors
        if step_qf:
            kpa.kpa_append(cfg, w.batch, 1, x1, W, pos1, w.capacity, kc, vc, None, ws1, stream=stream)
            kpa.kpa_decode_qf(cfg, w.batch, qf1, w.batch, 1, None, kc, vc, w.capacity, len1, w.n_tok + 1, scale,
                              out1, wsd, stream=stream)
        else:
            kpa.kpa_append(cfg, w.batch, 1, x1, W, pos1, w.capacity, kc, vc, q1, ws1, stream=stream)
            kpa.kpa_decode(cfg, w.batch, q1, None, kc, vc, w.capacity, len1, w.n_tok + 1, scale, out1, wsd,
                           stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(a.warmup):
            append()
            prefill()
            decode_step()
        stream.synchronize()
        sampler.start()
        t_end = time.time() + a.settle_seconds
        while time.time() < t_end:
            append()
            prefill()
            decode_step()
            stream.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4 * a.steps)]
        for i in range(a.steps):
            ev[4 * i].record(stream)
            append()
            ev[4 * i + 1].record(stream)
            prefill()
            ev[4 * i + 2].record(stream)
            decode_step()
            ev[4 * i + 3].record(stream)
        stream.synchronize()
        torch.cuda.synchronize()
        clocks = sampler.stop()
        # end to end through the API: pinned x -> device, the step, out and the step's out -> pinned host
        x_host, x1_host = inp["x"].pin_memory(), inp["x_step"].pin_memory()
        out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        out1_host = torch.empty(out1.shape, dtype=out1.dtype).pin_memory()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(a.steps):
            x.copy_(x_host, non_blocking=True)
            x1.copy_(x1_host, non_blocking=True)
            append()
            prefill()
            decode_step()
            out_host.copy_(out, non_blocking=True)
            out1_host.copy_(out1, non_blocking=True)
        e1.record(stream)
        e1.synchronize()
    code = kpa.kpa_read_device_error(stream)
    if code != 0:
        raise RuntimeError(f"device error word {code}")

    def part(k):
        return float(np.mean([ev[4 * i + k].elapsed_time(ev[4 * i + k + 1]) for i in range(a.steps)])) * 1e-3

    t_app, t_pre, t_dec = part(0), part(1), part(2)
    t_step = max_over_ranks(t_app + t_pre + t_dec, world, dev)
    ms_e2e = max_over_ranks(e0.elapsed_time(e1) / a.steps, world, dev)
    tokens_all = sum_over_ranks(M + w.batch, world, dev)         # chunk tokens + the decoded token
    peak, peak_sus, kind = _bf16_peak()
    hbm, hbm_kind = _hbm_peak()
    pre_tf, app_tf = pre_flop / t_pre / 1e12, proj_flop / t_app / 1e12
    line = {"metric": "append + causal prefill + decode step, tokens/s (2048-token chunks); "
                      "TFLOP/s vs B200 bf16 peak",
            "value": tokens_all / t_step, "unit": "tokens/s", "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": t_step * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16 in, fp32 accumulate (prefill MMA in fp16)",
            "data": "synthetic (seeded)",
            "config": {"workload": w.name, "batch": w.batch, "seq_len": w.n_tok, "d_model": s.d_model,
                       "l2": "projection input 67 MB and prefill output 134 MB per step exceed L2",
                       "parallelism": f"replicas x{world} (batch-sharded, no exchange)"},
            "roofline": {"bound": "tensor", "achieved": pre_tf, "peak": peak, "unit": "TFLOP/s",
                         "frac": pre_tf / peak, "traffic": None,
                         "peak_source": f"{kind} bf16_tflops (burst; fp16 dense rate is the same)",
                         "kernel": f"kpa_prefill ({prefill_kernel})", "algorithmic_flop_per_launch": pre_flop,
                         "launch_us": t_pre * 1e6},
            "append": {"achieved_tflops": app_tf, "frac": app_tf / peak, "launch_us": t_app * 1e6,
                       "algorithmic_flop_per_launch": proj_flop},
            "decode_step": {"launch_us": t_dec * 1e6, "cache_bytes": dec_bytes,
                            "achieved_gbs": dec_bytes / t_dec / 1e9, "hbm_peak_gbs": hbm,
                            "note": "append of one token per sequence + decode over 2049 slots from its query "
                                    "factors (latency bound)"},
            "e2e": {"value": tokens_all / (ms_e2e * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": int(x_host.numel() * 2 + x1_host.numel() * 2),
                    "d2h_bytes_per_step": int(out_host.numel() * 4 + out1_host.numel() * 4),
                    "ms_per_step": ms_e2e},
            "clocks": clocks, "gpu_launches": a.steps * launches_per_step}
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        line["cpu_baseline"], _ = _cpu_baseline_prefill(w, inp, a.cpu_seconds)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_split(a):
    """One sequence split across the ranks (strong scaling): rank r holds the tokens
    split_range(L, world, r) of every layer's cache in slots 0 .. (kpa_append_factors_pos
    rotates them at their global positions), decodes them with the query's global
    position (kpa_decode_lse), and per layer the ranks' (out, lse) are all-gathered over
    NCCL and merged on every rank (kpa_merge_lse).  Timed per step with CUDA events, the
    max over ranks; the value counts each sequence's tokens once."""
    import torch
    import torch.distributed as dist
    import factorised_kv_attention_b200 as kpa
    from workloads import decode_inputs

    rank, world, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    w = _workload(a.workload, a)
    s = w.shape
    first = decode_inputs(w.replace(seed=rank_seed(0)))      # every rank draws the same sequences
    lens = first["seq_len"].numpy()
    L = int(lens.max())
    lo, hi = split_range(L, world, rank)
    n = hi - lo
    cap = max(8, (n + 7) // 8 * 8)
    elt = 2 if w.dtype == "bf16" else 4
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    layer_bytes = int(lens.sum()) * (s.e_k + s.e_v) * elt
    local_bytes = int(np.clip(lens - lo, 0, n).sum()) * (s.e_k + s.e_v) * elt
    layers = a.layers or max(2, int(np.ceil(4 * l2 / max(local_bytes, 1))))
    cfg = kpa.make_config(s, w.dtype)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    zero = torch.zeros(w.batch, dtype=torch.int32, device=dev)
    off = torch.full((w.batch,), lo, dtype=torch.int32, device=dev)
    seq_local = torch.from_numpy(np.clip(lens - lo, 0, n).astype(np.int32)).to(dev)
    q_pos = first["q_pos"].to(dev)
    max_local = int(seq_local.max().item())
    kcs, vcs, qs = [], [], []
    for layer in range(layers):
        inp = first if layer == 0 else decode_inputs(w.replace(seed=rank_seed(0, layer)))
        kc = torch.zeros(w.batch * cap * s.e_k, dtype=tdt, device=dev)
        vc = torch.zeros(w.batch * cap * s.e_v, dtype=tdt, device=dev)
        if n > 0:
            kpa.kpa_append_factors_pos(cfg, w.batch, n, inp["kf"][:, lo:hi].contiguous().to(dev),
                                       inp["vf"][:, lo:hi].contiguous().to(dev), zero, off, cap, kc, vc)
        kcs.append(kc)
        vcs.append(vc)
        qs.append(inp["q"].to(dev))
        del inp
    ws = torch.zeros(max(kpa.kpa_decode_workspace_size(cfg, w.batch, max_local), 256), dtype=torch.uint8,
                     device=dev)
    out_l = torch.empty(w.batch, s.h, s.dh, dtype=torch.float32, device=dev)
    lse_l = torch.empty(w.batch, s.h, dtype=torch.float32, device=dev)
    outs = [torch.empty(w.batch, s.h, s.dh, dtype=torch.float32, device=dev) for _ in range(layers)]
    sm_scale = 1.0 / float(np.sqrt(s.dh))
    stream = torch.cuda.current_stream(dev)

    def step():
        for layer in range(layers):
            kpa.kpa_decode_lse(cfg, w.batch, qs[layer], q_pos, kcs[layer], vcs[layer], cap, seq_local, max_local,
                               sm_scale, out_l, lse_l, ws, stream=stream)
            po, pl = gather_parts(out_l, lse_l, world)
            kpa.kpa_merge_lse(po, pl, outs[layer], stream=stream)

    for _ in range(a.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(a.steps + 1)]
    ev[0].record(stream)
    for i in range(a.steps):
        step()
        ev[i + 1].record(stream)
    ev[-1].synchronize()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    per = np.array([ev[i].elapsed_time(ev[i + 1]) for i in range(a.steps)])
    ms_step = max_over_ranks(ev[0].elapsed_time(ev[-1]), world, dev) / a.steps
    code = kpa.kpa_read_device_error(stream)
    if code != 0:
        raise RuntimeError(f"device error word {code}")
    t_layer = ms_step * 1e-3 / layers
    peak, peak_kind = _hbm_peak()
    n_split, _, _ = kpa.kpa_decode_plan(cfg, w.batch, max(max_local, 1))
    line = {"metric": METRIC, "value": int(lens.sum()) * layers / (ms_step * 1e-3), "unit": "tokens/s",
            "n_gpus": world, "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic (seeded, shapes of the pages' workloads)",
            "config": dict(_config_json(w, layers, lens, world),
                           parallelism=f"sequence split across {world} rank(s): contiguous token ranges, one "
                                       "all-gather of (out, lse) per layer, log-sum-exp merge",
                           tokens_per_rank=n, splits_per_sequence_per_rank=n_split),
            "roofline": {"bound": "hbm", "achieved": layer_bytes / t_layer / 1e9, "peak": peak * world, "unit": "GB/s",
                         "frac": layer_bytes / t_layer / 1e9 / (peak * world), "traffic": None,
                         "peak_source": f"{peak_kind} hbm_gbs x {world} GPU(s)",
                         "kernel": "kpa_decode_lse + all-gather + kpa_merge_lse, per layer",
                         "algorithmic_bytes_per_launch": layer_bytes, "launch_us": t_layer * 1e6},
            "ms_per_step_percentiles": {"median": float(np.median(per)), "p10": float(np.percentile(per, 10)),
                                        "p90": float(np.percentile(per, 90))},
            "gpu_launches": a.steps * layers * 3}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_sweep(a):
    """The FlashTPA decoding benchmark grid ("Tensor Product Attention Is All You Need"
    explainer, decoding-speed figures: sequence 2^12 .. 2^19, batch 1 .. 16) on the
    pages' TPA shape (h = 32, d_h = 64, R_K = R_V = 1).  Per point: caches filled through
    kpa_append_factors from device-drawn factors, enough layer copies to exceed 4 x L2
    (at least 2), the decodes of one step in a CUDA graph, timed with CUDA events over
    a.steps replays after a.warmup.  One JSON line per point (rank 0, 1 GPU)."""
    import torch
    import factorised_kv_attention_b200 as kpa
    from workloads import FLASHTPA_DECODE, device_decode_factors

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peak, peak_kind = _hbm_peak()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    s = FLASHTPA_DECODE.shape
    cfg = kpa.make_config(s, "bf16")
    stream = torch.cuda.Stream(device=dev)
    for log_len in range(12, 20):
        for batch in (1, 2, 4, 8, 16):
            L = 1 << log_len
            w = FLASHTPA_DECODE.replace(batch=batch, capacity=L, length=L, name=f"FlashTPA shape B={batch} L={L}")
            layer_bytes = batch * L * (s.e_k + s.e_v) * 2
            layers = max(2, int(np.ceil(4 * l2 / layer_bytes)))
            start = torch.zeros(batch, dtype=torch.int32, device=dev)
            seq_len = torch.full((batch,), L, dtype=torch.int32, device=dev)
            q_pos = seq_len.clone()
            kcs, vcs, qs = [], [], []
            for layer in range(layers):
                kf, vf, q = device_decode_factors(w, dev, 1000 * log_len + 10 * batch + layer)
                kc = torch.empty(batch * L * s.e_k, dtype=torch.bfloat16, device=dev)
                vc = torch.empty(batch * L * s.e_v, dtype=torch.bfloat16, device=dev)
                kpa.kpa_append_factors(cfg, batch, L, kf, vf, start, L, kc, vc)
                kcs.append(kc)
                vcs.append(vc)
                qs.append(q)
                del kf, vf
            outs = [torch.empty(batch, s.h, s.dh, dtype=torch.float32, device=dev) for _ in range(layers)]
            ws = torch.zeros(max(kpa.kpa_decode_workspace_size(cfg, batch, L), 256), dtype=torch.uint8, device=dev)
            scale = 1.0 / float(np.sqrt(s.dh))

            def step():
                for i in range(layers):
                    kpa.kpa_decode(cfg, batch, qs[i], q_pos, kcs[i], vcs[i], L, seq_len, L, scale, outs[i], ws,
                                   stream=stream)

            with torch.cuda.stream(stream):
                step()
            stream.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                step()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(a.steps + 1)]
            with torch.cuda.stream(stream):          # replays run on the stream the events time
                for _ in range(a.warmup):
                    graph.replay()
                stream.synchronize()
                ev[0].record(stream)
                for i in range(a.steps):
                    graph.replay()
                    ev[i + 1].record(stream)
            ev[-1].synchronize()
            per = np.array([ev[i].elapsed_time(ev[i + 1]) for i in range(a.steps)]) / layers * 1e3   # us per call
            code = kpa.kpa_read_device_error(stream)
            if code != 0:
                raise RuntimeError(f"device error word {code}")
            us = float(np.median(per))
            n_split, tps, launches = kpa.kpa_decode_plan(cfg, batch, L)
            print(json.dumps({"sweep": "flashtpa", "batch": batch, "seq_len": L, "layers": layers,
                              "us_per_call_median": us, "us_p10": float(np.percentile(per, 10)),
                              "us_p90": float(np.percentile(per, 90)),
                              "cached_tokens_per_s": batch * L / (us * 1e-6),
                              "achieved_gbs": layer_bytes / (us * 1e-6) / 1e9, "peak_gbs": peak,
                              "frac": layer_bytes / (us * 1e-6) / 1e9 / peak, "peak_source": peak_kind,
                              "splits_per_sequence": n_split, "tokens_per_split": tps, "launches": launches}),
                  flush=True)
            del graph, kcs, vcs, qs, outs, ws
            torch.cuda.empty_cache()
    return 0


def main(argv=None):
    a = _args(argv)
    if a.impl == "reference":
        return run_reference(a)
    if a.sweep:
        return run_sweep(a)
    if a.split_sequence:
        return run_split(a)
    if a.workload == "append_prefill":
        return run_append_prefill(a)
    return run_kpa(a)


if __name__ == "__main__":
    sys.exit(main())
