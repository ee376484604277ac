"""Seeded synthetic workloads shaped like the pages' KPA / TPA configurations.

This module holds only shapes and random-number draws: no RoPE, no Kronecker
product, no attention.  Both the float64 oracle (through the tests) and the CUDA
library (through the tests, the smoke check and the benchmark) take their inputs
from here, so the two sides see bit-identical values.

Draw order for a decode workload (numpy PCG64, ``default_rng(seed)``):
  1. per-sequence lengths, when ragged (integers uniform on [lo, hi] inclusive);
  2. the query ``q`` [B][h][d_h] ~ N(0, q_std^2);
  3. key factor records, sequence by sequence, rows 0 .. len_b-1, ~ N(0, std^2);
  4. value factor records, same order.
Rows at or beyond a sequence's length stay zero.  Values are drawn in float32
and rounded to bfloat16 (round to nearest even) for bf16 workloads.

An append / prefill workload draws x [B][n][d_model] ~ N(0, 1) and then the
merged projection weights W [N][d_model] ~ N(0, w_std^2), then the x of one
decode step [B][1][d_model].
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Shape:
    """Kronecker split of the heads (h = h1*h2) and features (d_h = d1*d2)."""
    h1: int
    h2: int
    d1: int
    d2: int
    r_k: int
    r_v: int
    r_q: int = 0
    d_model: int = 0
    rope_base: float = 10000.0
    shared_b: int = 0          # 1: one B factor for keys and values (B^K_r = B^V_r, r_k == r_v)
    order: int = 2             # 3: third-order TPA, key a (x) b (x) c with h2 = 1, d1 = d_b, d2 = d_c

    @property
    def h(self) -> int:
        return self.h1 * self.h2

    @property
    def dh(self) -> int:
        return self.d1 * self.d2

    @property
    def e_k(self) -> int:
        """Elements in one token's key record [A_0..A_{R-1} | B_0..B_{R-1}], or for a
        third-order shape [a_0..a_{R-1} | b_0..b_{R-1} | c_0..c_{R-1}]."""
        if self.order == 3:
            return self.r_k * (self.h1 + self.d1 + self.d2)
        return self.r_k * (self.h1 * self.d1 + self.h2 * self.d2)

    @property
    def e_v(self) -> int:
        """Elements in one token's value record: [A_0.. | B_0..], or [A_0..] alone when
        the B factors are shared with the keys."""
        if self.order == 3:
            return self.r_v * (self.h1 + self.d1 + self.d2)
        if self.shared_b:
            return self.r_v * self.h1 * self.d1
        return self.r_v * (self.h1 * self.d1 + self.h2 * self.d2)

    @property
    def e_q(self) -> int:
        return self.r_q * (self.h1 * self.d1 + self.h2 * self.d2)

    @property
    def n_proj(self) -> int:
        """Output columns of the merged projection: Q, K and V factor records."""
        return self.e_q + self.e_k + self.e_v


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    shape: Shape
    batch: int
    capacity: int
    dtype: str                      # "f32" or "bf16"
    factor_std: float
    q_std: float
    seed: int = 0
    length: int = 0                 # fixed length (all sequences) when > 0
    ragged: tuple = ()              # (lo, hi) inclusive when lengths are drawn
    q_pos_offset: int = 0           # q_pos = length_b + offset

    def replace(self, **kw) -> "DecodeWorkload":
        return dataclasses.replace(self, **kw)


@dataclass(frozen=True)
class AppendWorkload:
    name: str
    shape: Shape
    batch: int
    n_tok: int
    capacity: int
    x_std: float = 1.0
    w_std: float = 0.02
    seed: int = 0
    start: int = 0

    def replace(self, **kw) -> "AppendWorkload":
        return dataclasses.replace(self, **kw)


# --- the five configurations ------------------------------------------------
# C1: tiny KPA decode, fp32, factors ~N(0,1), q ~N(0,1)/sqrt(d_h), q at 256.
TINY_KPA = DecodeWorkload(
    name="tiny KPA decode (B=1, h=2x4, d_h=8x8, R=2+2, L=256, fp32)",
    shape=Shape(h1=2, h2=4, d1=8, d2=8, r_k=2, r_v=2, rope_base=10000.0),
    batch=1, capacity=256, dtype="f32", factor_std=1.0, q_std=1.0 / 8.0, seed=0, length=256)

# C2: TPA degenerate split decode.
TPA_DECODE = DecodeWorkload(
    name="TPA decode (B=8, h=16x1, d_h=1x64, R=2+2, L=4096, bf16)",
    shape=Shape(h1=16, h2=1, d1=1, d2=64, r_k=2, r_v=2, rope_base=10000.0),
    batch=8, capacity=4096, dtype="bf16", factor_std=1.0 / np.sqrt(2.0), q_std=1.0 / 8.0,
    seed=0, length=4096)

# C3: KPA medium decode, ragged lengths uniform on [1024, 8192].
KPA_MEDIUM = DecodeWorkload(
    name="KPA medium decode (B=32, h=4x8, d_h=8x16, R=4+4, L~U[1024,8192], bf16)",
    shape=Shape(h1=4, h2=8, d1=8, d2=16, r_k=4, r_v=4, rope_base=10000.0),
    batch=32, capacity=8192, dtype="bf16", factor_std=0.5, q_std=1.0 / np.sqrt(128.0),
    seed=0, ragged=(1024, 8192))

# C4: KPA long-context decode, 2^19 tokens, RoPE base 5e5.
KPA_LONG = DecodeWorkload(
    name="KPA long decode (B=1, h=4x8, d_h=8x16, R=2+2, L=2^19, bf16, base 5e5)",
    shape=Shape(h1=4, h2=8, d1=8, d2=16, r_k=2, r_v=2, rope_base=500000.0),
    batch=1, capacity=1 << 19, dtype="bf16", factor_std=1.0 / np.sqrt(2.0),
    q_std=1.0 / np.sqrt(128.0), seed=0, length=1 << 19)

# C5: append (merged projection + factor RoPE + cache write) then causal prefill,
# then one decode step at position 2048.
APPEND_PREFILL = AppendWorkload(
    name="KPA append+prefill (B=8, n=2048, d_model=2048, h=4x4, d_h=8x16, R_Q=6, R=2+2)",
    shape=Shape(h1=4, h2=4, d1=8, d2=16, r_k=2, r_v=2, r_q=6, d_model=2048, rope_base=10000.0),
    batch=8, n_tok=2048, capacity=2112, seed=0)

# The append+prefill configuration on other splits of the same h = 16 heads and
# d_h = 128 features: the TPA split of "Kronecker Product Attention", section 2.2
# (h1 = h, d1 = 1), and the KPA split at rank 4.  Same chunk, batch, d_model and R_Q.
APPEND_PREFILL_SPLITS = {
    "kpa_h4x4_d8x16_r2": APPEND_PREFILL,
    "tpa_h16_d1x128_r2": APPEND_PREFILL.replace(
        name="TPA append+prefill (B=8, n=2048, d_model=2048, h=16x1, d_h=1x128, R_Q=6, R=2+2)",
        shape=dataclasses.replace(APPEND_PREFILL.shape, h1=16, h2=1, d1=1, d2=128)),
    "kpa_h4x4_d8x16_r4": APPEND_PREFILL.replace(
        name="KPA append+prefill (B=8, n=2048, d_model=2048, h=4x4, d_h=8x16, R_Q=6, R=4+4)",
        shape=dataclasses.replace(APPEND_PREFILL.shape, r_k=4, r_v=4)),
    # the KPA paper's 353M models (section 3.2): d_model 1024, h = 16 as 4x4, d_h = 64 as
    # 8x8, R = 2; the same chunk, batch and R_Q
    "kpa353m_h4x4_d8x8_r2": APPEND_PREFILL.replace(
        name="KPA append+prefill, 353M model split (B=8, n=2048, d_model=1024, h=4x4, d_h=8x8, R_Q=6, R=2+2)",
        shape=dataclasses.replace(APPEND_PREFILL.shape, d2=8, d_model=1024)),
}

# The decoding benchmark shape of the FlashTPA figures ("Tensor Product Attention Is
# All You Need" explainer, decoding-speed benchmarks): d_model 2048, h = 32, d_h = 64,
# R_Q = 16, R_K = R_V = 1, sequences 2^12 .. 2^19, batch 1 .. 16.  Here batch 1 at 2^19
# tokens; the sweep uses the bench overrides.  The dense query path ignores R_Q.
FLASHTPA_SHAPE = Shape(h1=32, h2=1, d1=1, d2=64, r_k=1, r_v=1, r_q=16, d_model=2048, rope_base=10000.0)
FLASHTPA_DECODE = DecodeWorkload(
    name="FlashTPA-shape decode (B=1, h=32x1, d_h=1x64, R=1+1, L=2^19, bf16)",
    shape=FLASHTPA_SHAPE, batch=1, capacity=1 << 19, dtype="bf16", factor_std=1.0, q_std=1.0 / 8.0,
    seed=0, length=1 << 19)

# The TPA decode with one B shared by keys and values ("Tensor Product Attention Is All
# You Need", section 5, "TPA KV with Shared B"): same sizes, key record [A^K | B]
# (B unrotated), value record [A^V].
TPA_SHARED_DECODE = dataclasses.replace(
    TPA_DECODE, name="TPA decode, shared B (B=8, h=16x1, d_h=1x64, R=2, L=4096, bf16)",
    shape=dataclasses.replace(TPA_DECODE.shape, shared_b=1))

# Third-order TPA ("Tensor Product Attention Is All You Need", Appendix C, as the
# explainer summarises it): the key of head h is (1/R) sum_r a_r[h] (b_r (x) c_r), b in
# R^{d_b}, c in R^{d_c}, d_h = d_b d_c = 64, so the sizes match the TPA decode above.
# The pages give no shape for it; this one keeps h, d_h, R, B and L of the TPA decode
# and splits d_h as 8 x 8.  Factors ~ N(0, 2^(1/3)) make a key entry's variance
# sigma^6 / R = 1.
TPA3_DECODE = DecodeWorkload(
    name="third-order TPA decode (B=8, h=16, d_h=8x8, R=2+2, L=4096, bf16)",
    shape=Shape(h1=16, h2=1, d1=8, d2=8, r_k=2, r_v=2, rope_base=10000.0, order=3),
    batch=8, capacity=4096, dtype="bf16", factor_std=float(2.0 ** (1.0 / 6.0)), q_std=1.0 / 8.0,
    seed=0, length=4096)

# The head splits that "Kronecker Product Attention" evaluates in section 3.2 (its tables
# 1 and 2): d1 = d2 = 8 (d_h = 64), R_K = R_V = 2, h = h1 x h2 with h = 16 (353M models)
# or 20 (773M models).  The pages give no decode workload for them; these use the TPA
# decode's batch, length and spreads.
KPA_SECTION32_SPLITS = {"4x4": (4, 4), "2x8": (2, 8), "8x2": (8, 2), "4x5": (4, 5), "2x10": (2, 10),
                        "10x2": (10, 2)}
KPA_SECTION32 = {
    f"kpa_h{name}_d8x8": DecodeWorkload(
        name=f"KPA decode, split h={h1}x{h2}, d_h=8x8 (B=8, R=2+2, L=4096, bf16)",
        shape=Shape(h1=h1, h2=h2, d1=8, d2=8, r_k=2, r_v=2, rope_base=10000.0),
        batch=8, capacity=4096, dtype="bf16", factor_std=1.0 / np.sqrt(2.0), q_std=1.0 / 8.0, seed=0,
        length=4096)
    for name, (h1, h2) in KPA_SECTION32_SPLITS.items()}

# The append+prefill configuration's h = 16, d_h = 128 in its TPA split and at rank 4,
# as decode workloads with the TPA decode's batch, length and spreads.
SPLIT_DECODES = {
    "tpa_h16_d1x128": DecodeWorkload(
        name="TPA decode, h=16x1, d_h=1x128 (B=8, R=2+2, L=4096, bf16)",
        shape=Shape(h1=16, h2=1, d1=1, d2=128, r_k=2, r_v=2, rope_base=10000.0),
        batch=8, capacity=4096, dtype="bf16", factor_std=1.0 / np.sqrt(2.0), q_std=1.0 / 8.0, seed=0,
        length=4096),
    "kpa_h4x4_d8x16_r4": DecodeWorkload(
        name="KPA decode, h=4x4, d_h=8x16 (B=8, R=4+4, L=4096, bf16)",
        shape=Shape(h1=4, h2=4, d1=8, d2=16, r_k=4, r_v=4, rope_base=10000.0),
        batch=8, capacity=4096, dtype="bf16", factor_std=0.5, q_std=1.0 / 8.0, seed=0, length=4096),
}

# The TPA explainer's 773M-parameter TPA model: h = 61 heads, d_h = 64, R_K = R_V = 2,
# 500 numbers per token ("KV Cache Efficiency at the Evaluated Configurations"); the
# TPA decode's batch, length and spreads.
TPA_H61_DECODE = DecodeWorkload(
    name="TPA decode, 773M model's h=61x1, d_h=1x64 (B=8, R=2+2, L=4096, bf16)",
    shape=Shape(h1=61, h2=1, d1=1, d2=64, r_k=2, r_v=2, rope_base=10000.0),
    batch=8, capacity=4096, dtype="bf16", factor_std=1.0 / np.sqrt(2.0), q_std=1.0 / 8.0, seed=0,
    length=4096)

DECODE_CONFIGS = {"tiny_kpa": TINY_KPA, "tpa_h61": TPA_H61_DECODE, "tpa_decode": TPA_DECODE, "kpa_medium": KPA_MEDIUM,
                  "kpa_long": KPA_LONG, "flashtpa": FLASHTPA_DECODE, "tpa_shared": TPA_SHARED_DECODE,
                  "tpa_order3": TPA3_DECODE, **KPA_SECTION32, **SPLIT_DECODES}


# --- draws ---------------------------------------------------------------------
def _round(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "f32":
        return t
    raise ValueError(dtype)


def lengths(w: DecodeWorkload, rng=None) -> np.ndarray:
    rng = rng if rng is not None else np.random.default_rng(w.seed)
    if w.ragged:
        lo, hi = w.ragged
        return rng.integers(lo, hi + 1, size=w.batch).astype(np.int32)
    return np.full(w.batch, w.length, dtype=np.int32)


def decode_inputs(w: DecodeWorkload) -> dict:
    """Seeded inputs of one decode step.

    Returns CPU tensors in the workload dtype: ``q`` [B][h][d_h], ``kf`` [B][cap][E_K]
    and ``vf`` [B][cap][E_V] (unrotated factor records), plus int32 ``seq_len`` and
    ``q_pos`` [B].
    """
    s = w.shape
    rng = np.random.default_rng(w.seed)
    L = lengths(w, rng)
    if int(L.max(initial=0)) > w.capacity:
        raise ValueError("lengths exceed capacity")
    q = rng.standard_normal((w.batch, s.h, s.dh), dtype=np.float32) * np.float32(w.q_std)
    kf = np.zeros((w.batch, w.capacity, s.e_k), dtype=np.float32)
    vf = np.zeros((w.batch, w.capacity, s.e_v), dtype=np.float32)
    for b in range(w.batch):
        kf[b, :L[b]] = rng.standard_normal((int(L[b]), s.e_k), dtype=np.float32) * np.float32(w.factor_std)
    for b in range(w.batch):
        vf[b, :L[b]] = rng.standard_normal((int(L[b]), s.e_v), dtype=np.float32) * np.float32(w.factor_std)
    return {
        "q": _round(q, w.dtype),
        "kf": _round(kf, w.dtype),
        "vf": _round(vf, w.dtype),
        "seq_len": torch.from_numpy(L.astype(np.int32)),
        "q_pos": torch.from_numpy((L + w.q_pos_offset).astype(np.int32)),
    }


def query_factor_inputs(w: DecodeWorkload, seed: int) -> torch.Tensor:
    """Seeded query factor records [B][E_Q], float32 ([A^Q_0..A^Q_{R_Q-1} | B^Q_0..],
    unrotated), each element ~ N(0, sigma^2) with sigma^2 = q_std sqrt(R_Q): the
    assembled query (1/R_Q) sum_r A^Q_r (x) B^Q_r then has the dense query's spread
    q_std per element."""
    s = w.shape
    if s.r_q <= 0:
        raise ValueError("the shape has no query factors (r_q = 0)")
    rng = np.random.default_rng([seed, 7])
    sigma = np.float32(np.sqrt(w.q_std * np.sqrt(s.r_q)))
    return torch.from_numpy(rng.standard_normal((w.batch, s.e_q), dtype=np.float32) * sigma)


def append_inputs(w: AppendWorkload) -> dict:
    """x [B][n][d_model] and W [N][d_model] (bf16), the decode-step x [B][1][d_model]
    and int32 ``start_pos`` [B]."""
    s = w.shape
    rng = np.random.default_rng(w.seed)
    x = rng.standard_normal((w.batch, w.n_tok, s.d_model), dtype=np.float32) * np.float32(w.x_std)
    W = rng.standard_normal((s.n_proj, s.d_model), dtype=np.float32) * np.float32(w.w_std)
    x_step = rng.standard_normal((w.batch, 1, s.d_model), dtype=np.float32) * np.float32(w.x_std)
    return {
        "x": _round(x, "bf16"),
        "W": _round(W, "bf16"),
        "x_step": _round(x_step, "bf16"),
        "start_pos": torch.full((w.batch,), w.start, dtype=torch.int32),
    }


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a float32 / bfloat16 tensor (for the oracle)."""
    return t.detach().to("cpu").to(torch.float64).numpy()


def device_decode_factors(w: DecodeWorkload, device, seed: int):
    """Factor records [B][capacity][E_K], [B][capacity][E_V] and the query [B][h][d_h]
    drawn on the device (torch's generator, seeded) for throughput sweeps whose sizes
    make host draws slow: every slot below the capacity holds a record ~ N(0, std^2),
    the query ~ N(0, q_std^2), rounded to the workload's dtype.  No parity test uses
    these draws; the oracle takes its inputs from decode_inputs."""
    s = w.shape
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    kf = (torch.randn(w.batch, w.capacity, s.e_k, generator=g, device=device) * w.factor_std).to(dt)
    vf = (torch.randn(w.batch, w.capacity, s.e_v, generator=g, device=device) * w.factor_std).to(dt)
    q = (torch.randn(w.batch, s.h, s.dh, generator=g, device=device) * w.q_std).to(dt)
    return kf, vf, q
