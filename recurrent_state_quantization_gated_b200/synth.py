"""Seeded synthetic inputs for the quantized gated Delta-rule decode workloads.

This module only draws random numbers and shapes them like the decode workloads of
"STEPQuant: When and Where Errors Matter in Delta-Rule Recurrent State Quantization"
(Qwen-style Gated DeltaNet and Kimi-Delta-style layers, Table C1; outlier rows and columns,
§4.2). It holds none of the method's arithmetic: no quantiser, no scale fit, no recurrence,
no calibration statistic. The CUDA library's tests, the benchmark and the CPU oracle's tests
all draw their inputs from here, so both sides consume identical bytes.

Recipe (NumPy ``Generator(PCG64)``; every stream is keyed by ``SeedSequence`` so any step or
sequence can be drawn on its own):

* q, k ~ N(0, 1) fp32, L2-normalised per (step, sequence, head), rounded to bf16 (RNE).
* v ~ N(0, 1) (Student-t with 3 degrees of freedom for the long-rollout workload), bf16.
* beta = sigmoid(N(0, 1)) fp32 per (step, sequence, head).
* gate: a logit a ~ N(-4, 1) is drawn once per unit (per head, or per (head, key channel)
  for the channel-gated workload) and held fixed over steps and sequences;
  g = exp(-softplus(a)) in fp32. The long-rollout workload instead splits the heads 50/50,
  by a seeded permutation, into g = 0.999 and g = 0.9.
* S0 ~ N(0, 0.1^2); for the 128-wide workloads every row and every column of a head is
  multiplied by an exp(N(0, 1)) factor drawn per (head, row) and (head, column), shared by
  all sequences (structural outlier rows and columns).
* The tiny workload's bit map gives exactly half the key rows of each head 4 bits and the
  other half 8 bits, by a seeded permutation.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

_STREAM_STRUCTURE = 0
_STREAM_STATE = 1
_STREAM_TOKENS = 2
_STREAM_BITS = 3
CALIB_SEED_OFFSET = 1000
CALIB_STEPS = 32


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    B: int
    H: int
    d: int
    T: int
    gate_per_channel: bool
    nominal_bits: int
    candidates: tuple
    alloc: str            # "half48" | "dp_head" | "lagrange_row"
    outliers: bool
    v_dist: str           # "normal" | "t3"
    gate_split: bool = False
    pivot_frac: float = 0.0   # share of allocation units kept as FP16 pivots (App. C.2)
    seed: int = 0
    _cache: dict = field(default_factory=dict, compare=False, repr=False)

    @property
    def tiles(self) -> int:
        return self.B * self.H

    @property
    def n_pivots(self) -> int:
        """FP16 pivot units of one layer: key rows (row allocation) or heads (head allocation)."""
        units = self.H * self.d if self.alloc == "lagrange_row" else self.H
        return int(round(self.pivot_frac * units))


_SPECS = [
    dict(name="tiny_b2_h2_d64_t16", B=2, H=2, d=64, T=16, gate_per_channel=False,
         nominal_bits=6, candidates=(4, 8), alloc="half48", outliers=False, v_dist="normal"),
    dict(name="gdn_b64_h32_d128_t256", B=64, H=32, d=128, T=256, gate_per_channel=False,
         nominal_bits=6, candidates=(4, 6, 8), alloc="dp_head", outliers=True, v_dist="normal"),
    dict(name="kda_b256_h32_d128_t128", B=256, H=32, d=128, T=128, gate_per_channel=True,
         nominal_bits=6, candidates=(4, 6, 8), alloc="lagrange_row", outliers=True,
         v_dist="normal", pivot_frac=512 / 81920),
    dict(name="gdn4_b1024_h16_d128_t64", B=1024, H=16, d=128, T=64, gate_per_channel=False,
         nominal_bits=4, candidates=(2, 4, 8), alloc="lagrange_row", outliers=True,
         v_dist="normal"),
    dict(name="drift_b128_h32_d128_t4096", B=128, H=32, d=128, T=4096, gate_per_channel=False,
         nominal_bits=6, candidates=(4, 6, 8), alloc="lagrange_row", outliers=True,
         v_dist="t3", gate_split=True),
]

N_WORKLOADS = len(_SPECS)


def workload(index: int, seed: int = 0, **overrides) -> Workload:
    """The index-th decode workload (0 = tiny oracle case). ``overrides`` may shrink B or T
    for tests (same distributions, fewer sequences or steps)."""
    spec = dict(_SPECS[index])
    spec.update(overrides)
    return Workload(index=index, seed=seed, **spec)


def _rng(*key) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(k) for k in key])))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bfloat16 (nearest, ties to even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def unit_gates(wl: Workload) -> np.ndarray:
    """Per-unit retention gates, fp32: [H] (head gates) or [H][d] (key-channel gates)."""
    key = ("gates",)
    if key not in wl._cache:
        rng = _rng(wl.seed, wl.index, _STREAM_STRUCTURE, 0)
        if wl.gate_split:
            g = np.full(wl.H, 0.9, dtype=np.float32)
            g[rng.permutation(wl.H)[: wl.H // 2]] = np.float32(0.999)
        else:
            shape = (wl.H, wl.d) if wl.gate_per_channel else (wl.H,)
            a = rng.normal(-4.0, 1.0, size=shape)
            g = np.exp(-np.logaddexp(0.0, a)).astype(np.float32)
        wl._cache[key] = g
    return wl._cache[key]


def outlier_factors(wl: Workload):
    """Row and column magnitude factors [H][d] each (ones when the workload has none)."""
    key = ("outliers",)
    if key not in wl._cache:
        if wl.outliers:
            rng = _rng(wl.seed, wl.index, _STREAM_STRUCTURE, 1)
            rows = np.exp(rng.normal(0.0, 1.0, size=(wl.H, wl.d)))
            cols = np.exp(rng.normal(0.0, 1.0, size=(wl.H, wl.d)))
        else:
            rows = np.ones((wl.H, wl.d))
            cols = np.ones((wl.H, wl.d))
        wl._cache[key] = (rows, cols)
    return wl._cache[key]


def initial_state_seq(wl: Workload, b: int) -> np.ndarray:
    """Initial state of sequence b: fp32 [H][d][d] (row = key channel, column = value channel)."""
    rows, cols = outlier_factors(wl)
    rng = _rng(wl.seed, wl.index, _STREAM_STATE, b)
    s = rng.normal(0.0, 0.1, size=(wl.H, wl.d, wl.d))
    s = s * rows[:, :, None] * cols[:, None, :]
    return s.astype(np.float32)


def initial_state(wl: Workload, seqs=None) -> np.ndarray:
    """Initial states fp32 [len(seqs)][H][d][d] (all sequences by default)."""
    seqs = range(wl.B) if seqs is None else seqs
    return np.stack([initial_state_seq(wl, b) for b in seqs])


def tokens(wl: Workload, t: int, calib: bool = False, seqs=None):
    """Decode inputs of step t: dict with q, k [B][H][d] and v [B][H][d] (bf16 bits, uint16),
    beta [B][H] fp32 and gate [B][H] or [B][H][d] fp32. ``calib`` draws the calibration
    stream (seed + 1000) instead. ``seqs`` keeps a subset of sequences (same draws)."""
    seed = wl.seed + (CALIB_SEED_OFFSET if calib else 0)
    rng = _rng(seed, wl.index, _STREAM_TOKENS, t)
    B, H, d = wl.B, wl.H, wl.d
    q = rng.normal(size=(B, H, d))
    k = rng.normal(size=(B, H, d))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    if wl.v_dist == "t3":
        v = rng.standard_t(3.0, size=(B, H, d))
    else:
        v = rng.normal(size=(B, H, d))
    beta = (1.0 / (1.0 + np.exp(-rng.normal(size=(B, H))))).astype(np.float32)
    g = unit_gates(wl)
    gate = np.broadcast_to(g, (B,) + g.shape).astype(np.float32)
    out = dict(q=f32_to_bf16_bits(q.astype(np.float32)), k=f32_to_bf16_bits(k.astype(np.float32)),
               v=f32_to_bf16_bits(v.astype(np.float32)), beta=beta, gate=np.ascontiguousarray(gate))
    if seqs is not None:
        idx = np.asarray(list(seqs))
        out = {name: np.ascontiguousarray(a[idx]) for name, a in out.items()}
    return out


def calib_tokens(wl: Workload, seqs=None):
    """The calibration stream: CALIB_STEPS steps stacked on a leading axis."""
    steps = [tokens(wl, t, calib=True, seqs=seqs) for t in range(CALIB_STEPS)]
    return {name: np.stack([s[name] for s in steps]) for name in steps[0]}


def half_bits(wl: Workload) -> np.ndarray:
    """Bit map [H][d] uint8 with exactly d/2 rows at 4 bits and d/2 at 8 bits per head."""
    rng = _rng(wl.seed, wl.index, _STREAM_BITS, 0)
    bits = np.full((wl.H, wl.d), 8, dtype=np.uint8)
    for h in range(wl.H):
        bits[h, rng.permutation(wl.d)[: wl.d // 2]] = 4
    return bits


def random_bits(H: int, d: int, choices=(2, 4, 6, 8), seed: int = 0) -> np.ndarray:
    """A seeded bit map drawn uniformly from ``choices`` (test inputs with mixed widths)."""
    rng = _rng(seed, 99, _STREAM_BITS, 1)
    return rng.choice(np.asarray(choices, dtype=np.uint8), size=(H, d)).astype(np.uint8)


def random_tile_state(B: int, H: int, d: int, seed: int = 0, scale: float = 0.1) -> np.ndarray:
    """Plain N(0, scale^2) states with log-normal row/column factors, for unit tests."""
    rng = _rng(seed, 98, _STREAM_STATE, 0)
    s = rng.normal(0.0, scale, size=(B, H, d, d))
    s *= np.exp(rng.normal(size=(B, H, d, 1))) * np.exp(rng.normal(size=(B, H, 1, d)))
    return s.astype(np.float32)


def random_weights(H: int, d: int, seed: int = 0) -> np.ndarray:
    """Non-uniform positive row-impact factors (mean 1 per head), for unit tests."""
    rng = _rng(seed, 97, _STREAM_STRUCTURE, 2)
    w = np.exp(rng.normal(0.0, 0.5, size=(H, d)))
    return (w / w.mean(axis=1, keepdims=True)).astype(np.float32)
