"""State container and offline calibration built on the libstepq entry points.

``QuantizedState`` keeps one layer's packed recurrent states (codes, fp16 row/column scales,
the frozen bit map, row-impact vector and packed layout) resident on the GPU and advances them
with the fused decode kernel. ``calibrate`` runs the offline part of STEPQuant (App. C.2): row
impact (App. B.3) and candidate distortions (App. A.3) on the GPU, lifetime weighting (§3.2,
App. A.3) and the discrete allocation (multiple-choice DP or Lagrangian) in the host library.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from . import api


@dataclass
class Layout:
    bits: np.ndarray          # uint8 [H][d] (host copy)
    head_off: np.ndarray      # int64 [H]
    bytes_per_seq: int
    d: int
    bits_dev: torch.Tensor
    head_off_dev: torch.Tensor

    @classmethod
    def build(cls, bits: np.ndarray, d: int, device="cuda") -> "Layout":
        bits = np.ascontiguousarray(np.asarray(bits, dtype=np.uint8))
        head_off, bps, _ = api.stepq_packed_layout(bits, d, B=1)
        return cls(bits, head_off, bps, d, torch.from_numpy(bits).to(device),
                   torch.from_numpy(head_off).to(device))

    @property
    def H(self) -> int:
        return self.bits.shape[0]

    @property
    def pivots(self) -> int:
        """1 when the bit map holds FP16 pivot rows (width 16)."""
        return int((self.bits == 16).any())

    @property
    def mixed(self) -> int:
        """1 when some head's key rows have different widths (a row-level allocation)."""
        return int((self.bits != self.bits[:, :1]).any())

    @property
    def widths(self) -> int:
        """Bit mask of the row widths the bit map holds (bit b for width b)."""
        return api.width_mask(self.bits)


class QuantizedState:
    """Packed states of B sequences x H heads (one layer)."""

    def __init__(self, layout: Layout, w: torch.Tensor, packed: torch.Tensor, r: torch.Tensor, c: torch.Tensor):
        self.layout, self.w, self.packed, self.r, self.c = layout, w, packed, r, c

    @classmethod
    def from_fp32(cls, S: torch.Tensor, layout: Layout, w: torch.Tensor) -> "QuantizedState":
        """Post-training quantisation of initial states S [B,H,d,d] (fit, then pack)."""
        r, c = api.stepq_fit_scales(S, w, layout.bits_dev)
        packed = api.stepq_pack_state(S, layout.bits_dev, layout.head_off_dev, layout.bytes_per_seq, r, c)
        return cls(layout, w, packed, r, c)

    @property
    def B(self) -> int:
        return self.r.shape[0]

    def unpack(self) -> torch.Tensor:
        L = self.layout
        return api.stepq_unpack_state(self.packed, L.bits_dev, L.head_off_dev, L.bytes_per_seq, self.r, self.c)

    def step(self, q, k, v, beta, gate, o=None) -> torch.Tensor:
        """One decode token for every sequence, updating the state in place; returns o [B,H,d]."""
        L = self.layout
        _, _, _, o = api.stepq_decode_step(q, k, v, beta, gate, L.bits_dev, self.w, L.head_off_dev,
                                           L.bytes_per_seq, self.packed, self.r, self.c,
                                           self.packed, self.r, self.c, o, pivots=L.pivots, mixed=L.mixed,
                                           widths=L.widths)
        return o

    def nbytes(self) -> int:
        return self.packed.numel() + 2 * (self.r.numel() + self.c.numel())


class WindowState:
    """States of B sequences x H heads on the per-window 8-bit format (LeapQuant's per-window
    quantisation): rowwise-absmax INT8 between windows, the open window's buffered updates in
    fp32. step() decodes one token; every `window` tokens the state is requantised once."""

    def __init__(self, codes: torch.Tensor, s: torch.Tensor, window: int):
        B, H, d, _ = codes.shape
        self.codes, self.s, self.window, self.t = codes, s, int(window), 0
        dev = codes.device
        self.kbuf = torch.empty((window, B, H, d), dtype=torch.bfloat16, device=dev)
        self.ubuf = torch.empty((window, B, H, d), dtype=torch.float32, device=dev)
        self.lbuf = torch.empty((window, B, H), dtype=torch.float32, device=dev)

    @classmethod
    def from_fp32(cls, S: torch.Tensor, window: int) -> "WindowState":
        codes, s = api.stepq_int8_quantize_state(S)
        return cls(codes, s, window)

    def step(self, q, k, v, beta, gate, o=None) -> torch.Tensor:
        """One decode token for every sequence; returns o [B,H,d]."""
        o = api.stepq_leap_step(self.window, self.t, q, k, v, beta, gate, self.codes, self.s, self.kbuf, self.ubuf,
                                self.lbuf, o)
        self.t = (self.t + 1) % self.window
        return o

    def nbytes(self) -> int:
        return self.codes.numel() + 2 * self.s.numel()


# The horizon H of the lifetime sum (App. A.3) is not stated; 2048, the length of the calibration
# segments (App. C.2), is taken for it.
LIFETIME_HORIZON = 2048


def mean_log_retention(gate) -> np.ndarray:
    """ell_u = E[log r_{t,u}] over a calibration gate stream (App. A.3, mean log retention):
    gate [T][B][H] gives one value per head [H], gate [T][B][H][d] one per key channel [H][d]."""
    g = gate.detach().cpu().numpy() if isinstance(gate, torch.Tensor) else np.asarray(gate)
    return np.log(g.astype(np.float64)).mean(axis=(0, 1))


def lifetime(ell, horizon: int = LIFETIME_HORIZON) -> np.ndarray:
    """L_u = sum over 0 <= j < horizon of exp(2 j ell_u) (App. A.3): the squared error a unit
    keeps over the horizon per unit injected once. Summed term by term in increasing j, in
    float64: the discrete allocation compares lifetime-weighted costs of nearly equal size, so
    the series is evaluated in its plain order rather than through a closed form whose last bits
    differ."""
    x = 2.0 * np.asarray(ell, dtype=np.float64)
    total = np.zeros_like(x)
    for j in range(int(horizon)):
        total += np.exp(j * x)
    return total


def calibrate(alloc: str, candidates, nominal_bits: int, S0: torch.Tensor, calib: dict, n_pivots: int = 0,
              horizon: int = LIFETIME_HORIZON):
    """Offline calibration of one layer. Returns (bits uint8 numpy [H][d], w float32 [H][d] on GPU).

    alloc: "dp_head" (head units, Eq. 17 distortion, multiple-choice DP) or "lagrange_row"
    (key-row units, Eq. 18 distortion, Lagrangian allocation with repair).
    S0: the sample states [B,H,d,d] on the GPU; calib: the calibration stream as GPU tensors
    with a leading step axis. Unit lifetimes come from the stream's mean log retention (App.
    A.3): a head unit averages the log gate over its key channels, a key row under a head gate
    takes its head's; ``horizon`` is the number of steps the lifetime sums over.
    n_pivots: units kept in FP16 (width 16; App. C.2): key rows ranked by the lifetime-weighted
    error reduction L_u (d_u(nominal) - d_u(16)), then the other rows' distortions measured
    again without the pivots in the column fit; heads ranked by residual risk L_u d_u(b_u)
    after a first allocation. A pivot counts 8 bits of the integer budget (App. D accounting).
    """
    w = api.stepq_row_impact(calib["q"], calib["k"], calib["beta"], calib["gate"])
    H, d = w.shape
    cand = [int(b) for b in candidates]
    ell = mean_log_retention(calib["gate"])
    rows, heads = [], []
    for b in cand:
        d_row, d_head = api.stepq_calib_distortion(S0, w, b)
        rows.append(d_row.cpu().numpy())
        heads.append(d_head.cpu().numpy())
    if alloc == "dp_head":
        dist = np.stack(heads, axis=1)
        ell_h = ell if ell.ndim == 1 else ell.mean(axis=1)
        J = lifetime(ell_h, horizon)[:, None] * dist
        bh = api.stepq_allocate_bits(J, cand, nominal_bits * H, mode=1)
        if n_pivots:
            risk = J[np.arange(H), [cand.index(int(b)) for b in bh]]
            piv = np.sort(np.lexsort((np.arange(H), -risk))[:n_pivots])
            rest = np.setdiff1d(np.arange(H), piv)
            bh = bh.astype(np.uint8)
            bh[rest] = api.stepq_allocate_bits(J[rest], cand, nominal_bits * H - 8 * n_pivots, mode=1)
            bh[piv] = 16
        return np.repeat(bh[:, None], d, axis=1).astype(np.uint8), w
    if alloc == "lagrange_row":
        ell_r = ell.reshape(-1) if ell.ndim == 2 else np.repeat(ell, d)
        n = H * d
        L = lifetime(ell_r, horizon)
        if not n_pivots:
            dist = np.stack([x.reshape(-1) for x in rows], axis=1)
            br = api.stepq_allocate_bits(L[:, None] * dist, cand, nominal_bits * n, mode=0)
            return br.reshape(H, d).astype(np.uint8), w
        d16 = api.stepq_calib_distortion(S0, w, 16)[0].cpu().numpy().reshape(-1)
        dnom = (rows[cand.index(int(nominal_bits))] if int(nominal_bits) in cand else
                api.stepq_calib_distortion(S0, w, nominal_bits)[0].cpu().numpy()).reshape(-1)
        score = L * (dnom - d16)
        piv = np.sort(np.lexsort((np.arange(n), -score))[:n_pivots])
        rest = np.setdiff1d(np.arange(n), piv)
        dist = []
        for b in cand:
            m = np.full(n, b, dtype=np.uint8)
            m[piv] = 16
            bits_dev = torch.from_numpy(m.reshape(H, d)).to(S0.device)
            dist.append(api.stepq_calib_distortion_bits(S0, w, bits_dev)[0].cpu().numpy().reshape(-1))
        dist = np.stack(dist, axis=1)
        br = np.zeros(n, dtype=np.uint8)
        br[rest] = api.stepq_allocate_bits(L[rest, None] * dist[rest], cand, nominal_bits * n - 8 * n_pivots, mode=0)
        br[piv] = 16
        return br.reshape(H, d), w
    raise ValueError(f"unknown allocation {alloc!r}")


TOKEN_FIELDS = ("q", "k", "v", "beta", "gate")


def _token_parts(tok: dict):
    """(name, uint8 view, dtype, shape, offset) of each token input in the packed order; every
    part starts on a 16-byte boundary (the library's alignment rule)."""
    parts, off = [], 0
    for name in TOKEN_FIELDS:
        a = np.ascontiguousarray(tok[name])
        raw = a.view(np.uint8).reshape(-1)
        parts.append((name, raw, a.dtype, a.shape, off))
        off += (raw.size + 15) // 16 * 16
    return parts, off


def pack_tokens(tok: dict) -> np.ndarray:
    """The token inputs of one step (or one chunk) as one contiguous byte buffer:
    q | k | v | beta | gate, so that moving them to the GPU is a single copy."""
    parts, size = _token_parts(tok)
    buf = np.zeros(size, dtype=np.uint8)
    for _, raw, _, _, off in parts:
        buf[off:off + raw.size] = raw
    return buf


def token_views(buf: torch.Tensor, like: dict) -> dict:
    """Typed views (q, k, v bf16; beta, gate fp32) into a packed token buffer `buf` (uint8, on
    any device) laid out by pack_tokens for host tokens shaped like `like`."""
    parts, size = _token_parts(like)
    if buf.numel() != size:
        raise ValueError(f"packed token buffer holds {buf.numel()} bytes, expected {size}")
    out = {}
    for name, raw, dtype, shape, off in parts:
        seg = buf[off:off + raw.size]
        out[name] = seg.view(torch.bfloat16 if dtype == np.uint16 else torch.float32).view(shape)
    return out


def to_device_tokens(tok: dict, device="cuda") -> dict:
    """Host token arrays (bf16 bit patterns as uint16) to GPU tensors of the right dtypes."""
    out = {}
    for name in ("q", "k", "v"):
        out[name] = torch.from_numpy(np.ascontiguousarray(tok[name]).view(np.int16)).to(device).view(torch.bfloat16)
    out["beta"] = torch.from_numpy(np.ascontiguousarray(tok["beta"], dtype=np.float32)).to(device)
    out["gate"] = torch.from_numpy(np.ascontiguousarray(tok["gate"], dtype=np.float32)).to(device)
    return out
