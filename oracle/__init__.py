"""Plain CPU oracle for the quantized gated Delta-rule decode step (test infrastructure).

This package is TEST INFRASTRUCTURE. Only the test suite, the package's ``smoke()`` check and
the benchmark's CPU-baseline leg may import it. It wraps ``stepq_oracle.c`` (plain C, compiled
here with gcc at -O2 -ffp-contract=off) through ctypes and shares no code with the CUDA
library. See the header of ``stepq_oracle.c`` for what each function follows in
"STEPQuant: When and Where Errors Matter in Delta-Rule Recurrent State Quantization".

Array conventions (NumPy, C-contiguous):
  state S          float32 [B][H][dk][dv]   (row = key channel i, column = value channel j)
  q, k             uint16 bf16 bits [B][H][dk];  v: uint16 [B][H][dv]
  beta             float32 [B][H];  gate: float32 [B][H] or [B][H][dk]
  bits             uint8 [H][dk];  w: float32 [H][dk]
  r, c             uint16 binary16 bits [B][H][dk], [B][H][dv]
  packed           uint8 [B * bytes_per_seq]
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "stepq_oracle.c"
_BUILD = _HERE / "_build"
_LIB_PATH = _BUILD / "libstepq_oracle.so"
_lib = None

ORC_OK, ORC_EINVAL, ORC_EUNSUPPORTED, ORC_EBUDGET = 0, 1, 2, 4


def build(force: bool = False) -> Path:
    """Compile the oracle library with gcc (plain C99, no fused multiply-add)."""
    _BUILD.mkdir(exist_ok=True)
    if force or not _LIB_PATH.exists() or _LIB_PATH.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB_PATH.with_suffix(f".{os.getpid()}.tmp")
        cmd = ["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-fPIC", "-shared", "-o", str(tmp), str(_SRC), "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(str(build()))
        _lib.orc_scale_to_half.restype = ctypes.c_uint16
        _lib.orc_scale_to_half.argtypes = [ctypes.c_double]
        _lib.orc_half_to_float.restype = ctypes.c_float
        _lib.orc_half_to_float.argtypes = [ctypes.c_uint16]
        _lib.orc_float_to_half.restype = ctypes.c_uint16
        _lib.orc_float_to_half.argtypes = [ctypes.c_float]
        _lib.orc_layout.restype = ctypes.c_int64
        _lib.orc_tile_bytes.restype = ctypes.c_int64
    return _lib


def _p(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else ctypes.c_void_p(0)


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


def _check(rc, what):
    if rc != ORC_OK:
        raise RuntimeError(f"oracle {what} failed with status {rc}")


# ---------------------------------------------------------------------------------------------
# scalars and layout
# ---------------------------------------------------------------------------------------------

def scale_to_half(x: float) -> int:
    return int(lib().orc_scale_to_half(float(x)))


def half_to_float(h) -> np.ndarray:
    return np.asarray(h, dtype=np.uint16).view(np.float16).astype(np.float32)


def layout(bits: np.ndarray, dv: int):
    """(head_off int64 [H], bytes_per_seq) for a bit map [H][dk]."""
    bits = _c(bits, np.uint8)
    H, dk = bits.shape
    head_off = np.zeros(H, dtype=np.int64)
    n = lib().orc_layout(H, dk, dv, _p(bits), _p(head_off))
    return head_off, int(n)


def tile_bytes(bits_row: np.ndarray, dv: int) -> int:
    bits_row = _c(bits_row, np.uint8)
    return int(lib().orc_tile_bytes(len(bits_row), dv, _p(bits_row)))


# ---------------------------------------------------------------------------------------------
# tile-level
# ---------------------------------------------------------------------------------------------

def quantise_tile(X, bits, r, c):
    X = _c(X, np.float32); bits = _c(bits, np.uint8); r = _c(r, np.uint16); c = _c(c, np.uint16)
    dk, dv = X.shape
    codes = np.zeros((dk, dv), dtype=np.int32)
    lib().orc_quantise_tile(dk, dv, _p(X), _p(bits), _p(r), _p(c), _p(codes))
    return codes


def pack_codes(codes, bits):
    codes = _c(codes, np.int32); bits = _c(bits, np.uint8)
    dk, dv = codes.shape
    out = np.zeros(tile_bytes(bits, dv), dtype=np.uint8)
    lib().orc_pack_codes(dk, dv, _p(bits), _p(codes), _p(out))
    return out


def unpack_codes(packed, bits, dv):
    packed = _c(packed, np.uint8); bits = _c(bits, np.uint8)
    dk = len(bits)
    codes = np.zeros((dk, dv), dtype=np.int32)
    lib().orc_unpack_codes(dk, dv, _p(bits), _p(packed), _p(codes))
    return codes


def fit_tile(X, w, bits, detail=False):
    X = _c(X, np.float32); w = _c(w, np.float32); bits = _c(bits, np.uint8)
    dk, dv = X.shape
    r = np.zeros(dk, dtype=np.uint16); c = np.zeros(dv, dtype=np.uint16)
    if not detail:
        lib().orc_fit_tile(dk, dv, _p(X), _p(w), _p(bits), _p(r), _p(c))
        return r, c
    c0 = np.zeros(dv, dtype=np.float32); z0 = np.zeros((dk, dv), dtype=np.int32)
    c1 = np.zeros(dv, dtype=np.float64)
    lib().orc_fit_tile_detail(dk, dv, _p(X), _p(w), _p(bits), _p(r), _p(c), _p(c0), _p(z0), _p(c1))
    return r, c, dict(c0=c0, z0=z0, c1=c1)


def fit_columns(X, w, bits, r, detail=False):
    """The column half of the fit at given binary16 row scales r (App. C.1): the no-clip start,
    the codes at (r, c0) and one weighted least-squares update; returns c (binary16 bits), and
    with ``detail`` also dict(c0, z0, c1) as fit_tile does."""
    X = _c(X, np.float32); w = _c(w, np.float32); bits = _c(bits, np.uint8); r = _c(r, np.uint16)
    dk, dv = X.shape
    c = np.zeros(dv, dtype=np.uint16)
    c0 = np.zeros(dv, dtype=np.float32); z0 = np.zeros((dk, dv), dtype=np.int32)
    c1 = np.zeros(dv, dtype=np.float64)
    lib().orc_fit_columns_detail(dk, dv, _p(X), _p(w), _p(bits), _p(r), _p(c), _p(c0), _p(z0), _p(c1))
    return (c, dict(c0=c0, z0=z0, c1=c1)) if detail else c


def ls_columns(X, w, bits, r, z, cfall):
    """The fixed-code least-squares column update alone (App. C.1) at binary16 row scales r and
    integer codes z [dk][dv]; a column with a zero denominator keeps cfall. Returns
    (c binary16 bits, c1 float64 before rounding)."""
    X = _c(X, np.float32); w = _c(w, np.float32); bits = _c(bits, np.uint8); r = _c(r, np.uint16)
    z = _c(z, np.int32); cfall = _c(cfall, np.float32)
    dk, dv = X.shape
    c = np.zeros(dv, dtype=np.uint16); c1 = np.zeros(dv, dtype=np.float64)
    lib().orc_ls_columns(dk, dv, _p(X), _p(w), _p(bits), _p(r), _p(z), _p(cfall), _p(c), _p(c1))
    return c, c1


def pack_tile(X, bits, r, c):
    X = _c(X, np.float32); bits = _c(bits, np.uint8); r = _c(r, np.uint16); c = _c(c, np.uint16)
    dk, dv = X.shape
    out = np.zeros(tile_bytes(bits, dv), dtype=np.uint8)
    lib().orc_pack_tile(dk, dv, _p(X), _p(bits), _p(r), _p(c), _p(out))
    return out


def unpack_tile(packed, bits, r, c, dv):
    packed = _c(packed, np.uint8); bits = _c(bits, np.uint8); r = _c(r, np.uint16); c = _c(c, np.uint16)
    dk = len(bits)
    X = np.zeros((dk, dv), dtype=np.float32)
    lib().orc_unpack_tile(dk, dv, _p(packed), _p(bits), _p(r), _p(c), _p(X))
    return X


def delta_update(S, q, k, v, beta, gate):
    """One gated Delta-rule update in float64. gate: scalar or [dk]. Returns (X, o)."""
    S = _c(S, np.float64)
    dk, dv = S.shape
    g = np.broadcast_to(np.asarray(gate, dtype=np.float64), (dk,)).copy()
    q = _c(q, np.float64); k = _c(k, np.float64); v = _c(v, np.float64)
    X = np.zeros((dk, dv)); o = np.zeros(dv)
    lib().orc_delta_update(dk, dv, _p(S), _p(q), _p(k), _p(v), ctypes.c_double(float(beta)), _p(g),
                           _p(X), _p(o))
    return X, o


def int8_quantise_tile(X):
    X = _c(X, np.float32)
    dk, dv = X.shape
    codes = np.zeros((dk, dv), dtype=np.int8); s = np.zeros(dk, dtype=np.uint16)
    lib().orc_int8_quantise_tile(dk, dv, _p(X), _p(codes), _p(s))
    return codes, s


# ---------------------------------------------------------------------------------------------
# batch-level (the same calls as the CUDA library's C-ABI)
# ---------------------------------------------------------------------------------------------

def _dims(S_or_shape):
    return S_or_shape.shape if hasattr(S_or_shape, "shape") else S_or_shape


def fit_scales(S, w, bits, nthreads=0):
    S = _c(S, np.float32); w = _c(w, np.float32); bits = _c(bits, np.uint8)
    B, H, dk, dv = S.shape
    r = np.zeros((B, H, dk), dtype=np.uint16); c = np.zeros((B, H, dv), dtype=np.uint16)
    _check(lib().orc_fit_scales(B, H, dk, dv, _p(S), _p(w), _p(bits), _p(r), _p(c), nthreads), "fit_scales")
    return r, c


def pack_state(S, bits, r, c, nthreads=0):
    S = _c(S, np.float32); bits = _c(bits, np.uint8); r = _c(r, np.uint16); c = _c(c, np.uint16)
    B, H, dk, dv = S.shape
    head_off, bps = layout(bits, dv)
    packed = np.zeros(B * bps, dtype=np.uint8)
    _check(lib().orc_pack_state(B, H, dk, dv, _p(S), _p(bits), _p(head_off), ctypes.c_int64(bps),
                                _p(r), _p(c), _p(packed), nthreads), "pack_state")
    return packed


def unpack_state(packed, bits, r, c, nthreads=0):
    packed = _c(packed, np.uint8); bits = _c(bits, np.uint8); r = _c(r, np.uint16); c = _c(c, np.uint16)
    B, H, dk = r.shape
    dv = c.shape[2]
    head_off, bps = layout(bits, dv)
    S = np.zeros((B, H, dk, dv), dtype=np.float32)
    _check(lib().orc_unpack_state(B, H, dk, dv, _p(packed), _p(bits), _p(head_off), ctypes.c_int64(bps),
                                  _p(r), _p(c), _p(S), nthreads), "unpack_state")
    return S


def decode_step(tok, bits, w, packed, r, c, nthreads=0):
    """One quantized decode step over all tiles. tok: dict(q, k, v, beta, gate).
    Returns (packed_out, r_out, c_out, o)."""
    q = _c(tok["q"], np.uint16); k = _c(tok["k"], np.uint16); v = _c(tok["v"], np.uint16)
    beta = _c(tok["beta"], np.float32); gate = _c(tok["gate"], np.float32)
    bits = _c(bits, np.uint8); w = _c(w, np.float32)
    packed = _c(packed, np.uint8); r = _c(r, np.uint16); c = _c(c, np.uint16)
    B, H, dk = q.shape
    dv = v.shape[2]
    gpc = int(gate.ndim == 3)
    head_off, bps = layout(bits, dv)
    p_out = np.zeros_like(packed); r_out = np.zeros_like(r); c_out = np.zeros_like(c)
    o = np.zeros((B, H, dv), dtype=np.float32)
    _check(lib().orc_decode_step(B, H, dk, dv, gpc, _p(q), _p(k), _p(v), _p(beta), _p(gate), _p(bits),
                                 _p(w), _p(head_off), ctypes.c_int64(bps), _p(packed), _p(r), _p(c),
                                 _p(p_out), _p(r_out), _p(c_out), _p(o), nthreads), "decode_step")
    return p_out, r_out, c_out, o


def prefill_chunk(toks, bits, w, packed, r, c, nthreads=0):
    """A prefill chunk: toks holds q, k, v, beta, gate with a leading token axis [C][B][H]...;
    returns (packed_out, r_out, c_out, o [C][B][H][dv])."""
    q = _c(toks["q"], np.uint16); k = _c(toks["k"], np.uint16); v = _c(toks["v"], np.uint16)
    beta = _c(toks["beta"], np.float32); gate = _c(toks["gate"], np.float32)
    bits = _c(bits, np.uint8); w = _c(w, np.float32)
    packed = _c(packed, np.uint8); r = _c(r, np.uint16); c = _c(c, np.uint16)
    C, B, H, dk = q.shape
    dv = v.shape[3]
    gpc = int(gate.ndim == 4)
    head_off, bps = layout(bits, dv)
    p_out = np.zeros_like(packed); r_out = np.zeros_like(r); c_out = np.zeros_like(c)
    o = np.zeros((C, B, H, dv), dtype=np.float32)
    _check(lib().orc_prefill_chunk(C, B, H, dk, dv, gpc, _p(q), _p(k), _p(v), _p(beta), _p(gate), _p(bits),
                                   _p(w), _p(head_off), ctypes.c_int64(bps), _p(packed), _p(r), _p(c),
                                   _p(p_out), _p(r_out), _p(c_out), _p(o), nthreads), "prefill_chunk")
    return p_out, r_out, c_out, o


def leap_window(toks, codes, s, nthreads=0):
    """A window of W tokens on the per-window 8-bit state (LeapQuant's per-window quantisation
    as read from its abstract): toks holds q, k, v, beta, gate with a leading token axis
    [W][B][H]...; the state is the rowwise-absmax INT8 codes [B][H][dk][dv] with scales s
    (binary16 bits) [B][H][dk]. Every token's readout comes from the exact (float64) running
    state; the window's final state is quantised once. Returns (codes_out, s_out, o [W][B][H][dv])."""
    q = _c(toks["q"], np.uint16); k = _c(toks["k"], np.uint16); v = _c(toks["v"], np.uint16)
    beta = _c(toks["beta"], np.float32); gate = _c(toks["gate"], np.float32)
    codes = _c(codes, np.int8); s = _c(s, np.uint16)
    W, B, H, dk = q.shape
    dv = v.shape[3]
    gpc = int(gate.ndim == 4)
    c_out = np.zeros_like(codes); s_out = np.zeros_like(s)
    o = np.zeros((W, B, H, dv), dtype=np.float32)
    _check(lib().orc_leap_window(W, B, H, dk, dv, gpc, _p(q), _p(k), _p(v), _p(beta), _p(gate), _p(codes),
                                 _p(s), _p(c_out), _p(s_out), _p(o), nthreads), "leap_window")
    return c_out, s_out, o


def decode_step_fp32(tok, S, nthreads=0):
    q = _c(tok["q"], np.uint16); k = _c(tok["k"], np.uint16); v = _c(tok["v"], np.uint16)
    beta = _c(tok["beta"], np.float32); gate = _c(tok["gate"], np.float32)
    S = _c(S, np.float32)
    B, H, dk, dv = S.shape
    S_out = np.zeros_like(S); o = np.zeros((B, H, dv), dtype=np.float32)
    _check(lib().orc_decode_step_fp32(B, H, dk, dv, int(gate.ndim == 3), _p(q), _p(k), _p(v), _p(beta),
                                      _p(gate), _p(S), _p(S_out), _p(o), nthreads), "decode_step_fp32")
    return S_out, o


def int8_quantise_state(S):
    S = _c(S, np.float32)
    B, H, dk, dv = S.shape
    codes = np.zeros((B, H, dk, dv), dtype=np.int8); s = np.zeros((B, H, dk), dtype=np.uint16)
    lib().orc_int8_quantise_state(B, H, dk, dv, _p(S), _p(codes), _p(s))
    return codes, s


def decode_step_int8(tok, codes, s, nthreads=0):
    q = _c(tok["q"], np.uint16); k = _c(tok["k"], np.uint16); v = _c(tok["v"], np.uint16)
    beta = _c(tok["beta"], np.float32); gate = _c(tok["gate"], np.float32)
    codes = _c(codes, np.int8); s = _c(s, np.uint16)
    B, H, dk, dv = codes.shape
    c_out = np.zeros_like(codes); s_out = np.zeros_like(s); o = np.zeros((B, H, dv), dtype=np.float32)
    _check(lib().orc_decode_step_int8(B, H, dk, dv, int(gate.ndim == 3), _p(q), _p(k), _p(v), _p(beta),
                                      _p(gate), _p(codes), _p(s), _p(c_out), _p(s_out), _p(o), nthreads),
           "decode_step_int8")
    return c_out, s_out, o


# ---------------------------------------------------------------------------------------------
# offline calibration
# ---------------------------------------------------------------------------------------------

def row_impact(calib):
    """w [H][dk] from a calibration stream dict(q, k, beta, gate) with a leading step axis."""
    q = _c(calib["q"], np.uint16); k = _c(calib["k"], np.uint16)
    beta = _c(calib["beta"], np.float32); gate = _c(calib["gate"], np.float32)
    T, B, H, dk = q.shape
    w = np.zeros((H, dk), dtype=np.float32)
    _check(lib().orc_row_impact(T, B, H, dk, int(gate.ndim == 4), _p(q), _p(k), _p(beta), _p(gate), _p(w)),
           "row_impact")
    return w


def float_to_half(x: float) -> int:
    """The binary16 bits of an FP16 pivot value (nearest-even, saturating)."""
    return int(lib().orc_float_to_half(float(x)))


def calib_distortion_bits(S, w, bits, nthreads=0):
    """(d_row [H][dk], d_head [H]) under the per-row bit map bits [H][dk] (16 = FP16 pivot)."""
    S = _c(S, np.float32); w = _c(w, np.float32); bits = _c(bits, np.uint8)
    B, H, dk, dv = S.shape
    d_row = np.zeros((H, dk)); d_head = np.zeros(H)
    _check(lib().orc_calib_distortion_bits(B, H, dk, dv, _p(S), _p(w), _p(bits), _p(d_row), _p(d_head), nthreads),
           "calib_distortion_bits")
    return d_row, d_head


def calib_distortion(S, w, b, nthreads=0):
    """(d_row [H][dk], d_head [H]) at uniform width b over the sample states S [B][H][dk][dv]."""
    S = _c(S, np.float32); w = _c(w, np.float32)
    B, H, dk, dv = S.shape
    d_row = np.zeros((H, dk)); d_head = np.zeros(H)
    _check(lib().orc_calib_distortion(B, H, dk, dv, _p(S), _p(w), int(b), _p(d_row), _p(d_head), nthreads),
           "calib_distortion")
    return d_row, d_head


def allocate_bits(J, cand, budget, mode):
    """Bit widths (uint8 [n_units]) minimising sum J[u][k] with exactly ``budget`` bits.
    mode 1: multiple-choice DP; mode 0: Lagrangian allocation with repair."""
    J = _c(J, np.float64)
    cand = _c(cand, np.int32)
    n, nc = J.shape
    out = np.zeros(n, dtype=np.uint8)
    rc = lib().orc_allocate_bits(n, nc, _p(cand), _p(J), ctypes.c_int64(int(budget)), int(mode), _p(out))
    if rc != ORC_OK:
        raise ValueError(f"oracle allocate_bits failed with status {rc}")
    return out


# The horizon H of the lifetime sum (App. A.3) is not stated; 2048, the length of the calibration
# segments (App. C.2), is taken for it.
LIFETIME_HORIZON = 2048


def mean_log_retention(gate):
    """ell_u = E_cal[log r_{t,u}] (App. A.3, "Mean log retention"): the mean over the steps and
    sequences of a calibration gate stream, gate [T][B][H] (head units, result [H]) or
    [T][B][H][dk] (key-channel units, result [H][dk])."""
    g = np.asarray(gate, dtype=np.float64)
    return np.log(g).mean(axis=(0, 1))


def lifetime(ell, horizon=LIFETIME_HORIZON):
    """L_u = sum_{j=0}^{horizon-1} exp(2 j ell_u) (App. A.3), summed term by term: the squared
    error a unit keeps over the horizon, per unit of squared error injected once, when each step
    retains exp(ell_u) of it."""
    ell = np.asarray(ell, dtype=np.float64)
    total = np.zeros_like(ell)
    for j in range(int(horizon)):
        total += np.exp(2.0 * j * ell)
    return total


def objective(d, ell, horizon=LIFETIME_HORIZON):
    """J_u(b) = L_u d_u(b): lifetime-weighted distortion, d [n_units][n_cand], ell [n_units]."""
    return lifetime(ell, horizon)[:, None] * np.asarray(d, dtype=np.float64)


def pivot_order(score):
    """Units by descending score, ties to the lower index."""
    score = np.asarray(score, dtype=np.float64)
    return np.lexsort((np.arange(score.size), -score))


def calibrate(alloc, candidates, nominal_bits, S0, calib, n_pivots=0, horizon=LIFETIME_HORIZON):
    """The offline calibration done by the oracle (App. A.3, B.3, C.2): returns
    (bits uint8 [H][dk] or None, w float32 [H][dk]).

    alloc: "dp_head" (head units, multiple-choice DP, Eq. 17 distortion) or "lagrange_row"
    (key-row units, Lagrangian allocation with repair, Eq. 18 distortion); any other value
    returns bits=None (the caller supplies a fixed map). S0: the sample states [B][H][dk][dv];
    calib: the calibration stream. Each unit's lifetime L_u comes from the mean log retention of
    the stream's gates (App. A.3): a head unit averages the log gate over its key channels, a
    key-row unit under a head gate takes its head's value; ``horizon`` is the H of that sum.

    n_pivots > 0 keeps that many units in FP16 (width 16, App. C.2, Table C1):
      key rows: ranked by the lifetime-weighted reduction of error from the integer format at
        the nominal width to FP16, L_u (d_u(b_nominal) - d_u(16)); with the pivots fixed the
        candidate distortions of the other rows are measured again with the pivots left out
        of the shared column fit, and those rows are allocated;
      heads: allocated first; the heads with the largest residual risk L_u d_u(b_u) become
        pivots and the other heads are allocated again.
    Each pivot unit counts 8 bits toward the integer budget n_units * nominal_bits and its
    other 8 bits come on top (the (16 - 8) accounting of App. D), so the remaining units share
    n_units * nominal_bits - 8 n_pivots bits."""
    w = row_impact(calib)
    H, dk = w.shape
    if alloc not in ("dp_head", "lagrange_row"):
        return None, w
    cand = [int(b) for b in candidates]
    ell = mean_log_retention(calib["gate"])                    # [H] or [H][dk]
    drows, dheads = [], []
    for b in cand:
        dr, dh = calib_distortion(S0, w, b)
        drows.append(dr)
        dheads.append(dh)
    if alloc == "dp_head":
        dist = np.stack(dheads, axis=1)                          # [H][n_cand]
        ell_h = ell if ell.ndim == 1 else ell.mean(axis=1)
        J = objective(dist, ell_h, horizon)
        bh = allocate_bits(J, cand, nominal_bits * H, mode=1)
        if n_pivots:
            risk = J[np.arange(H), [cand.index(int(b)) for b in bh]]
            piv = np.sort(pivot_order(risk)[:n_pivots])
            rest = np.setdiff1d(np.arange(H), piv)
            bh = bh.astype(np.uint8)
            bh[rest] = allocate_bits(J[rest], cand, nominal_bits * H - 8 * n_pivots, mode=1)
            bh[piv] = 16
        return np.repeat(bh[:, None], dk, axis=1).astype(np.uint8), w
    ell_r = ell.reshape(-1) if ell.ndim == 2 else np.repeat(ell, dk)
    n = H * dk
    if not n_pivots:
        dist = np.stack([dr.reshape(-1) for dr in drows], axis=1)   # [H*dk][n_cand]
        br = allocate_bits(objective(dist, ell_r, horizon), cand, nominal_bits * n, mode=0)
        return br.reshape(H, dk).astype(np.uint8), w
    d16, _ = calib_distortion(S0, w, 16)
    dnom = drows[cand.index(int(nominal_bits))] if int(nominal_bits) in cand else \
        calib_distortion(S0, w, nominal_bits)[0]
    score = lifetime(ell_r, horizon) * (dnom.reshape(-1) - d16.reshape(-1))
    piv = np.sort(pivot_order(score)[:n_pivots])
    rest = np.setdiff1d(np.arange(n), piv)
    dist = []
    for b in cand:
        m = np.full(n, b, dtype=np.uint8)
        m[piv] = 16
        dist.append(calib_distortion_bits(S0, w, m.reshape(H, dk))[0].reshape(-1))
    dist = np.stack(dist, axis=1)
    br = np.zeros(n, dtype=np.uint8)
    br[rest] = allocate_bits(objective(dist[rest], ell_r[rest], horizon), cand, nominal_bits * n - 8 * n_pivots,
                             mode=0)
    br[piv] = 16
    return br.reshape(H, dk), w
