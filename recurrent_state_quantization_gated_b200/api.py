"""Python binding of libstepq: the entry points of include/stepq.h under the same names,
taking PyTorch CUDA tensors. Argument marshalling only; every step runs in the CUDA library.

Tensor conventions (all C-contiguous; device tensors on the current CUDA device):
  S float32 [B,H,d,d] (row = key channel, column = value channel)
  q, k, v bfloat16 [B,H,d]; beta float32 [B,H]; gate float32 [B,H] or [B,H,d]
  bits uint8 [H,d]; w float32 [H,d]; head_off int64 [H]
  r, c float16 [B,H,d]; packed uint8 [B*bytes_per_seq]; o float32 [B,H,d]
  INT8 state: codes int8 [B,H,d,d], s float16 [B,H,d]
All calls are queued on torch's current CUDA stream.
"""
from __future__ import annotations

import ctypes
import weakref

import numpy as np
import torch

from ._lib import Dims, call, lib

__all__ = [
    "stepq_packed_layout", "stepq_fit_scales", "stepq_pack_state", "stepq_unpack_state",
    "stepq_decode_step", "stepq_decode_step_split", "stepq_prefill_chunk",
    "stepq_prefill_chunk_seq", "stepq_prefill_chunk_wy", "stepq_decode_step_fp32", "stepq_int8_quantize_state",
    "stepq_decode_step_int8", "stepq_leap_step", "stepq_row_impact", "stepq_calib_distortion", "stepq_calib_distortion_bits", "stepq_calib_distortion_static",
    "stepq_allocate_bits",
    "stepq_read_device_flags", "stepq_selftest_wait", "stepq_build_info",
]


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t: torch.Tensor, dtype: torch.dtype, name: str):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name} is on {t.device}; the calls run on the current device, "
                         f"cuda:{torch.cuda.current_device()}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _sizes(**tensors):
    """Each tensor (name=(tensor, elements)) must hold at least that many elements, so that no
    kernel reads or writes past a buffer given through the C ABI (which sees only pointers)."""
    for name, (t, n) in tensors.items():
        if t is None:
            continue
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor")
        if t.numel() < n:
            raise ValueError(f"{name}: {t.numel()} elements, the call needs {n}")


_LAYOUTS_CHECKED = {}


def _check_layout(bits, head_off, bytes_per_seq):
    """head_off and bytes_per_seq must be the packed layout of the bit map (stepq_packed_layout:
    each head's range holds its tile, and the sequence holds every head). Checked on the host
    the first time a (bits, head_off) pair is seen -- one device-to-host read of each, then
    remembered while neither tensor is modified in place -- so make the first call with a new
    layout outside CUDA-graph capture; during capture an unchecked pair is left to the kernels,
    which check every tile's range themselves, skip a tile that does not fit and raise bit 2 of
    the device error word."""
    if not (isinstance(bits, torch.Tensor) and isinstance(head_off, torch.Tensor)):
        return
    key = (id(bits), bits._version, id(head_off), head_off._version, int(bytes_per_seq))
    if key in _LAYOUTS_CHECKED:
        return
    if bits.is_cuda and torch.cuda.is_current_stream_capturing():
        return
    if bits.dim() != 2 or head_off.numel() < bits.shape[0]:
        raise ValueError(f"bits must be [H, d] and head_off [H]; got {tuple(bits.shape)} and {tuple(head_off.shape)}")
    H, d = bits.shape
    want_off, want_bps, _ = stepq_packed_layout(bits.detach().cpu().numpy(), d)
    got = head_off.detach().reshape(-1)[:H].cpu().numpy()
    if not np.array_equal(got, want_off) or int(bytes_per_seq) != want_bps:
        raise ValueError("head_off / bytes_per_seq do not match the bit map's packed layout "
                         f"(bytes_per_seq {int(bytes_per_seq)}, expected {want_bps}); "
                         "take them from stepq_packed_layout(bits)")
    _LAYOUTS_CHECKED[key] = True
    for t in (bits, head_off):
        weakref.finalize(t, _LAYOUTS_CHECKED.pop, key, None)


def _dims(B, H, d, gate_per_channel=0, pivots=0, mixed=0, widths=0):
    return Dims(int(B), int(H), int(d), int(d), int(gate_per_channel), int(pivots), int(mixed), int(widths))


def width_mask(bits) -> int:
    """The bit mask of the row widths a bit map holds (bit b for width b), from a host array or
    a tensor (a device tensor is read back: one synchronisation)."""
    if isinstance(bits, torch.Tensor):
        vals = torch.unique(bits).cpu().tolist()
    else:
        vals = np.unique(np.asarray(bits)).tolist()
    m = 0
    for b in vals:
        m |= 1 << int(b)
    return m


def _widths(bits, widths, mixed):
    """The widths field of a decode call: as given, else read from the bit map when the launch
    takes the per-row path (mixed) -- except while a CUDA graph is being captured, where no
    device read is possible and 0 (undeclared: the generic per-row code, same results) is used."""
    if widths is not None:
        return int(widths)
    if not mixed:
        return 0
    if isinstance(bits, torch.Tensor) and bits.is_cuda and torch.cuda.is_current_stream_capturing():
        return 0
    return width_mask(bits)


def _has_pivots(bits, pivots):
    """The pivots flag of a decode call: as given, else read from the bit map (a device
    reduction and a host read; pass it to avoid both)."""
    return int(bool((bits == 16).any().item())) if pivots is None else int(bool(pivots))


def _has_mixed(bits, mixed):
    """The mixed flag of a decode call (some head's key rows have different widths): as given,
    else read from the bit map (a device reduction and a host read; pass it to avoid both)."""
    if mixed is not None:
        return int(bool(mixed))
    return int(bool((bits != bits[:, :1]).any().item()))


def stepq_build_info() -> str:
    return lib().stepq_build_info().decode()


def stepq_packed_layout(bits_host, dv: int, B: int = 1):
    """(head_off int64 numpy [H], bytes_per_seq, total_bytes) for a host bit map [H][dk]."""
    bits_host = np.ascontiguousarray(np.asarray(bits_host, dtype=np.uint8))
    H, dk = bits_host.shape
    head_off = np.zeros(H, dtype=np.int64)
    bps = ctypes.c_int64(0)
    total = ctypes.c_int64(0)
    call("stepq_packed_layout", Dims(B, H, dk, dv, 0), bits_host.ctypes.data_as(ctypes.c_void_p),
         head_off.ctypes.data_as(ctypes.c_void_p), ctypes.byref(bps), ctypes.byref(total))
    return head_off, bps.value, total.value


def stepq_fit_scales(S, w, bits, r=None, c=None):
    B, H, d, _ = S.shape
    r = torch.empty((B, H, d), dtype=torch.float16, device=S.device) if r is None else r
    c = torch.empty((B, H, d), dtype=torch.float16, device=S.device) if c is None else c
    _sizes(S=(S, B * H * d * d), w=(w, H * d), bits=(bits, H * d), r=(r, B * H * d), c=(c, B * H * d))
    call("stepq_fit_scales", _dims(B, H, d), _ptr(S, torch.float32, "S"), _ptr(w, torch.float32, "w"),
         _ptr(bits, torch.uint8, "bits"), _ptr(r, torch.float16, "r"), _ptr(c, torch.float16, "c"), _stream())
    return r, c


def stepq_pack_state(S, bits, head_off, bytes_per_seq, r, c, packed=None):
    B, H, d, _ = S.shape
    packed = torch.empty(B * bytes_per_seq, dtype=torch.uint8, device=S.device) if packed is None else packed
    _sizes(S=(S, B * H * d * d), bits=(bits, H * d), head_off=(head_off, H), r=(r, B * H * d), c=(c, B * H * d),
           packed=(packed, B * int(bytes_per_seq)))
    _check_layout(bits, head_off, bytes_per_seq)
    call("stepq_pack_state", _dims(B, H, d), _ptr(S, torch.float32, "S"), _ptr(bits, torch.uint8, "bits"),
         _ptr(head_off, torch.int64, "head_off"), ctypes.c_int64(int(bytes_per_seq)),
         _ptr(r, torch.float16, "r"), _ptr(c, torch.float16, "c"), _ptr(packed, torch.uint8, "packed"), _stream())
    return packed


def stepq_unpack_state(packed, bits, head_off, bytes_per_seq, r, c, S_out=None):
    B, H, d = r.shape
    S_out = torch.empty((B, H, d, d), dtype=torch.float32, device=r.device) if S_out is None else S_out
    _sizes(packed=(packed, B * int(bytes_per_seq)), bits=(bits, H * d), head_off=(head_off, H), c=(c, B * H * d),
           S_out=(S_out, B * H * d * d))
    _check_layout(bits, head_off, bytes_per_seq)
    call("stepq_unpack_state", _dims(B, H, d), _ptr(packed, torch.uint8, "packed"), _ptr(bits, torch.uint8, "bits"),
         _ptr(head_off, torch.int64, "head_off"), ctypes.c_int64(int(bytes_per_seq)),
         _ptr(r, torch.float16, "r"), _ptr(c, torch.float16, "c"), _ptr(S_out, torch.float32, "S_out"), _stream())
    return S_out


def _step_sizes(B, H, d, gpc, k, v, beta, gate, bits, w, head_off, bytes_per_seq, packed_in, r_in, c_in,
                packed_out, r_out, c_out, o, C=1):
    """Element counts of a decode step's (C = 1) or a prefill chunk's buffers."""
    n = B * H * d
    return dict(k=(k, C * n), v=(v, C * n), beta=(beta, C * B * H), gate=(gate, C * B * H * (d if gpc else 1)),
                bits=(bits, H * d), w=(w, H * d), head_off=(head_off, H),
                packed_in=(packed_in, B * int(bytes_per_seq)), r_in=(r_in, n), c_in=(c_in, n),
                packed_out=(packed_out, B * int(bytes_per_seq)), r_out=(r_out, n), c_out=(c_out, n), o=(o, C * n))


def stepq_decode_step(q, k, v, beta, gate, bits, w, head_off, bytes_per_seq, packed_in, r_in, c_in,
                      packed_out=None, r_out=None, c_out=None, o=None, pivots=None, mixed=None, widths=None):
    """One fused quantized decode step; outputs may alias the inputs (in-place update).
    pivots / mixed / widths: the bit map's FP16 pivot rows / rows of different widths within a
    head / mask of the widths present (None: read from the bit map). Returns (packed_out, r_out,
    c_out, o)."""
    B, H, d = q.shape
    gpc = 1 if gate.dim() == 3 else 0
    packed_out = torch.empty_like(packed_in) if packed_out is None else packed_out
    r_out = torch.empty_like(r_in) if r_out is None else r_out
    c_out = torch.empty_like(c_in) if c_out is None else c_out
    o = torch.empty((B, H, d), dtype=torch.float32, device=q.device) if o is None else o
    _sizes(**_step_sizes(B, H, d, gpc, k, v, beta, gate, bits, w, head_off, bytes_per_seq, packed_in, r_in, c_in,
                         packed_out, r_out, c_out, o))
    _check_layout(bits, head_off, bytes_per_seq)
    mixed = _has_mixed(bits, mixed)
    call("stepq_decode_step", _dims(B, H, d, gpc, _has_pivots(bits, pivots), mixed, _widths(bits, widths, mixed)),
         _ptr(q, torch.bfloat16, "q"),
         _ptr(k, torch.bfloat16, "k"),
         _ptr(v, torch.bfloat16, "v"), _ptr(beta, torch.float32, "beta"), _ptr(gate, torch.float32, "gate"),
         _ptr(bits, torch.uint8, "bits"), _ptr(w, torch.float32, "w"), _ptr(head_off, torch.int64, "head_off"),
         ctypes.c_int64(int(bytes_per_seq)), _ptr(packed_in, torch.uint8, "packed_in"),
         _ptr(r_in, torch.float16, "r_in"), _ptr(c_in, torch.float16, "c_in"),
         _ptr(packed_out, torch.uint8, "packed_out"), _ptr(r_out, torch.float16, "r_out"),
         _ptr(c_out, torch.float16, "c_out"), _ptr(o, torch.float32, "o"), _stream())
    return packed_out, r_out, c_out, o


def stepq_decode_step_split(q, k, v, beta, gate, bits, w, head_off, bytes_per_seq, packed_in, r_in, c_in,
                            packed_out=None, r_out=None, c_out=None, o=None, x_ws=None, side_stream=None,
                            refit=True, pivots=None):
    """The split form: the first kernel (o, X) on the current stream, refit and pack on
    side_stream after it; the current stream then waits for the side stream unless the caller
    passes its own side_stream (and orders it). refit=False runs the first kernel only.
    Returns (packed_out, r_out, c_out, o, x_ws)."""
    B, H, d = q.shape
    gpc = 1 if gate.dim() == 3 else 0
    o = torch.empty((B, H, d), dtype=torch.float32, device=q.device) if o is None else o
    x_ws = torch.empty((B, H, d, d), dtype=torch.float32, device=q.device) if x_ws is None else x_ws
    if refit:
        packed_out = torch.empty_like(packed_in) if packed_out is None else packed_out
        r_out = torch.empty_like(r_in) if r_out is None else r_out
        c_out = torch.empty_like(c_in) if c_out is None else c_out
    own = side_stream is None and refit
    side = torch.cuda.Stream() if own else side_stream
    _sizes(x_ws=(x_ws, B * H * d * d),
           **_step_sizes(B, H, d, gpc, k, v, beta, gate, bits, w, head_off, bytes_per_seq, packed_in, r_in, c_in,
                         packed_out, r_out, c_out, o))
    _check_layout(bits, head_off, bytes_per_seq)
    opt = lambda t, dt, n: _ptr(t, dt, n) if t is not None else None
    call("stepq_decode_step_split", _dims(B, H, d, gpc, _has_pivots(bits, pivots)), _ptr(q, torch.bfloat16, "q"),
         _ptr(k, torch.bfloat16, "k"),
         _ptr(v, torch.bfloat16, "v"), _ptr(beta, torch.float32, "beta"), _ptr(gate, torch.float32, "gate"),
         _ptr(bits, torch.uint8, "bits"), _ptr(w, torch.float32, "w"), _ptr(head_off, torch.int64, "head_off"),
         ctypes.c_int64(int(bytes_per_seq)), _ptr(packed_in, torch.uint8, "packed_in"),
         _ptr(r_in, torch.float16, "r_in"), _ptr(c_in, torch.float16, "c_in"),
         opt(packed_out, torch.uint8, "packed_out"), opt(r_out, torch.float16, "r_out"),
         opt(c_out, torch.float16, "c_out"), _ptr(o, torch.float32, "o"), _ptr(x_ws, torch.float32, "x_ws"),
         _stream(), ctypes.c_void_p(side.cuda_stream if side is not None else 0))
    if own:
        torch.cuda.current_stream().wait_stream(side)
    return packed_out, r_out, c_out, o, x_ws


def stepq_prefill_chunk(q, k, v, beta, gate, bits, w, head_off, bytes_per_seq, packed_in, r_in, c_in,
                        packed_out=None, r_out=None, c_out=None, o=None, pivots=None, form=None, mixed=None):
    """A prefill chunk: q, k, v [C,B,H,d], beta [C,B,H], gate [C,B,H] or [C,B,H,d]; the state is
    reconstructed once, updated C times in fp32 and packed once. form: None (the library picks),
    "seq" (tokens one after another on the register tile) or "wy" (the chunked WY form on the
    tensor cores; d = 128, C <= 64). Returns (packed_out, r_out,
    c_out, o [C,B,H,d])."""
    C, B, H, d = q.shape
    gpc = 1 if gate.dim() == 4 else 0
    packed_out = torch.empty_like(packed_in) if packed_out is None else packed_out
    r_out = torch.empty_like(r_in) if r_out is None else r_out
    c_out = torch.empty_like(c_in) if c_out is None else c_out
    o = torch.empty((C, B, H, d), dtype=torch.float32, device=q.device) if o is None else o
    name = {None: "stepq_prefill_chunk", "seq": "stepq_prefill_chunk_seq", "wy": "stepq_prefill_chunk_wy"}[form]
    _sizes(**_step_sizes(B, H, d, gpc, k, v, beta, gate, bits, w, head_off, bytes_per_seq, packed_in, r_in, c_in,
                         packed_out, r_out, c_out, o, C=C))
    _check_layout(bits, head_off, bytes_per_seq)
    call(name, _dims(B, H, d, gpc, _has_pivots(bits, pivots), _has_mixed(bits, mixed)), ctypes.c_int(int(C)),
         _ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"), _ptr(v, torch.bfloat16, "v"),
         _ptr(beta, torch.float32, "beta"), _ptr(gate, torch.float32, "gate"), _ptr(bits, torch.uint8, "bits"),
         _ptr(w, torch.float32, "w"), _ptr(head_off, torch.int64, "head_off"), ctypes.c_int64(int(bytes_per_seq)),
         _ptr(packed_in, torch.uint8, "packed_in"), _ptr(r_in, torch.float16, "r_in"),
         _ptr(c_in, torch.float16, "c_in"), _ptr(packed_out, torch.uint8, "packed_out"),
         _ptr(r_out, torch.float16, "r_out"), _ptr(c_out, torch.float16, "c_out"), _ptr(o, torch.float32, "o"),
         _stream())
    return packed_out, r_out, c_out, o


def stepq_decode_step_fp32(q, k, v, beta, gate, S_in, S_out=None, o=None):
    B, H, d = q.shape
    gpc = 1 if gate.dim() == 3 else 0
    S_out = torch.empty_like(S_in) if S_out is None else S_out
    o = torch.empty((B, H, d), dtype=torch.float32, device=q.device) if o is None else o
    n = B * H * d
    _sizes(k=(k, n), v=(v, n), beta=(beta, B * H), gate=(gate, B * H * (d if gpc else 1)), S_in=(S_in, n * d),
           S_out=(S_out, n * d), o=(o, n))
    call("stepq_decode_step_fp32", _dims(B, H, d, gpc), _ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"),
         _ptr(v, torch.bfloat16, "v"), _ptr(beta, torch.float32, "beta"), _ptr(gate, torch.float32, "gate"),
         _ptr(S_in, torch.float32, "S_in"), _ptr(S_out, torch.float32, "S_out"), _ptr(o, torch.float32, "o"),
         _stream())
    return S_out, o


def stepq_int8_quantize_state(S, codes=None, s=None):
    B, H, d, _ = S.shape
    codes = torch.empty((B, H, d, d), dtype=torch.int8, device=S.device) if codes is None else codes
    s = torch.empty((B, H, d), dtype=torch.float16, device=S.device) if s is None else s
    _sizes(S=(S, B * H * d * d), codes=(codes, B * H * d * d), s=(s, B * H * d))
    call("stepq_int8_quantize_state", _dims(B, H, d), _ptr(S, torch.float32, "S"),
         _ptr(codes, torch.int8, "codes"), _ptr(s, torch.float16, "s"), _stream())
    return codes, s


def stepq_decode_step_int8(q, k, v, beta, gate, codes_in, s_in, codes_out=None, s_out=None, o=None):
    B, H, d = q.shape
    gpc = 1 if gate.dim() == 3 else 0
    codes_out = torch.empty_like(codes_in) if codes_out is None else codes_out
    s_out = torch.empty_like(s_in) if s_out is None else s_out
    o = torch.empty((B, H, d), dtype=torch.float32, device=q.device) if o is None else o
    n = B * H * d
    _sizes(k=(k, n), v=(v, n), beta=(beta, B * H), gate=(gate, B * H * (d if gpc else 1)),
           codes_in=(codes_in, n * d), s_in=(s_in, n), codes_out=(codes_out, n * d), s_out=(s_out, n), o=(o, n))
    call("stepq_decode_step_int8", _dims(B, H, d, gpc), _ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"),
         _ptr(v, torch.bfloat16, "v"), _ptr(beta, torch.float32, "beta"), _ptr(gate, torch.float32, "gate"),
         _ptr(codes_in, torch.int8, "codes_in"), _ptr(s_in, torch.float16, "s_in"),
         _ptr(codes_out, torch.int8, "codes_out"), _ptr(s_out, torch.float16, "s_out"), _ptr(o, torch.float32, "o"),
         _stream())
    return codes_out, s_out, o


def stepq_leap_step(window, t, q, k, v, beta, gate, codes, s, kbuf, ubuf, lbuf, o=None):
    """Token t of a window on the per-window 8-bit state: q, k, v [B,H,d], beta, gate [B,H];
    codes int8 [B,H,d,d] and s fp16 [B,H,d] (rewritten at the window's last token); buffers
    kbuf bf16 [window,B,H,d], ubuf fp32 [window,B,H,d], lbuf fp32 [window,B,H]. Returns o."""
    B, H, d = q.shape
    o = torch.empty((B, H, d), dtype=torch.float32, device=q.device) if o is None else o
    n, W = B * H * d, int(window)
    _sizes(k=(k, n), v=(v, n), beta=(beta, B * H), gate=(gate, B * H), codes=(codes, n * d), s=(s, n),
           kbuf=(kbuf, W * n), ubuf=(ubuf, W * n), lbuf=(lbuf, W * B * H), o=(o, n))
    call("stepq_leap_step", _dims(B, H, d, 0), ctypes.c_int(int(window)), ctypes.c_int(int(t)),
         _ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"), _ptr(v, torch.bfloat16, "v"),
         _ptr(beta, torch.float32, "beta"), _ptr(gate, torch.float32, "gate"), _ptr(codes, torch.int8, "codes"),
         _ptr(s, torch.float16, "s"), _ptr(kbuf, torch.bfloat16, "kbuf"), _ptr(ubuf, torch.float32, "ubuf"),
         _ptr(lbuf, torch.float32, "lbuf"), _ptr(o, torch.float32, "o"), _stream())
    return o


def stepq_row_impact(q, k, beta, gate, w_out=None):
    """Row impact w [H,d] from a calibration stream with a leading step axis: q, k [T,B,H,d]."""
    T, B, H, d = q.shape
    gpc = 1 if gate.dim() == 4 else 0
    w_out = torch.empty((H, d), dtype=torch.float32, device=q.device) if w_out is None else w_out
    _sizes(k=(k, T * B * H * d), beta=(beta, T * B * H), gate=(gate, T * B * H * (d if gpc else 1)),
           w_out=(w_out, H * d))
    call("stepq_row_impact", _dims(B, H, d, gpc), ctypes.c_int(T), _ptr(q, torch.bfloat16, "q"),
         _ptr(k, torch.bfloat16, "k"), _ptr(beta, torch.float32, "beta"), _ptr(gate, torch.float32, "gate"),
         _ptr(w_out, torch.float32, "w_out"), _stream())
    return w_out


def stepq_calib_distortion(S, w, b, d_row=None, d_head=None, scratch=None):
    """(d_row float64 [H,d], d_head float64 [H]) at the uniform width b over the states S."""
    B, H, d, _ = S.shape
    dev = S.device
    d_row = torch.empty((H, d), dtype=torch.float64, device=dev) if d_row is None else d_row
    d_head = torch.empty((H,), dtype=torch.float64, device=dev) if d_head is None else d_head
    scratch = torch.empty((B, H, d), dtype=torch.float64, device=dev) if scratch is None else scratch
    _sizes(S=(S, B * H * d * d), w=(w, H * d), d_row=(d_row, H * d), d_head=(d_head, H), scratch=(scratch, B * H * d))
    call("stepq_calib_distortion", _dims(B, H, d), _ptr(S, torch.float32, "S"), _ptr(w, torch.float32, "w"),
         ctypes.c_int(int(b)), _ptr(d_row, torch.float64, "d_row"), _ptr(d_head, torch.float64, "d_head"),
         _ptr(scratch, torch.float64, "scratch"), _stream())
    return d_row, d_head


def stepq_calib_distortion_bits(S, w, bits, d_row=None, d_head=None, scratch=None):
    """(d_row float64 [H,d], d_head float64 [H]) under the per-row bit map bits (uint8 [H,d],
    16 = FP16 pivot row) over the states S."""
    B, H, d, _ = S.shape
    dev = S.device
    d_row = torch.empty((H, d), dtype=torch.float64, device=dev) if d_row is None else d_row
    d_head = torch.empty((H,), dtype=torch.float64, device=dev) if d_head is None else d_head
    scratch = torch.empty((B, H, d), dtype=torch.float64, device=dev) if scratch is None else scratch
    _sizes(S=(S, B * H * d * d), w=(w, H * d), bits=(bits, H * d), d_row=(d_row, H * d), d_head=(d_head, H),
           scratch=(scratch, B * H * d))
    call("stepq_calib_distortion_bits", _dims(B, H, d), _ptr(S, torch.float32, "S"), _ptr(w, torch.float32, "w"),
         _ptr(bits, torch.uint8, "bits"), _ptr(d_row, torch.float64, "d_row"), _ptr(d_head, torch.float64, "d_head"),
         _ptr(scratch, torch.float64, "scratch"), _stream())
    return d_row, d_head


def stepq_calib_distortion_static(S, w, b, d_row=None, d_head=None):
    """stepq_calib_distortion on the library's static device work space (B*H*d at most
    STEPQ_STATIC_SCRATCH_ROWS; overlapping calls on one device race)."""
    B, H, d, _ = S.shape
    dev = S.device
    d_row = torch.empty((H, d), dtype=torch.float64, device=dev) if d_row is None else d_row
    d_head = torch.empty((H,), dtype=torch.float64, device=dev) if d_head is None else d_head
    _sizes(S=(S, B * H * d * d), w=(w, H * d), d_row=(d_row, H * d), d_head=(d_head, H))
    call("stepq_calib_distortion_static", _dims(B, H, d), _ptr(S, torch.float32, "S"), _ptr(w, torch.float32, "w"),
         ctypes.c_int(int(b)), _ptr(d_row, torch.float64, "d_row"), _ptr(d_head, torch.float64, "d_head"), _stream())
    return d_row, d_head


def stepq_allocate_bits(J, cand, budget_bits: int, mode: int):
    """Host bit allocation: uint8 numpy [n_units] with exactly budget_bits bits in total."""
    J = np.ascontiguousarray(np.asarray(J, dtype=np.float64))
    cand = np.ascontiguousarray(np.asarray(cand, dtype=np.int32))
    n, nc = J.shape
    out = np.zeros(n, dtype=np.uint8)
    call("stepq_allocate_bits", ctypes.c_int(n), ctypes.c_int(nc), cand.ctypes.data_as(ctypes.c_void_p),
         J.ctypes.data_as(ctypes.c_void_p), ctypes.c_int64(int(budget_bits)), ctypes.c_int(int(mode)),
         out.ctypes.data_as(ctypes.c_void_p))
    return out


def stepq_read_device_flags() -> int:
    flags = ctypes.c_uint32(0)
    call("stepq_read_device_flags", ctypes.byref(flags))
    return flags.value


def stepq_selftest_wait(limit_ns: int) -> None:
    """One bounded wait that nothing completes, on the current stream: after limit_ns it gives
    up and raises bit 0 of the device error word (read it with stepq_read_device_flags)."""
    call("stepq_selftest_wait", ctypes.c_uint64(int(limit_ns)), _stream())
