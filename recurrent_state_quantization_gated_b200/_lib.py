"""ctypes loader for libstepq.so (the C ABI declared in include/stepq.h).

There is no fallback: if the CUDA library is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

LIB_PATH = Path(__file__).resolve().with_name("libstepq.so")

STEPQ_OK, STEPQ_EINVAL, STEPQ_EUNSUPPORTED, STEPQ_EALIGN, STEPQ_EBUDGET, STEPQ_ECUDA = range(6)
_NAMES = {0: "OK", 1: "EINVAL", 2: "EUNSUPPORTED", 3: "EALIGN", 4: "EBUDGET", 5: "ECUDA"}

# Every entry point of include/stepq.h.
SYMBOLS = (
    "stepq_last_error", "stepq_packed_layout", "stepq_fit_scales", "stepq_pack_state",
    "stepq_unpack_state", "stepq_decode_step", "stepq_decode_step_split", "stepq_prefill_chunk",
    "stepq_prefill_chunk_seq", "stepq_prefill_chunk_wy",
    "stepq_decode_step_fp32",
    "stepq_int8_quantize_state", "stepq_decode_step_int8", "stepq_leap_step", "stepq_row_impact",
    "stepq_calib_distortion", "stepq_calib_distortion_bits", "stepq_calib_distortion_static", "stepq_allocate_bits", "stepq_read_device_flags", "stepq_selftest_wait",
    "stepq_build_info",
)


class StepqError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed: STEPQ_{_NAMES.get(code, code)}: {msg}")
        self.code = code


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("dk", ctypes.c_int), ("dv", ctypes.c_int),
                ("gate_per_channel", ctypes.c_int), ("pivots", ctypes.c_int), ("mixed", ctypes.c_int),
                ("widths", ctypes.c_int)]


_lib = None

P = ctypes.c_void_p
I = ctypes.c_int
I64 = ctypes.c_int64

_SIGNATURES = {
    "stepq_last_error": ([], ctypes.c_char_p),
    "stepq_build_info": ([], ctypes.c_char_p),
    "stepq_packed_layout": ([Dims, P, P, P, P], I),
    "stepq_fit_scales": ([Dims, P, P, P, P, P, P], I),
    "stepq_pack_state": ([Dims, P, P, P, I64, P, P, P, P], I),
    "stepq_unpack_state": ([Dims, P, P, P, I64, P, P, P, P], I),
    "stepq_decode_step": ([Dims, P, P, P, P, P, P, P, P, I64, P, P, P, P, P, P, P, P], I),
    "stepq_decode_step_split": ([Dims, P, P, P, P, P, P, P, P, I64, P, P, P, P, P, P, P, P, P, P], I),
    "stepq_prefill_chunk": ([Dims, I, P, P, P, P, P, P, P, P, I64, P, P, P, P, P, P, P, P], I),
    "stepq_prefill_chunk_seq": ([Dims, I, P, P, P, P, P, P, P, P, I64, P, P, P, P, P, P, P, P], I),
    "stepq_prefill_chunk_wy": ([Dims, I, P, P, P, P, P, P, P, P, I64, P, P, P, P, P, P, P, P], I),
    "stepq_decode_step_fp32": ([Dims, P, P, P, P, P, P, P, P, P], I),
    "stepq_int8_quantize_state": ([Dims, P, P, P, P], I),
    "stepq_decode_step_int8": ([Dims, P, P, P, P, P, P, P, P, P, P, P], I),
    "stepq_leap_step": ([Dims, I, I, P, P, P, P, P, P, P, P, P, P, P, P], I),
    "stepq_row_impact": ([Dims, I, P, P, P, P, P, P], I),
    "stepq_calib_distortion": ([Dims, P, P, I, P, P, P, P], I),
    "stepq_calib_distortion_static": ([Dims, P, P, I, P, P, P], I),
    "stepq_calib_distortion_bits": ([Dims, P, P, P, P, P, P, P], I),
    "stepq_allocate_bits": ([I, I, P, P, I64, I, P], I),
    "stepq_read_device_flags": ([P], I),
    "stepq_selftest_wait": ([ctypes.c_uint64, P], I),
}


def lib() -> ctypes.CDLL:
    """The loaded CUDA library. Raises if it has not been built (no CPU fallback exists)."""
    global _lib
    if _lib is None:
        if not LIB_PATH.exists():
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m recurrent_state_quantization_gated_b200.build`")
        handle = ctypes.CDLL(str(LIB_PATH))
        for name, (args, res) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.argtypes = args
            fn.restype = res
        _lib = handle
    return _lib


def call(name: str, *args) -> None:
    rc = getattr(lib(), name)(*args)
    if rc != STEPQ_OK:
        raise StepqError(name, rc, lib().stepq_last_error().decode())
