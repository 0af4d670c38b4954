"""The C-ABI library without a GPU: it loads, exports every entry point include/stepq.h
declares, its host-only calls (packed layout, bit allocation) agree bit for bit with the
oracle, and argument errors are reported before anything touches CUDA."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from recurrent_state_quantization_gated_b200 import _lib, api, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "stepq.h")).read()
    return sorted(set(re.findall(r"STEPQ_API\s+[\w\s\*]*?\b(stepq_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    declared = _declared()
    assert len(declared) >= 14
    lib = _lib.lib()
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(_lib.SYMBOLS) == declared


def test_build_info():
    assert "sm_100a" in api.stepq_build_info()


@pytest.mark.parametrize("d", [64, 128])
def test_layout_matches_oracle(d):
    bits = synth.random_bits(7, d, seed=5)
    head_off, bps, total = api.stepq_packed_layout(bits, d, B=3)
    ho, obps = oracle.layout(bits, d)
    np.testing.assert_array_equal(head_off, ho)
    assert bps == obps and total == 3 * obps


@pytest.mark.parametrize("mode,cand,mean", [(1, [4, 6, 8], 6), (1, [2, 4, 6, 8], 4), (0, [4, 6, 8], 6),
                                            (0, [2, 4, 8], 4), (0, [2, 4, 6, 8], 4), (0, [4, 6, 8], 5)])
def test_allocation_is_bit_exact_with_oracle(mode, cand, mean):
    rng = np.random.default_rng(mode * 10 + mean)
    for n in (2, 9, 64, 500 if mode == 0 else 40):
        L = rng.exponential(size=(n, 1)) * 30
        d = np.sort(rng.exponential(size=(n, len(cand))) * 4.0 ** -np.array(cand), axis=1)[:, ::-1]
        J = L * d
        budget = n * mean
        if budget % 2:
            continue
        np.testing.assert_array_equal(api.stepq_allocate_bits(J, cand, budget, mode),
                                      oracle.allocate_bits(J, cand, budget, mode))


def test_allocation_ties_and_repair_match_oracle():
    rng = np.random.default_rng(77)
    cand = [4, 6, 8]
    for trial in range(30):
        n = int(rng.integers(2, 30))
        J = rng.integers(0, 5, size=(n, 3)).astype(np.float64)    # many exact ties
        if trial % 3 == 0:
            J[:, 1] = J[:, 0] + 0.5                                 # middle width off the hull
        for mode in (0, 1):
            for budget in (4 * n + 2, 6 * n, 8 * n - 2):
                try:
                    want = oracle.allocate_bits(J, cand, budget, mode)
                except ValueError:
                    with pytest.raises(_lib.StepqError):
                        api.stepq_allocate_bits(J, cand, budget, mode)
                    continue
                np.testing.assert_array_equal(api.stepq_allocate_bits(J, cand, budget, mode), want)


def test_allocation_rejects_infeasible_and_bad_arguments():
    with pytest.raises(_lib.StepqError) as e:
        api.stepq_allocate_bits(np.ones((3, 3)), [4, 6, 8], 13, 1)
    assert e.value.code == _lib.STEPQ_EBUDGET
    with pytest.raises(_lib.StepqError) as e:
        api.stepq_allocate_bits(np.ones((3, 3)), [6, 4, 8], 18, 0)
    assert e.value.code == _lib.STEPQ_EINVAL
    with pytest.raises(_lib.StepqError):
        api.stepq_allocate_bits(np.full((2, 3), np.nan), [4, 6, 8], 12, 0)


def _dims(B=2, H=2, d=128, gpc=0, pivots=0):
    return _lib.Dims(B, H, d, d, gpc, pivots)


def _fake(addr=0x10000):
    return ctypes.c_void_p(addr)


def test_device_calls_validate_before_touching_cuda():
    lib = _lib.lib()
    P = _fake
    # unsupported head width
    rc = lib.stepq_fit_scales(_dims(d=96), P(), P(), P(), P(), P(), None)
    assert rc == _lib.STEPQ_EUNSUPPORTED
    # null pointer
    rc = lib.stepq_fit_scales(_dims(), P(), ctypes.c_void_p(0), P(), P(), P(), None)
    assert rc == _lib.STEPQ_EINVAL and b"w is NULL" in lib.stepq_last_error()
    # misaligned pointer
    rc = lib.stepq_unpack_state(_dims(), P(0x10008), P(), P(), 4096, P(), P(), P(), None)
    assert rc == _lib.STEPQ_EALIGN
    # bad bytes_per_seq
    rc = lib.stepq_decode_step(_dims(), *([P()] * 8), 4097, *([P()] * 7), None)
    assert rc == _lib.STEPQ_EINVAL
    # bad gate flag
    rc = lib.stepq_decode_step_fp32(_dims(gpc=3), *([P()] * 8), None)
    assert rc == _lib.STEPQ_EINVAL
    # width outside {2,4,6,8}
    rc = lib.stepq_calib_distortion(_dims(), P(), P(), 5, P(), P(), P(), None)
    assert rc == _lib.STEPQ_EUNSUPPORTED
    # empty batch is a no-op that never launches
    assert lib.stepq_decode_step(_dims(B=0), *([P()] * 8), 4096, *([P()] * 7), None) == _lib.STEPQ_OK
    # a widths mask with a bit other than 2, 4, 6, 8, 16
    d = _dims()
    d.mixed, d.widths = 1, (1 << 4) | (1 << 5)
    rc = lib.stepq_decode_step(d, *([P()] * 8), 4096, *([P()] * 7), None)
    assert rc == _lib.STEPQ_EINVAL and b"widths" in lib.stepq_last_error()
    # unsupported width in a layout
    bits = np.full((1, 64), 3, dtype=np.uint8)
    with pytest.raises(_lib.StepqError) as e:
        api.stepq_packed_layout(bits, 64)
    assert e.value.code == _lib.STEPQ_EUNSUPPORTED


def test_new_entry_points_validate_before_touching_cuda():
    lib = _lib.lib()
    P = _fake
    # prefill: chunk must be positive; an empty batch is a no-op
    rc = lib.stepq_prefill_chunk(_dims(), 0, *([P()] * 8), 4096, *([P()] * 7), None)
    assert rc == _lib.STEPQ_EINVAL and b"chunk" in lib.stepq_last_error()
    assert lib.stepq_prefill_chunk(_dims(B=0), 4, *([P()] * 8), 4096, *([P()] * 7), None) == _lib.STEPQ_OK
    rc = lib.stepq_prefill_chunk(_dims(), 4, *([P()] * 8), 4097, *([P()] * 7), None)
    assert rc == _lib.STEPQ_EINVAL
    # split form: the work space is required
    rc = lib.stepq_decode_step_split(_dims(), *([P()] * 8), 4096, *([P()] * 7), ctypes.c_void_p(0), None, None)
    assert rc == _lib.STEPQ_EINVAL and b"x_ws is NULL" in lib.stepq_last_error()
    # distortion under a bit map: pointers checked; width 16 accepted by the uniform form
    rc = lib.stepq_calib_distortion_bits(_dims(), P(), P(), ctypes.c_void_p(0), P(), P(), P(), None)
    assert rc == _lib.STEPQ_EINVAL and b"bits is NULL" in lib.stepq_last_error()
    rc = lib.stepq_calib_distortion(_dims(), P(), P(), 12, P(), P(), P(), None)
    assert rc == _lib.STEPQ_EUNSUPPORTED
    # the static work space refuses sizes beyond its capacity before any CUDA call
    rc = lib.stepq_calib_distortion_static(_dims(B=8193, H=1, d=64), P(), P(), 4, P(), P(), None)
    assert rc == _lib.STEPQ_EINVAL and b"static work space" in lib.stepq_last_error()
    # FP16 pivot rows are a valid width in a layout
    bits = np.full((2, 64), 6, dtype=np.uint8)
    bits[1, :3] = 16
    head_off, bps, _ = api.stepq_packed_layout(bits, 64)
    assert bps == oracle.layout(bits, 64)[1] == 64 * 6 // 8 * 125 + 64 * 2 * 3


def test_tensor_core_prefill_refuses_shapes_it_does_not_cover():
    """stepq_prefill_chunk_wy: d = 128 and 1 <= chunk <= 64 (scalar or channel gates, FP16 pivot
    rows or not); anything else is STEPQ_EUNSUPPORTED (the sequential form covers it), checked
    before any CUDA call."""
    lib = _lib.lib()
    P = _fake
    args = (*([P()] * 8), 4096, *([P()] * 7), None)
    for dims, chunk in ((_dims(d=64), 8), (_dims(d=64, gpc=1, pivots=1), 8), (_dims(), 65)):
        rc = lib.stepq_prefill_chunk_wy(dims, chunk, *args)
        assert rc == _lib.STEPQ_EUNSUPPORTED and b"tensor-core chunk form" in lib.stepq_last_error()
    assert lib.stepq_prefill_chunk_wy(_dims(), 0, *args) == _lib.STEPQ_EINVAL
    assert lib.stepq_prefill_chunk_wy(_dims(B=0), 64, *args) == _lib.STEPQ_OK
    rc = lib.stepq_prefill_chunk_wy(_dims(), 64, *([P()] * 8), 4097, *([P()] * 7), None)
    assert rc == _lib.STEPQ_EINVAL


def test_per_window_step_validates_before_touching_cuda():
    """stepq_leap_step: scalar gates only; 0 <= t < window <= 256; pointers checked; an empty
    batch is a no-op."""
    lib = _lib.lib()
    P = _fake
    args = (*([P()] * 5), P(), P(), P(), P(), P(), P(), None)
    rc = lib.stepq_leap_step(_dims(gpc=1), 16, 0, *args)
    assert rc == _lib.STEPQ_EUNSUPPORTED and b"channel gates" in lib.stepq_last_error()
    for window, t in ((0, 0), (257, 0), (16, 16), (16, -1)):
        assert lib.stepq_leap_step(_dims(), window, t, *args) == _lib.STEPQ_EINVAL
    assert lib.stepq_leap_step(_dims(B=0), 16, 3, *args) == _lib.STEPQ_OK
    rc = lib.stepq_leap_step(_dims(), 16, 3, *([P()] * 5), P(), P(), ctypes.c_void_p(0), P(), P(), P(), None)
    assert rc == _lib.STEPQ_EINVAL and b"kbuf is NULL" in lib.stepq_last_error()


def test_wait_selftest_validates_its_limit_before_touching_cuda():
    lib = _lib.lib()
    for bad in (0, 999, 10**9 + 1):
        assert lib.stepq_selftest_wait(ctypes.c_uint64(bad), None) == _lib.STEPQ_EINVAL
    assert b"limit_ns" in lib.stepq_last_error()
