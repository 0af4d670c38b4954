"""The allocation-free distortion entry point, whose work space is a static device array,
against the allocating stepq_calib_distortion (and the oracle) through the C ABI. Collected
last so that it also runs after every other GPU test in the same process."""
import ctypes

import numpy as np
import pytest

import oracle
from recurrent_state_quantization_gated_b200 import synth
from tests.helpers import dev

pytestmark = pytest.mark.gpu


def test_static_work_space_matches_allocating_entry_point():
    """Two calls in a row, with different states and shapes, so the second overwrites what the
    first left in the shared array: each equals the allocating entry point within the
    distortion parity tolerance (1e-9 relative), and the oracle likewise."""
    import torch
    from recurrent_state_quantization_gated_b200 import api
    cases = [(3, 4, 128, 6, 70), (5, 3, 64, 4, 71)]
    for B, H, d, b, seed in cases:
        S = synth.random_tile_state(B, H, d, seed=seed)
        w = synth.random_weights(H, d, seed=seed + 1)
        dr_a, dh_a = api.stepq_calib_distortion(dev(S), dev(w), b)
        dr_s, dh_s = api.stepq_calib_distortion_static(dev(S), dev(w), b)
        torch.cuda.synchronize()
        np.testing.assert_allclose(dr_s.cpu().numpy(), dr_a.cpu().numpy(), rtol=1e-9, atol=0)
        np.testing.assert_allclose(dh_s.cpu().numpy(), dh_a.cpu().numpy(), rtol=1e-9, atol=0)
        dr_ref, dh_ref = oracle.calib_distortion(S, w, b)
        np.testing.assert_allclose(dr_s.cpu().numpy(), dr_ref, rtol=1e-9, atol=0)
        np.testing.assert_allclose(dh_s.cpu().numpy(), dh_ref, rtol=1e-9, atol=0)


def test_static_work_space_size_limit():
    """B*H*dk beyond STEPQ_STATIC_SCRATCH_ROWS is refused with STEPQ_EINVAL before any launch;
    the largest accepted size still runs."""
    import torch
    from recurrent_state_quantization_gated_b200 import _lib, api
    limit = 524288
    d, H = 128, 8
    B_max = limit // (H * d)
    w = torch.ones((H, d), device="cuda")
    d_row = torch.empty((H, d), dtype=torch.float64, device="cuda")
    d_head = torch.empty((H,), dtype=torch.float64, device="cuda")
    S = torch.zeros((B_max + 1, H, d, d), device="cuda")
    dims = _lib.Dims(B_max + 1, H, d, d, 0)
    rc = _lib.lib().stepq_calib_distortion_static(dims, ctypes.c_void_p(S.data_ptr()), ctypes.c_void_p(w.data_ptr()),
                                                  ctypes.c_int(4), ctypes.c_void_p(d_row.data_ptr()),
                                                  ctypes.c_void_p(d_head.data_ptr()), None)
    assert rc == 1                      # STEPQ_EINVAL
    assert b"static work space" in _lib.lib().stepq_last_error()
    with pytest.raises(_lib.StepqError):
        api.stepq_calib_distortion_static(S, w, 4)
    dr, dh = api.stepq_calib_distortion_static(S[:B_max], w, 4)
    torch.cuda.synchronize()
    assert (dr == 0).all() and (dh == 0).all()      # a zero state is represented exactly
