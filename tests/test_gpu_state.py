"""GPU parity of the state conversion kernels against the oracle: pack and unpack bit for bit,
the dual-axis fit within one binary16 ulp, calibration statistics, and the empty batch."""
import numpy as np
import pytest

import oracle
from recurrent_state_quantization_gated_b200 import synth
from tests.helpers import dev, half_ulps, host_half, with_pivots

pytestmark = pytest.mark.gpu


def _api():
    from recurrent_state_quantization_gated_b200 import api
    return api


# (d, B, H, widths, FP16 pivot rows added): width 16 in `widths` makes whole pivot heads too
CASES = [(64, 2, 3, (2, 4, 6, 8), 0), (128, 3, 5, (2, 4, 6, 8), 0), (128, 2, 4, (6,), 0), (64, 5, 1, (8,), 0),
         (128, 1, 37, (4, 8), 0), (64, 2, 3, (2, 4, 6, 8), 7), (128, 3, 5, (4, 6, 8), 11), (128, 2, 3, (16,), 0),
         (64, 3, 2, (4, 16), 0)]


def _bits(H, d, widths, npiv, seed):
    return with_pivots(synth.random_bits(H, d, choices=widths, seed=seed), npiv, seed + 100)


@pytest.mark.parametrize("d,B,H,widths,npiv", CASES)
def test_pack_unpack_bit_exact(d, B, H, widths, npiv):
    import torch
    api = _api()
    S = synth.random_tile_state(B, H, d, seed=d + B + H)
    bits = _bits(H, d, widths, npiv, seed=H)
    w = synth.random_weights(H, d, seed=B)
    r, c = oracle.fit_scales(S, w, bits)                    # scales from the oracle: inputs only
    packed_ref = oracle.pack_state(S, bits, r, c)
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    packed = api.stepq_pack_state(dev(S), dev(bits), dev(head_off), bps, dev(r, torch.float16), dev(c, torch.float16))
    np.testing.assert_array_equal(packed.cpu().numpy(), packed_ref)
    S_hat = api.stepq_unpack_state(dev(packed_ref), dev(bits), dev(head_off), bps, dev(r, torch.float16),
                                   dev(c, torch.float16))
    np.testing.assert_array_equal(S_hat.cpu().numpy().view(np.uint32),
                                  oracle.unpack_state(packed_ref, bits, r, c).view(np.uint32))


@pytest.mark.parametrize("d,B,H,widths,npiv", CASES)
def test_fit_scales_within_one_ulp(d, B, H, widths, npiv):
    api = _api()
    S = synth.random_tile_state(B, H, d, seed=2 * d + B)
    bits = _bits(H, d, widths, npiv, seed=H + 1)
    w = synth.random_weights(H, d, seed=B + 1)
    r_ref, c_ref = oracle.fit_scales(S, w, bits)
    r, c = api.stepq_fit_scales(dev(S), dev(w), dev(bits))
    r, c = host_half(r), host_half(c)
    assert half_ulps(r, r_ref).max() <= 1 and half_ulps(c, c_ref).max() <= 1
    assert (r != r_ref).mean() < 1e-3 and (c != c_ref).mean() < 1e-3


def test_fit_of_zero_and_constant_tiles():
    api = _api()
    d, H = 128, 2
    S = np.zeros((2, H, d, d), dtype=np.float32)
    S[1, 1] = 0.25
    bits = synth.random_bits(H, d, seed=4)
    w = np.ones((H, d), dtype=np.float32)
    r_ref, c_ref = oracle.fit_scales(S, w, bits)
    r, c = api.stepq_fit_scales(dev(S), dev(w), dev(bits))
    np.testing.assert_array_equal(host_half(r), r_ref)
    np.testing.assert_array_equal(host_half(c), c_ref)
    assert (r_ref[0] == np.float16(2.0 ** -14).view(np.uint16)).all()


def test_empty_batch_is_a_no_op():
    import torch
    api = _api()
    d, H = 64, 2
    bits = synth.random_bits(H, d, seed=1)
    head_off, bps, total = api.stepq_packed_layout(bits, d, B=0)
    assert total == 0
    S = torch.zeros((0, H, d, d), device="cuda")
    r, c = api.stepq_fit_scales(S, dev(np.ones((H, d), np.float32)), dev(bits))
    assert r.numel() == 0 and c.numel() == 0
    torch.cuda.synchronize()


def test_row_impact_matches_oracle():
    import torch
    api = _api()
    for idx, over in ((2, dict(B=6, H=3)), (1, dict(B=5, H=4)), (0, {})):
        wl = synth.workload(idx, **over)
        cal = synth.calib_tokens(wl)
        w_ref = oracle.row_impact(cal)
        w = api.stepq_row_impact(dev(cal["q"], torch.bfloat16), dev(cal["k"], torch.bfloat16), dev(cal["beta"]),
                                 dev(cal["gate"]))
        np.testing.assert_allclose(w.cpu().numpy(), w_ref, rtol=1e-6)


@pytest.mark.parametrize("d", [64, 128])
def test_calib_distortion_matches_oracle(d):
    api = _api()
    S = synth.random_tile_state(3, 4, d, seed=40 + d)
    w = synth.random_weights(4, d, seed=41)
    for b in (2, 4, 6, 8):
        dr_ref, dh_ref = oracle.calib_distortion(S, w, b)
        dr, dh = api.stepq_calib_distortion(dev(S), dev(w), b)
        np.testing.assert_allclose(dr.cpu().numpy(), dr_ref, rtol=1e-9, atol=0)
        np.testing.assert_allclose(dh.cpu().numpy(), dh_ref, rtol=1e-9, atol=0)


@pytest.mark.parametrize("d", [64, 128])
def test_calib_distortion_under_a_bit_map_with_pivots(d):
    api = _api()
    S = synth.random_tile_state(3, 4, d, seed=50 + d)
    w = synth.random_weights(4, d, seed=51)
    bits = _bits(4, d, (4, 6, 8), 9, seed=52)
    dr_ref, dh_ref = oracle.calib_distortion_bits(S, w, bits)
    dr, dh = api.stepq_calib_distortion_bits(dev(S), dev(w), dev(bits))
    np.testing.assert_allclose(dr.cpu().numpy(), dr_ref, rtol=1e-9, atol=0)
    np.testing.assert_allclose(dh.cpu().numpy(), dh_ref, rtol=1e-9, atol=0)
    dr16, _ = api.stepq_calib_distortion(dev(S), dev(w), 16)
    np.testing.assert_allclose(dr16.cpu().numpy(), oracle.calib_distortion(S, w, 16)[0], rtol=1e-9, atol=0)


def test_calibration_allocation_matches_oracle():
    """The whole offline calibration of two synthetic workloads gives the oracle's bit maps."""
    import torch
    from recurrent_state_quantization_gated_b200 import runtime
    for idx, over in ((1, dict(B=4, H=6)), (2, dict(B=4, H=3))):
        wl = synth.workload(idx, **over)
        S0 = synth.initial_state(wl)
        cal = synth.calib_tokens(wl)
        bits_ref, w_ref = oracle.calibrate(wl.alloc, wl.candidates, wl.nominal_bits, S0, cal,
                                           n_pivots=wl.n_pivots)
        cal_dev = dict(q=dev(cal["q"], torch.bfloat16), k=dev(cal["k"], torch.bfloat16), beta=dev(cal["beta"]),
                       gate=dev(cal["gate"]))
        bits, w = runtime.calibrate(wl.alloc, wl.candidates, wl.nominal_bits, dev(S0), cal_dev,
                                    n_pivots=wl.n_pivots)
        np.testing.assert_allclose(w.cpu().numpy(), w_ref, rtol=1e-6)
        np.testing.assert_array_equal(bits, bits_ref)
        assert int((bits == 16).sum()) == wl.n_pivots * (1 if wl.alloc == "lagrange_row" else wl.d)
        assert bits.astype(np.int64).sum() == wl.nominal_bits * bits.size + 8 * int((bits == 16).sum())
