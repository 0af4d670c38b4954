"""Pins of the oracle's FP16 pivot rows (STEPQuant App. C.2; Table C2 steps 1 and 6): width
16 keeps a key row's values in binary16, stored after the integer rows of the tile, outside the
shared column fit; pivot selection and the (16 - 8) budget accounting of App. D."""
import numpy as np
import pytest

import oracle
from recurrent_state_quantization_gated_b200 import synth


def _f16(x):
    return np.asarray(x, dtype=np.float32).astype(np.float16)


def test_float_to_half_is_ieee_round_to_nearest_even_with_saturation():
    rng = np.random.default_rng(1)
    xs = np.concatenate([
        rng.normal(0, 1, 2000), rng.normal(0, 1e-5, 500),          # normals and subnormals
        rng.uniform(-65000, 65000, 500),
        [0.0, -0.0, 6.1035156e-05, 5.9604645e-08, 2.9802322e-08, 65504.0, -65504.0],
        1.0 + np.array([1, 3, 5]) * 2.0 ** -11,                   # exact ties between neighbours
    ]).astype(np.float32)
    got = np.array([oracle.float_to_half(x) for x in xs], dtype=np.uint16)
    np.testing.assert_array_equal(got, _f16(xs).view(np.uint16))
    for x in (65520.0, 1e6, -7e4, np.float32(3e38)):
        assert oracle.float_to_half(x) == (0x7BFF if x > 0 else 0xFBFF)


def _tile(d=64, seed=0, pivots=(0, 5, 17)):
    rng = np.random.default_rng(seed)
    X = (rng.normal(0, 0.1, (d, d)) * np.exp(rng.normal(0, 1, (d, 1)))).astype(np.float32)
    bits = rng.choice(np.array([2, 4, 6, 8], np.uint8), d)
    bits[list(pivots)] = 16
    w = np.exp(rng.normal(0, 0.3, d)).astype(np.float32)
    return X, bits, w


@pytest.mark.parametrize("spike", [False, True])
def test_fit_ignores_pivot_rows(spike):
    """The column scales of a tile with pivot rows are those of the tile without them; the row
    factors of the other rows are unchanged; a pivot row's factor is the usual R1 value. With
    `spike`, a pivot row holds one entry 50 times its row's largest (the kind of outlier a pivot
    keeps); were that row in the shared column fit, it would set its column's scale."""
    X, bits, w = _tile()
    if spike:
        X[0, 7] = 50.0 * np.abs(X[0]).max()
    keep = bits != 16
    r, c = oracle.fit_tile(X, w, bits)
    r2, c2 = oracle.fit_tile(np.ascontiguousarray(X[keep]), np.ascontiguousarray(w[keep]), bits[keep])
    np.testing.assert_array_equal(c, c2)
    np.testing.assert_array_equal(r[keep], r2)
    b8 = bits.copy()
    b8[~keep] = 8
    r8, _ = oracle.fit_tile(X, w, b8)
    np.testing.assert_array_equal(r[~keep], r8[~keep])


def test_pivot_rows_round_trip_and_sit_after_the_integer_rows():
    X, bits, w = _tile(seed=2)
    d = X.shape[1]
    r, c = oracle.fit_tile(X, w, bits)
    packed = oracle.pack_tile(X, bits, r, c)
    assert packed.size == oracle.tile_bytes(bits, d) == sum(d * int(b) // 8 for b in bits)
    Xh = oracle.unpack_tile(packed, bits, r, c, d)
    piv = np.flatnonzero(bits == 16)
    np.testing.assert_array_equal(Xh[piv], _f16(X[piv]).astype(np.float32))
    # the pivot rows' binary16 values fill the end of the tile, in key order
    tail = packed[-2 * d * piv.size:].view(np.uint16).reshape(piv.size, d)
    np.testing.assert_array_equal(tail, _f16(X[piv]).view(np.uint16))
    # integer rows reconstruct as in a tile without the pivots
    keep = bits != 16
    p2 = oracle.pack_tile(np.ascontiguousarray(X[keep]), bits[keep], r[keep], c)
    np.testing.assert_array_equal(packed[:p2.size], p2)


def test_distortion_at_width_16_is_the_binary16_rounding_error():
    S = synth.random_tile_state(3, 2, 64, seed=4)
    w = synth.random_weights(2, 64, seed=5)
    d_row, d_head = oracle.calib_distortion(S, w, 16)
    e = (_f16(S).astype(np.float64) - S.astype(np.float64)) ** 2
    np.testing.assert_allclose(d_row, e.mean(axis=(0, 3)), rtol=1e-12, atol=0)
    np.testing.assert_allclose(d_head, (w.astype(np.float64)[None, :, :, None] ** 2 * e).mean(axis=(0, 2, 3)),
                               rtol=1e-12, atol=0)


def test_decode_stores_pivot_rows_as_binary16_of_the_update():
    d, H = 64, 2
    wl = synth.workload(2, B=1, H=H, d=d)
    S0 = synth.initial_state(wl)
    rng = np.random.default_rng(7)
    bits = rng.choice(np.array([4, 6, 8], np.uint8), (H, d))
    bits[0, [3, 40]] = 16
    bits[1, 9] = 16
    w = synth.random_weights(H, d, seed=8)
    r, c = oracle.fit_scales(S0, w, bits)
    packed = oracle.pack_state(S0, bits, r, c)
    tok = synth.tokens(wl, 0)
    p1, r1, c1, o = oracle.decode_step(tok, bits, w, packed, r, c)
    S_hat = oracle.unpack_state(packed, bits, r, c)
    S1 = oracle.unpack_state(p1, bits, r1, c1)
    for h in range(H):
        X, o_ref = oracle.delta_update(S_hat[0, h], synth.bf16_bits_to_f32(tok["q"][0, h]),
                                       synth.bf16_bits_to_f32(tok["k"][0, h]), synth.bf16_bits_to_f32(tok["v"][0, h]),
                                       float(tok["beta"][0, h]), tok["gate"][0, h])
        np.testing.assert_allclose(o[0, h], o_ref, rtol=1e-6, atol=1e-7)
        piv = bits[h] == 16
        np.testing.assert_array_equal(S1[0, h][piv], _f16(X.astype(np.float32)[piv]).astype(np.float32))


def test_row_pivots_take_the_largest_lifetime_weighted_gain_and_the_budget_adds_8_bits_each():
    wl = synth.workload(2, B=3, H=2, d=64)
    S0 = synth.initial_state(wl)
    cal = synth.calib_tokens(wl)
    P = 5
    bits, w = oracle.calibrate(wl.alloc, wl.candidates, wl.nominal_bits, S0, cal, n_pivots=P)
    piv = np.flatnonzero(bits.reshape(-1) == 16)
    assert piv.size == P
    assert bits.astype(np.int64).sum() == wl.nominal_bits * bits.size + 8 * P
    assert set(np.unique(bits[bits != 16])) <= set(wl.candidates)
    d16, _ = oracle.calib_distortion(S0, w, 16)
    dnom, _ = oracle.calib_distortion(S0, w, wl.nominal_bits)
    gain = oracle.lifetime(np.log(synth.unit_gates(wl).astype(np.float64))).reshape(-1) * (dnom - d16).reshape(-1)
    assert gain[piv].min() >= np.delete(gain, piv).max()


def test_head_pivots_take_the_largest_residual_risk():
    wl = synth.workload(1, B=3, H=6, d=64)
    S0 = synth.initial_state(wl)
    cal = synth.calib_tokens(wl)
    b0, w = oracle.calibrate(wl.alloc, wl.candidates, wl.nominal_bits, S0, cal)
    b1, _ = oracle.calibrate(wl.alloc, wl.candidates, wl.nominal_bits, S0, cal, n_pivots=1)
    heads0, heads1 = b0[:, 0], b1[:, 0]
    assert (b1 == b1[:, :1]).all() and (heads1 == 16).sum() == 1
    assert heads1.astype(np.int64).sum() == wl.nominal_bits * wl.H + 8
    risk = []
    for h, b in enumerate(heads0):
        _, dh = oracle.calib_distortion(S0, w, int(b))
        risk.append(oracle.lifetime(np.log(synth.unit_gates(wl).astype(np.float64)))[h] * dh[h])
    assert heads1[int(np.argmax(risk))] == 16
