"""Pins of the oracle's key-row-aware dual-axis fit (STEPQuant §4.3, App. C.1): the row
factor definition, the no-clip column initialisation, the least-squares optimality of the
fixed-code column update, and the decode step as the composition the workflow table lists."""
import numpy as np
import pytest

import oracle
from recurrent_state_quantization_gated_b200 import synth


def _tile(d=128, seed=0):
    S = synth.random_tile_state(1, 1, d, seed=seed)[0, 0]
    bits = synth.random_bits(1, d, seed=seed + 1)[0]
    w = synth.random_weights(1, d, seed=seed + 2)[0]
    return S, bits, w


@pytest.mark.parametrize("d", [64, 128])
def test_row_factor_is_mean_abs_over_impact(d):
    S, bits, w = _tile(d, 3)
    r, _ = oracle.fit_tile(S, w, bits)
    m = np.abs(S.astype(np.float64)).mean(axis=1)
    expect = np.clip(np.maximum(m, 2.0 ** -14) / w.astype(np.float64), 2.0 ** -14, 65504).astype(np.float16)
    np.testing.assert_array_equal(r, expect.view(np.uint16))


def test_zero_row_factor_is_the_floor_over_its_impact():
    """R1 floors the row mean at 2^-14 before dividing by the impact factor: an all-zero row with
    w_i = 1/2 gets r_i = 2^-13, and one with w_i = 2 gets 2^-15, clamped back up to 2^-14."""
    S, bits, w = _tile(64, 4)
    S[3] = 0.0
    S[4] = 0.0
    w[3], w[4] = 0.5, 2.0
    r, _ = oracle.fit_tile(S, w, bits)
    assert r[3] == np.float16(2.0 ** -13).view(np.uint16)
    assert r[4] == np.float16(2.0 ** -14).view(np.uint16)


def test_column_init_clips_nothing_and_is_tight():
    S, bits, w = _tile(128, 5)
    r, c, det = oracle.fit_tile(S, w, bits, detail=True)
    rf = oracle.half_to_float(r).astype(np.float64)
    bound = rf * 2.0 ** (8 - bits.astype(np.float64)) * (2.0 ** (bits.astype(np.float64) - 1) - 1)
    ratio = np.abs(S) / (bound[:, None] * det["c0"][None, :].astype(np.float64))
    assert ratio.max() <= 1 + 1e-6
    np.testing.assert_allclose(ratio.max(axis=0), 1.0, rtol=1e-6)   # some entry of each column reaches the edge
    qb = (2 ** (bits.astype(np.int64) - 1) - 1)
    assert np.all(np.abs(det["z0"]) <= qb[:, None])


@pytest.mark.parametrize("seed", [5, 6, 7])
def test_column_update_is_the_weighted_least_squares_optimum(seed):
    """For the fixed codes z0 the weighted objective sum_i w_i^2 (X_ij - r_i c_j z_ij)^2 has zero
    derivative in c_j at c1, and c1 does no worse than the initial scale c0."""
    S, bits, w = _tile(128, seed)
    r, c, det = oracle.fit_tile(S, w, bits, detail=True)
    rf = oracle.half_to_float(r).astype(np.float64)
    V = rf[:, None] * (2.0 ** (8 - bits.astype(np.float64)))[:, None] * det["z0"]
    W2 = (w.astype(np.float64) ** 2)[:, None]
    X = S.astype(np.float64)

    def objective(cvec):
        return np.sum(W2 * (X - V * cvec[None, :]) ** 2, axis=0)

    c1 = det["c1"]
    grad = -2 * np.sum(W2 * V * (X - V * c1[None, :]), axis=0)
    scale = 2 * np.sum(W2 * np.abs(V * X), axis=0) + 1e-300
    assert np.max(np.abs(grad) / scale) < 1e-12
    assert np.all(objective(c1) <= objective(det["c0"].astype(np.float64)) * (1 + 1e-12))
    for eps in (1e-3, -1e-3):                        # a local minimum along each column
        assert np.all(objective(c1 * (1 + eps)) >= objective(c1))
    np.testing.assert_array_equal(c, np.clip(c1, 2.0 ** -14, 65504).astype(np.float16).view(np.uint16))


def test_zero_column_keeps_initial_scale():
    S, bits, w = _tile(64, 9)
    S[:, 5] = 0.0
    r, c, det = oracle.fit_tile(S, w, bits, detail=True)
    assert det["c0"][5] == np.float32(2.0 ** -14)
    assert det["c1"][5] == det["c0"][5]
    assert c[5] == np.float16(2.0 ** -14).view(np.uint16)


def _representable_tile(d, seed):
    """A tile X_ij = r_i 2^(8-b_i) c_j z_ij exactly, with binary16 scales r, c, integer codes
    |z_ij| <= q_b and the code q_b in every column (so the no-clip start is c itself)."""
    rng = np.random.default_rng(seed)
    bits = rng.choice(np.array([2, 4, 6, 8], dtype=np.uint8), d)
    qb = 2 ** (bits.astype(np.int64) - 1) - 1
    z = np.stack([rng.integers(-q, q + 1, d) for q in qb])
    rows = rng.integers(0, d, d)                             # one entry per column at its row's edge
    z[rows, np.arange(d)] = qb[rows] * rng.choice([-1, 1], d)
    r = (2.0 ** rng.integers(-6, 2, d)).astype(np.float16)
    c = (2.0 ** rng.integers(-8, -2, d) * rng.choice([1.0, 1.25, 1.5, 1.75], d)).astype(np.float16)
    X = (r.astype(np.float64)[:, None] * 2.0 ** (8 - bits.astype(np.float64))[:, None]
         * c.astype(np.float64)[None, :] * z).astype(np.float32)
    return X, bits, r.view(np.uint16), c.view(np.uint16), z


@pytest.mark.parametrize("seed", [11, 12])
def test_column_fit_at_given_row_scales_is_exact_on_representable_tiles(seed):
    """At the row scales the tile was built with, the no-clip start is the column scale itself,
    the codes at (r, c0) are the tile's codes, and the least-squares update returns the same
    scale (App. C.1: the fit is exact where the state is exactly representable); at row scales
    twice as large every column scale halves."""
    d = 64
    X, bits, r, c, z = _representable_tile(d, seed)
    w = synth.random_weights(1, d, seed=seed)[0]
    got, det = oracle.fit_columns(X, w, bits, r, detail=True)
    np.testing.assert_array_equal(det["z0"], z)
    np.testing.assert_array_equal(got, c)
    r2 = (r.view(np.float16).astype(np.float64) * 2).astype(np.float16).view(np.uint16)
    half = (c.view(np.float16).astype(np.float64) / 2).astype(np.float16).view(np.uint16)
    np.testing.assert_array_equal(oracle.fit_columns(X, w, bits, r2), half)


def test_least_squares_update_alone():
    """The fixed-code least-squares update (App. C.1) on its own: the codes a representable tile
    was built from give its column scales back; the weights' common scale cancels; an all-zero
    column of codes keeps its fallback scale; at the tile fit's own codes it is the fit's c."""
    d = 64
    X, bits, r, c, z = _representable_tile(d, 14)
    w = synth.random_weights(1, d, seed=14)[0]
    fall = np.full(d, 0.5, dtype=np.float32)
    got, c1 = oracle.ls_columns(X, w, bits, r, z, fall)
    np.testing.assert_array_equal(got, c)
    np.testing.assert_array_equal(oracle.ls_columns(X, 4.0 * w, bits, r, z, fall)[0], c)
    z0 = z.copy()
    z0[:, 3] = 0
    got0, c10 = oracle.ls_columns(X, w, bits, r, z0, fall)
    assert c10[3] == 0.5 and got0[3] == np.float16(0.5).view(np.uint16)
    S, bits2, w2 = _tile(128, 15)
    r2, c2, det = oracle.fit_tile(S, w2, bits2, detail=True)
    np.testing.assert_array_equal(oracle.ls_columns(S, w2, bits2, r2, det["z0"], det["c0"])[0], c2)


def test_column_fit_is_the_column_half_of_the_tile_fit():
    S, bits, w = _tile(128, 13)
    r, c = oracle.fit_tile(S, w, bits)
    np.testing.assert_array_equal(oracle.fit_columns(S, w, bits, r), c)


@pytest.mark.parametrize("gpc", [False, True])
def test_decode_tile_is_unpack_update_fit_pack(gpc):
    """Table C2: reconstruct, update, emit the readout before requantisation, refit, repack."""
    d = 64
    wl = synth.workload(0)
    S = synth.random_tile_state(1, 1, d, seed=12)
    bits = synth.half_bits(wl)[:1]
    w = synth.random_weights(1, d, seed=13)
    r, c = oracle.fit_scales(S, w, bits)
    packed = oracle.pack_state(S, bits, r, c)
    tok = synth.tokens(wl, 0, seqs=[0])
    tok = {k: v[:, :1] for k, v in tok.items()}
    if gpc:
        tok["gate"] = np.ascontiguousarray(np.linspace(0.9, 1.0, d, dtype=np.float32)[None, None, :])
    p1, r1, c1, o = oracle.decode_step(tok, bits, w, packed, r, c)
    Shat = oracle.unpack_state(packed, bits, r, c)[0, 0].astype(np.float64)
    qf = synth.bf16_bits_to_f32(tok["q"][0, 0]); kf = synth.bf16_bits_to_f32(tok["k"][0, 0])
    vf = synth.bf16_bits_to_f32(tok["v"][0, 0])
    g = tok["gate"][0, 0]
    X, o_ref = oracle.delta_update(Shat, qf, kf, vf, float(tok["beta"][0, 0]), g)
    np.testing.assert_allclose(o[0, 0], o_ref.astype(np.float32), rtol=0, atol=0)
    X32 = X.astype(np.float32)
    rr, cc = oracle.fit_tile(X32, w[0], bits[0])
    np.testing.assert_array_equal(r1[0, 0], rr)
    np.testing.assert_array_equal(c1[0, 0], cc)
    np.testing.assert_array_equal(p1, oracle.pack_tile(X32, bits[0], rr, cc))
