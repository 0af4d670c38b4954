"""Pins of the oracle's packed layout and quantiser contract: exhaustive code round trips,
bytes built independently with word arithmetic, the printed state sizes of STEPQuant (App. D,
App. F), the half-step error bound of §2.2 and the reduction of the 8-bit setting to plain
INT8 quantisation."""
import os

import numpy as np
import pytest

import oracle
from recurrent_state_quantization_gated_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_sizes():
    vals = {}
    for line in open(os.path.join(GOLDEN, "state_sizes.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, value = line.split()[:2]
        vals[name] = float(value)
    return vals


def _qmax(b):
    return 2 ** (int(b) - 1) - 1


@pytest.mark.parametrize("b", [2, 4, 6, 8])
@pytest.mark.parametrize("dv", [64, 128])
def test_every_code_round_trips(b, dv):
    qb = _qmax(b)
    allq = np.arange(-qb, qb + 1)
    dk = 8
    codes = np.resize(allq, dk * dv).reshape(dk, dv)
    codes = np.roll(codes, 3, axis=1)
    bits = np.full(dk, b, dtype=np.uint8)
    packed = oracle.pack_codes(codes, bits)
    assert packed.size == dk * dv * b // 8
    np.testing.assert_array_equal(oracle.unpack_codes(packed, bits, dv), codes)


def _expected_row_bytes(q, b):
    """Independent construction from 32-bit little-endian words: a 2- or 8-bit row holds field
    j at bit (j*b) mod 32 of word floor(j*b/32); a 4-bit row holds columns 4g..4g+3 in the
    16-bit halfword g in nibble order 0, 2, 1, 3; a 6-bit row = 4-bit low plane + 2-bit high
    plane."""
    q = np.asarray(q, dtype=np.int64)
    if b == 6:
        u = q & 63
        return np.concatenate([_expected_row_bytes(u & 15, 4), _expected_row_bytes(u >> 4, 2)])
    if b == 4:
        halves = []
        for g in range(0, len(q), 4):
            c = [int(x) & 15 for x in q[g:g + 4]]
            halves.append(c[0] | (c[2] << 4) | (c[1] << 8) | (c[3] << 12))
        return np.array(halves, dtype="<u2").view(np.uint8)
    per_word = 32 // b
    words = []
    for w0 in range(0, len(q), per_word):
        word = 0
        for f, val in enumerate(q[w0:w0 + per_word]):
            word |= (int(val) & ((1 << b) - 1)) << (f * b)
        words.append(word)
    return np.array(words, dtype="<u4").view(np.uint8)


def test_bytes_match_word_construction_mixed_rows():
    rng = np.random.default_rng(0)
    dv = 64
    bits = np.array([2, 4, 6, 8, 8, 6, 4, 2], dtype=np.uint8)
    codes = np.stack([rng.integers(-_qmax(b), _qmax(b) + 1, size=dv) for b in bits])
    packed = oracle.pack_codes(codes, bits)
    expected = np.concatenate([_expected_row_bytes(codes[i], int(b)) for i, b in enumerate(bits)])
    np.testing.assert_array_equal(packed, expected)


def test_hand_written_row():
    """A 4-bit row of codes 1, -1, 7, -7, 0, ...: nibbles 0x1, 0xF, 0x7, 0x9 stored in the
    order of columns 0, 2, 1, 3 -> halfword 0x9F71 -> bytes 71 9F."""
    codes = np.zeros((1, 64), dtype=np.int32)
    codes[0, :4] = [1, -1, 7, -7]
    packed = oracle.pack_codes(codes, np.array([4], dtype=np.uint8))
    assert packed[0] == 0x71 and packed[1] == 0x9F and not packed[2:].any()
    codes6 = np.zeros((1, 64), dtype=np.int32)
    codes6[0, :2] = [-31, 17]   # 6-bit two's complement 0b100001, 0b010001
    p6 = oracle.pack_codes(codes6, np.array([6], dtype=np.uint8))
    assert p6[0] == 0x01 and p6[1] == 0x01   # low nibbles 1 (col 0, bits 0-3) and 1 (col 1, bits 8-11)
    assert p6[32] == 0x06         # high crumbs 0b10 (bits 0-1), 0b01 (bits 2-3)


def test_layout_offsets_and_alignment():
    bits = synth.random_bits(5, 128, seed=3)
    head_off, bps = oracle.layout(bits, 128)
    sizes = [16 * int(bits[h].astype(np.int64).sum()) for h in range(5)]
    np.testing.assert_array_equal(head_off, np.concatenate([[0], np.cumsum(sizes)[:-1]]))
    assert bps == sum(sizes)
    assert all(o % 16 == 0 for o in head_off) and bps % 16 == 0


def test_printed_state_sizes():
    g = _golden_sizes()
    d = int(g["head_dim"])
    heads = int(g["qwen_layers"] * g["qwen_heads_per_layer"])
    elems = heads * d * d
    assert elems * 4 == g["qwen_fp32_bytes_per_request"]
    bits6 = np.full((heads, d), 6, dtype=np.uint8)
    _, code_bytes = oracle.layout(bits6, d)
    scale_bytes = heads * (d + d) * 2                      # fp16 r and c per head
    pivots = int(g["qwen_pivot_heads"])
    pivot_surcharge = pivots * d * d * (16 - 8) // 8       # FP16 pivot counted as (16 - 8) extra bits
    total = code_bytes + scale_bytes + pivot_surcharge
    assert total == g["qwen6_bytes_with_pivot_scales"]
    assert total - pivots * (d + d) * 2 == g["qwen6_bytes_per_request"]
    assert round(total * 8 / elems, 3) == g["qwen6_bits_per_value"]
    assert round(g["qwen_fp32_bytes_per_request"] / g["qwen6_bytes_per_request"], 2) == g["qwen6_compression"]
    assert 16 * (d + d) / (d * d) == g["scale_bits_per_element"]
    kda_rows = int(g["kda_layers"] * g["kda_heads_per_layer"] * d)
    for nominal, key in ((6, "kda6_bits_per_value"), (4, "kda4_bits_per_value")):
        per_value = nominal + 16 / d + 16 / d + g["kda_pivot_rows"] / kda_rows * (16 - 8)
        assert round(per_value, 3) == g[key]


def _fit_pack_unpack(S, w, bits):
    r, c = oracle.fit_tile(S, w, bits)
    packed = oracle.pack_tile(S, bits, r, c)
    Xh = oracle.unpack_tile(packed, bits, r, c, S.shape[1])
    codes = oracle.unpack_codes(packed, bits, S.shape[1])
    return r, c, codes, Xh


@pytest.mark.parametrize("d", [64, 128])
def test_half_step_error_bound_and_clipping(d):
    """|x - x_hat| <= step/2 for every entry inside the codebook range, and a clipped entry
    lands on the end point: error |x| - q_b step (§2.2)."""
    S = synth.random_tile_state(2, 2, d, seed=8)
    bits_map = synth.random_bits(2, d, seed=9)
    w = synth.random_weights(2, d, seed=10)
    n_clipped = 0
    for bidx in range(2):
        for h in range(2):
            X = S[bidx, h]
            bits = bits_map[h]
            r, c, codes, Xh = _fit_pack_unpack(X, w[h], bits)
            rf = oracle.half_to_float(r).astype(np.float64)
            cf = oracle.half_to_float(c).astype(np.float64)
            norm = 2.0 ** (8 - bits.astype(np.float64))
            qb = (2.0 ** (bits.astype(np.float64) - 1) - 1)
            step = rf[:, None] * cf[None, :] * norm[:, None]
            assert np.all(np.abs(codes) <= qb[:, None])
            err = np.abs(X.astype(np.float64) - Xh.astype(np.float64))
            inside = np.abs(X) <= (qb[:, None] + 0.5) * step * (1 - 1e-6)
            assert np.all(err[inside] <= 0.5 * step[inside] * (1 + 2.0 ** -20) + 1e-30)
            clipped = np.abs(codes) == qb[:, None]
            out = clipped & ~inside
            n_clipped += out.sum()
            np.testing.assert_allclose(err[out], np.abs(X[out]) - qb[:, None].repeat(d, 1)[out] * step[out],
                                       rtol=1e-5)
    assert n_clipped > 0          # the clipped branch is exercised


def test_uniform_8bit_is_plain_int8_with_rank1_scales():
    """At 8 bits, x_hat = clip(rint(x / s), -127, 127) s with the rank-1 scale s = r (x) c
    (textbook symmetric INT8); the oracle's contract multiplies by reciprocals, so codes may
    differ from the division form only where x/s sits on a rounding tie."""
    S = synth.random_tile_state(1, 1, 128, seed=21)[0, 0]
    bits = np.full(128, 8, dtype=np.uint8)
    w = np.ones(128, dtype=np.float32)
    r, c, codes, Xh = _fit_pack_unpack(S, w, bits)
    s = oracle.half_to_float(r).astype(np.float64)[:, None] * oracle.half_to_float(c).astype(np.float64)[None, :]
    textbook = np.clip(np.rint(S.astype(np.float64) / s), -127, 127)
    diff = np.abs(textbook - codes)
    assert diff.max() <= 1 and (diff > 0).mean() < 1e-4
    np.testing.assert_allclose(Xh, (codes * s), rtol=2 ** -22)


def test_rowwise_absmax_int8_is_the_8bit_contract_with_unit_columns():
    """c = 1 and r_i = absmax_i / 127 turn the 8-bit STEPQuant contract into the rowwise-absmax
    INT8 baseline (§5.1) bit for bit; and that baseline equals the textbook quantiser."""
    S = synth.random_tile_state(1, 1, 64, seed=22)[0, 0]
    codes8, s8 = oracle.int8_quantise_tile(S)
    bits = np.full(64, 8, dtype=np.uint8)
    ones = np.full(64, 0x3C00, dtype=np.uint16)           # binary16 1.0
    codes = oracle.quantise_tile(S, bits, s8, ones)
    np.testing.assert_array_equal(codes, codes8.astype(np.int32))
    scale = oracle.half_to_float(s8).astype(np.float64)
    np.testing.assert_allclose(scale, [oracle.half_to_float(np.float16(m / 127.0).view(np.uint16))
                                       for m in np.abs(S).max(axis=1).astype(np.float64)], rtol=0)
    textbook = np.clip(np.rint(S / scale[:, None]), -127, 127)
    assert np.abs(textbook - codes8).max() <= 1 and (textbook != codes8).mean() < 1e-3


@pytest.mark.parametrize("b", [2, 4, 6, 8])
def test_quantiser_rounds_exact_half_steps_to_even(b):
    """With unit steps (r = 2^-(8-b), so that r 2^(8-b) = 1, and c = 1) the quantiser reduces to
    clip(rint(x), -q_b, q_b) with NumPy's rint (nearest, ties to even, R3), exact half steps
    included, and clips beyond the end points."""
    qb = _qmax(b)
    vals = np.concatenate([np.arange(-qb, qb) + 0.5, [0.25, -0.75, qb + 0.5, -qb - 3.0]])
    X = np.resize(vals, 2 * 64).reshape(2, 64).astype(np.float32)
    bits = np.full(2, b, dtype=np.uint8)
    r = np.full(2, np.float16(2.0 ** -(8 - b)).view(np.uint16), dtype=np.uint16)
    c = np.full(64, np.float16(1.0).view(np.uint16), dtype=np.uint16)
    codes = oracle.quantise_tile(X, bits, r, c)
    np.testing.assert_array_equal(codes, np.clip(np.rint(X.astype(np.float64)), -qb, qb))


def test_int8_baseline_rounds_exact_half_steps_to_even():
    """Rows whose absolute maximum is 127 get the scale s = 1 exactly, so the rowwise-absmax INT8
    baseline reduces to clip(rint(x), -127, 127): exact half steps go to the even neighbour."""
    vals = np.arange(-126, 126) + 0.5
    X = np.resize(vals, 4 * 64).reshape(4, 64).astype(np.float32)
    X[:, 0] = 127.0
    codes, s = oracle.int8_quantise_tile(X)
    assert (s == np.float16(1.0).view(np.uint16)).all()
    np.testing.assert_array_equal(codes, np.clip(np.rint(X.astype(np.float64)), -127, 127))


def test_scale_rounding_matches_numpy_binary16():
    rng = np.random.default_rng(2)
    xs = np.concatenate([np.exp(rng.uniform(np.log(2.0 ** -14), np.log(65504.0), 20000)),
                         [2.0 ** -14, 1.0, 65504.0, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11]])
    mine = np.array([oracle.scale_to_half(x) for x in xs], dtype=np.uint16)
    ref = xs.astype(np.float16).view(np.uint16)
    np.testing.assert_array_equal(mine, ref)
    assert oracle.scale_to_half(0.0) == np.float16(2.0 ** -14).view(np.uint16)
    assert oracle.scale_to_half(1e9) == np.float16(65504.0).view(np.uint16)
