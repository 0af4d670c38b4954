"""Host logic of runtime.Layout, on the CPU: the per-head byte offsets and bytes per sequence of
a bit map equal the oracle's layout (rows of (d/8) b_i bytes, heads in order), and the two flags
that select the decode step's kernel instantiation are read correctly from the map: `pivots`
(some row has width 16), `mixed` (some head's rows have different widths) and `widths` (the mask
of the widths present, bit b for width b)."""
import numpy as np
import pytest

import oracle
from recurrent_state_quantization_gated_b200 import runtime, synth
from tests.helpers import with_pivots


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("kind", ["uniform", "per_head", "mixed", "mixed_pivots", "head_pivot"])
def test_layout_and_flags(d, kind):
    H = 5
    if kind == "uniform":
        bits = np.full((H, d), 6, np.uint8)
    elif kind == "per_head":
        bits = np.repeat(np.array([2, 4, 6, 8, 4], np.uint8)[:, None], d, axis=1)
    elif kind == "mixed":
        bits = synth.random_bits(H, d, choices=(2, 4, 6, 8), seed=3)
    elif kind == "mixed_pivots":
        bits = with_pivots(synth.random_bits(H, d, choices=(4, 6, 8), seed=4), 5, 6)
    else:
        bits = np.repeat(np.array([4, 16, 6, 8, 6], np.uint8)[:, None], d, axis=1)
    L = runtime.Layout.build(bits, d, device="cpu")
    head_off, bps = oracle.layout(bits, d)
    np.testing.assert_array_equal(L.head_off, head_off)
    assert L.bytes_per_seq == bps == int(bits.astype(np.int64).sum()) * d // 8
    assert L.H == H and L.d == d
    assert L.pivots == int(kind in ("mixed_pivots", "head_pivot"))
    assert L.mixed == int(kind in ("mixed", "mixed_pivots"))
    assert L.widths == sum(1 << int(b) for b in np.unique(bits))
    np.testing.assert_array_equal(L.bits_dev.numpy(), bits)
    np.testing.assert_array_equal(L.head_off_dev.numpy(), head_off)
