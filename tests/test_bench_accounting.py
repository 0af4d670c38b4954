"""Host-side accounting of the benchmark and the runtime, without a GPU: the algorithmic bytes
each kernel must move (the roofline numerator), the bit-map properties that select kernel
instantiations, and the per-window state's token counter."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402
from recurrent_state_quantization_gated_b200 import runtime, synth  # noqa: E402


def test_decode_bytes_per_tile_match_the_state_format():
    """6-bit rows at d = 128: codes read + write 2 x 12,288, scales 2 x 512, q/k/v 768, beta and
    a scalar gate 8, o 512 = 26,888 B per tile (27,396 with channel gates)."""
    d, H, B = 128, 32, 64
    bits = np.full((H, d), 6, np.uint8)
    _, bps = oracle.layout(bits, d)
    assert bench.algorithmic_bytes(bps, B, H, d, False, "quant") == B * H * 26888
    assert bench.algorithmic_bytes(bps, B, H, d, True, "quant") == B * H * 27396
    # the 4-bit map: 18,696 B per tile
    _, bps4 = oracle.layout(np.full((H, d), 4, np.uint8), d)
    assert bench.algorithmic_bytes(bps4, B, H, d, False, "quant") == B * H * 18696


def test_prefill_and_window_bytes():
    d, H, B, C = 128, 2, 3, 64
    _, bps = oracle.layout(np.full((H, d), 6, np.uint8), d)
    small = 3 * 2 * d + 4 + 4 + 4 * d
    # a chunk moves the state once and every token's inputs and readout
    assert bench.algorithmic_bytes(bps, B, H, d, False, f"prefill:{C}") == \
        2 * B * bps + B * H * 2 * (2 * d + 2 * d) + C * B * H * small
    # a window token: INT8 tile and scales read, one buffered entry written, t entries read on
    # average (W - 1) / 2, and the window end's write and full buffer read spread over W tokens
    W = 16
    entry = 2 * d + 4 * d + 4
    per_tile = (d * d + 2 * d) + entry + (W - 1) / 2 * entry + (d * d + 2 * d + W * entry) / W
    assert bench.algorithmic_bytes(bps, B, H, d, False, f"leap:{W}") == int(B * H * per_tile) + B * H * small
    # a one-token window is the per-step INT8 step plus the (unused) buffer entry
    assert bench.algorithmic_bytes(bps, B, H, d, False, "leap:1") == \
        int(B * H * (2 * (d * d + 2 * d) + 2 * entry)) + B * H * small


def test_layout_flags_follow_the_bit_map():
    d, H = 64, 4
    heads_uniform = np.repeat(np.array([[4], [6], [8], [2]], np.uint8), d, axis=1)
    L = runtime.Layout.build(heads_uniform, d, device="cpu")
    assert L.mixed == 0 and L.pivots == 0
    mixed = heads_uniform.copy()
    mixed[2, 5] = 4
    assert runtime.Layout.build(mixed, d, device="cpu").mixed == 1
    piv = heads_uniform.copy()
    piv[1, :] = 16                                   # a pivot head: one width, pivots present
    Lp = runtime.Layout.build(piv, d, device="cpu")
    assert Lp.pivots == 1 and Lp.mixed == 0


def test_window_state_counts_tokens_modulo_the_window(monkeypatch):
    import torch
    from recurrent_state_quantization_gated_b200 import api
    seen = []
    monkeypatch.setattr(api, "stepq_leap_step", lambda window, t, *a, **k: seen.append((window, t)))
    codes = torch.zeros((2, 3, 64, 64), dtype=torch.int8)
    s = torch.zeros((2, 3, 64), dtype=torch.float16)
    st = runtime.WindowState(codes, s, 4)
    assert st.kbuf.shape == (4, 2, 3, 64) and st.ubuf.shape == (4, 2, 3, 64) and st.lbuf.shape == (4, 2, 3)
    for _ in range(9):
        st.step(None, None, None, None, None)
    assert seen == [(4, t % 4) for t in range(9)]
    assert st.t == 1
