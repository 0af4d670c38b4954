"""GPU parity of the per-window 8-bit state (LeapQuant's per-window quantisation as read from its
abstract: rowwise-absmax INT8 between windows, exact updates inside a window, the state
quantised once at the window's end) against the oracle: every token's readout within 1e-3
(max-normalised per tile; in practice about 1e-6), the window's end state with scales within one
binary16 ulp and codes within one step on at most 0.1 % of entries where the scales agree."""
import numpy as np
import pytest

import oracle
from recurrent_state_quantization_gated_b200 import synth
from tests.helpers import dev, half_ulps, host_half

pytestmark = pytest.mark.gpu


def _window(wl, W, t0=0):
    steps = [synth.tokens(wl, t0 + t) for t in range(W)]
    return {name: np.ascontiguousarray(np.stack([s[name] for s in steps])) for name in steps[0]}


def _run_gpu(wl, toks, codes, s, W):
    import torch
    from recurrent_state_quantization_gated_b200 import runtime
    st = runtime.WindowState(dev(codes, torch.int8), dev(s, torch.float16), W)
    outs = []
    for t in range(W):
        td = runtime.to_device_tokens({n: a[t] for n, a in toks.items()})
        outs.append(st.step(**td).cpu().numpy())
    torch.cuda.synchronize()
    return st, np.stack(outs)


def _compare(st, o_g, ref):
    c_r, s_r, o_r = ref
    err = np.abs(o_g - o_r).max(axis=-1) / np.maximum(np.abs(o_r).max(axis=-1), 1e-30)
    assert err.max() <= 1e-3, err.max()
    c_g, s_g = st.codes.cpu().numpy(), host_half(st.s)
    assert half_ulps(s_g, s_r).max() <= 1
    same = (s_g == s_r)[..., None] & np.ones_like(c_g, dtype=bool)
    d = np.abs(c_g.astype(np.int32) - c_r.astype(np.int32))
    assert d.max() <= 1
    assert (d[same] > 0).mean() <= 1e-3
    return err.max()


@pytest.mark.parametrize("d,B,H,W", [(64, 2, 3, 5), (128, 3, 4, 16), (128, 2, 2, 1), (128, 4, 8, 64)])
def test_window_matches_oracle(d, B, H, W):
    wl = synth.workload(1, B=B, H=H, d=d, seed=W + H)
    codes, s = oracle.int8_quantise_state(synth.initial_state(wl))
    toks = _window(wl, W)
    st, o_g = _run_gpu(wl, toks, codes, s, W)
    assert _compare(st, o_g, oracle.leap_window(toks, codes, s)) <= 1e-4
    from recurrent_state_quantization_gated_b200 import api
    assert api.stepq_read_device_flags() == 0


def test_consecutive_windows_and_a_zero_gate():
    """Two 12-token windows back to back (the second starts from the GPU's requantised state),
    with one exact zero gate and gates down to 0.3 in the second window."""
    wl = synth.workload(1, B=2, H=4, d=128, seed=9)
    codes, s = oracle.int8_quantise_state(synth.initial_state(wl))
    toks1, toks2 = _window(wl, 12), _window(wl, 12, t0=12)
    rng = np.random.default_rng(3)
    toks2["gate"] = rng.uniform(0.3, 1.0, toks2["gate"].shape).astype(np.float32)
    toks2["gate"][4, 1, 2] = 0.0
    st, o1 = _run_gpu(wl, toks1, codes, s, 12)
    _compare(st, o1, oracle.leap_window(toks1, codes, s))
    c1, s1 = st.codes.cpu().numpy(), host_half(st.s)
    st2, o2 = _run_gpu(wl, toks2, c1, s1, 12)
    _compare(st2, o2, oracle.leap_window(toks2, c1, s1))


def test_full_size_window_sampled():
    """The GDN-shaped batch (64 sequences x 32 heads, d = 128), a 16-token window in 16 launches;
    the oracle checks four sampled sequences (every head of each)."""
    wl = synth.workload(1)
    W = 16
    codes, s = oracle.int8_quantise_state(synth.initial_state(wl))
    toks = _window(wl, W)
    st, o_g = _run_gpu(wl, toks, codes, s, W)
    seqs = [0, 20, 41, wl.B - 1]
    sub = {n: np.ascontiguousarray(a[:, seqs]) for n, a in toks.items()}
    c_r, s_r, o_r = oracle.leap_window(sub, codes[seqs], s[seqs])

    class _Sub:
        pass
    view = _Sub()
    view.codes, view.s = st.codes[seqs], st.s[seqs]
    _compare(view, o_g[:, seqs], (c_r, s_r, o_r))
