"""Pins of the oracle's per-window 8-bit state (LeapQuant's abstract on the page "When Dynamic
Scaling Fails: A Scale-State Feedback Governs Recurrent-State Quantization in Linear-Attention
and SSM LLMs": quantise the state once at the end of a window; inside it, readouts come from
the fixed low-bit state plus the window's high-precision updates). A one-token window
is the per-step INT8 decode of §5.1; inside a window the readouts follow the affine form
S_t = A_t S_{t-1} + B_t of §2.1 started from the reconstructed state; the window's end state is
the textbook rowwise-absmax INT8 quantisation of that recurrence's final state."""
import numpy as np
import pytest

import oracle
from recurrent_state_quantization_gated_b200 import synth


def _window(wl, W, t0=0):
    steps = [synth.tokens(wl, t0 + t) for t in range(W)]
    return {name: np.ascontiguousarray(np.stack([s[name] for s in steps])) for name in steps[0]}


def _int8_state(wl):
    return oracle.int8_quantise_state(synth.initial_state(wl))


def test_one_token_window_is_the_per_step_int8_decode():
    wl = synth.workload(1, B=2, H=3, d=64)
    codes, s = _int8_state(wl)
    toks = _window(wl, 1)
    c1, s1, o1 = oracle.leap_window(toks, codes, s)
    c2, s2, o2 = oracle.decode_step_int8({k: v[0] for k, v in toks.items()}, codes, s)
    np.testing.assert_array_equal(c1, c2)
    np.testing.assert_array_equal(s1, s2)
    np.testing.assert_array_equal(o1[0], o2)


def _f16(x):
    return np.asarray(x, np.float32).astype(np.float16)


@pytest.mark.parametrize("gpc", [False, True])
def test_window_follows_the_affine_recurrence_and_quantises_once(gpc):
    wl = synth.workload(2 if gpc else 1, B=2, H=2, d=64)
    W = 11
    codes, s = _int8_state(wl)
    toks = _window(wl, W)
    c_out, s_out, o = oracle.leap_window(toks, codes, s)
    S_hat = s.view(np.float16).astype(np.float32)[..., None] * codes.astype(np.float32)
    for b in range(wl.B):
        for h in range(wl.H):
            S = S_hat[b, h].astype(np.float64)
            for t in range(W):
                q = synth.bf16_bits_to_f32(toks["q"][t, b, h]).astype(np.float64)
                k = synth.bf16_bits_to_f32(toks["k"][t, b, h]).astype(np.float64)
                v = synth.bf16_bits_to_f32(toks["v"][t, b, h]).astype(np.float64)
                beta = float(toks["beta"][t, b, h])
                g = np.broadcast_to(np.asarray(toks["gate"][t, b, h], dtype=np.float64), (wl.d,))
                A = (np.eye(wl.d) - beta * np.outer(k, k)) @ np.diag(g)
                S = A @ S + beta * np.outer(k, v)
                np.testing.assert_allclose(o[t, b, h], S.T @ q, rtol=2e-6, atol=1e-7 * np.abs(S).max())
            # textbook rowwise absmax INT8 of the final state: s = fp16(absmax / 127), clip(rint(X / s))
            X = S.astype(np.float32)
            s_ref = _f16(np.abs(X).max(axis=1) / np.float32(127.0))
            assert np.abs(s_out[b, h].astype(np.int32) - s_ref.view(np.uint16).astype(np.int32)).max() <= 1
            same = s_out[b, h] == s_ref.view(np.uint16)
            q_ref = np.clip(np.rint(X * (np.float32(1.0) / s_ref.astype(np.float32))[:, None]), -127, 127)
            d = np.abs(c_out[b, h].astype(np.int32) - q_ref.astype(np.int32))[same]
            assert d.max() <= 1 and (d > 0).mean() < 1e-3


def test_quantising_once_per_window_drifts_less_than_every_step():
    """The window's point (the pages' claim for per-window quantisation): with 8-bit codes, the
    readouts of a 32-token window stay closer to the FP32 recurrence than requantising after
    every token (the per-step INT8 decode), on the same inputs."""
    wl = synth.workload(1, B=2, H=4, d=64)
    W = 32
    codes0, s0 = _int8_state(wl)
    toks = _window(wl, W)
    _, _, o_win = oracle.leap_window(toks, codes0, s0)
    S_fp = synth.initial_state(wl)
    codes, s = codes0, s0
    err_step = err_win = 0.0
    for t in range(W):
        tok = {k: v[t] for k, v in toks.items()}
        S_fp, o_fp = oracle.decode_step_fp32(tok, S_fp)
        codes, s, o_step = oracle.decode_step_int8(tok, codes, s)
        err_step += np.linalg.norm(o_step - o_fp) / np.linalg.norm(o_fp)
        err_win += np.linalg.norm(o_win[t] - o_fp) / np.linalg.norm(o_fp)
    assert err_win < err_step
