"""Pins of the oracle's prefill chunk (the native chunk update on the unpacked state, the
boundary state packed once; STEPQuant App. F.1 and App. B.2): one token equals the decode
step; the readouts of a chunk follow the affine form S_t = A_t S_{t-1} + B_t of §2.1 with
A_t = (I - beta_t k_t k_t^T) D_t and B_t = beta_t k_t v_t^T; the boundary state is that
recurrence's final state, fitted and packed once."""
import numpy as np
import pytest

import oracle
from recurrent_state_quantization_gated_b200 import synth


def _chunk_inputs(wl, C):
    steps = [synth.tokens(wl, t) for t in range(C)]
    return {name: np.stack([s[name] for s in steps]) for name in steps[0]}


def _state(wl, seed):
    S0 = synth.initial_state(wl)
    bits = synth.random_bits(wl.H, wl.d, choices=(2, 4, 6, 8), seed=seed)
    w = synth.random_weights(wl.H, wl.d, seed=seed + 1)
    r, c = oracle.fit_scales(S0, w, bits)
    return bits, w, oracle.pack_state(S0, bits, r, c), r, c


def test_one_token_is_the_decode_step():
    wl = synth.workload(1, B=2, H=3, d=64)
    bits, w, packed, r, c = _state(wl, 3)
    toks = _chunk_inputs(wl, 1)
    one = oracle.prefill_chunk(toks, bits, w, packed, r, c)
    dec = oracle.decode_step({k: v[0] for k, v in toks.items()}, bits, w, packed, r, c)
    for a, b in zip(one[:3], dec[:3]):
        np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(one[3][0], dec[3])


@pytest.mark.parametrize("gpc", [False, True])
def test_chunk_follows_the_affine_recurrence_and_packs_its_final_state(gpc):
    wl = synth.workload(2 if gpc else 1, B=2, H=2, d=64)
    C = 9
    bits, w, packed, r, c = _state(wl, 5)
    toks = _chunk_inputs(wl, C)
    p_out, r_out, c_out, o = oracle.prefill_chunk(toks, bits, w, packed, r, c)
    S_hat = oracle.unpack_state(packed, bits, r, c).astype(np.float64)
    X = np.zeros_like(S_hat)
    for b in range(wl.B):
        for h in range(wl.H):
            S = S_hat[b, h]
            for t in range(C):
                q = synth.bf16_bits_to_f32(toks["q"][t, b, h]).astype(np.float64)
                k = synth.bf16_bits_to_f32(toks["k"][t, b, h]).astype(np.float64)
                v = synth.bf16_bits_to_f32(toks["v"][t, b, h]).astype(np.float64)
                beta = float(toks["beta"][t, b, h])
                g = np.broadcast_to(np.asarray(toks["gate"][t, b, h], dtype=np.float64), (wl.d,))
                A = (np.eye(wl.d) - beta * np.outer(k, k)) @ np.diag(g)
                S = A @ S + beta * np.outer(k, v)
                np.testing.assert_allclose(o[t, b, h], S.T @ q, rtol=2e-6, atol=1e-7 * np.abs(S).max())
            X[b, h] = S
    X32 = X.astype(np.float32)
    r_ref, c_ref = oracle.fit_scales(X32, w, bits)
    # r and c are continuous in X: equal, or one ulp apart where the float64 evaluation order
    # of the two forms puts an entry on the other side of a binary16 rounding boundary
    assert np.abs(r_out.astype(np.int32) - r_ref.astype(np.int32)).max() <= 1
    assert np.abs(c_out.astype(np.int32) - c_ref.astype(np.int32)).max() <= 1
    same = (r_out == r_ref).all() and (c_out == c_ref).all()
    if same:
        np.testing.assert_array_equal(p_out, oracle.pack_state(X32, bits, r_ref, c_ref))
