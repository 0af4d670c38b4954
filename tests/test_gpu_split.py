"""The split form of the decode step (reconstruction, update and readout in one kernel that
writes the updated state; refit and pack afterwards on a side stream): parity with the oracle
under the fused step's criteria, the updated state X against the oracle's, the readout
identical to the fused kernel's, and the first-kernel-only mode."""
import numpy as np
import pytest

import oracle
from recurrent_state_quantization_gated_b200 import synth
from tests.helpers import compare_decode, dev, host_half, oracle_updated_state, tokens_dev

pytestmark = pytest.mark.gpu


def _setup(d, B, H, widths, gpc, seed):
    wl = synth.workload(2 if gpc else 1, B=B, H=H, d=d, seed=seed)
    S0 = synth.initial_state(wl)
    bits = synth.random_bits(H, d, choices=widths, seed=seed + 3)
    w = synth.random_weights(H, d, seed=seed + 4)
    r, c = oracle.fit_scales(S0, w, bits)
    return wl, bits, w, dict(packed=oracle.pack_state(S0, bits, r, c), r=r, c=c)


def _oracle_X(tok, bits, w, st, d):
    S_hat = oracle.unpack_state(st["packed"], bits, st["r"], st["c"])
    B, H = S_hat.shape[:2]
    X = np.zeros_like(S_hat, dtype=np.float64)
    for b in range(B):
        for h in range(H):
            X[b, h], _ = oracle.delta_update(S_hat[b, h], synth.bf16_bits_to_f32(tok["q"][b, h]),
                                             synth.bf16_bits_to_f32(tok["k"][b, h]),
                                             synth.bf16_bits_to_f32(tok["v"][b, h]), float(tok["beta"][b, h]),
                                             tok["gate"][b, h])
    return X


@pytest.mark.parametrize("d,B,H,widths,gpc", [
    (64, 2, 2, (4, 8), False),
    (128, 3, 5, (2, 4, 6, 8), False),
    (128, 2, 7, (4, 6, 8), True),
])
def test_split_form_matches_oracle(d, B, H, widths, gpc):
    import torch
    from recurrent_state_quantization_gated_b200 import api
    wl, bits, w, st = _setup(d, B, H, widths, gpc, seed=d + H)
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    rates = []
    for t in range(3):                          # the GPU starts every step from the oracle's state
        tok = synth.tokens(wl, t)
        td = tokens_dev(tok)
        pk, r, c = dev(st["packed"]), dev(st["r"], torch.float16), dev(st["c"], torch.float16)
        p_g, r_g, c_g, o_g, X_g = api.stepq_decode_step_split(
            td["q"], td["k"], td["v"], td["beta"], td["gate"], dev(bits), dev(w), dev(head_off), bps, pk, r, c,
            pk, r, c)                           # in place
        torch.cuda.synchronize()
        ref = oracle.decode_step(tok, bits, w, st["packed"], st["r"], st["c"])
        rates.append(compare_decode((p_g.cpu().numpy(), host_half(r_g), host_half(c_g), o_g.cpu().numpy()), ref,
                                    bits, d, B, X_ref=oracle_updated_state(tok, bits, st["packed"], st["r"], st["c"]),
                                    label=f"split form d={d} B={B} H={H}", w=w))
        X_ref = _oracle_X(tok, bits, w, st, d)
        np.testing.assert_allclose(X_g.cpu().numpy(), X_ref, rtol=1e-5, atol=1e-6 * np.abs(X_ref).max())
        st = dict(packed=ref[0], r=ref[1], c=ref[2])
    assert max(x["at_gpu_scales"] for x in rates) <= 1e-3


def test_split_readout_equals_fused_and_first_kernel_mode():
    import torch
    from recurrent_state_quantization_gated_b200 import api
    d, B, H = 128, 4, 6
    wl, bits, w, st = _setup(d, B, H, (2, 4, 6, 8), False, seed=31)
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    td = tokens_dev(synth.tokens(wl, 5))
    args = (td["q"], td["k"], td["v"], td["beta"], td["gate"], dev(bits), dev(w), dev(head_off), bps)
    pk, r, c = dev(st["packed"]), dev(st["r"], torch.float16), dev(st["c"], torch.float16)
    _, _, _, o_fused = api.stepq_decode_step(*args, pk, r, c)
    _, _, _, o_split, X_all = api.stepq_decode_step_split(*args, pk, r, c)
    p_none, r_none, c_none, o_first, X_first = api.stepq_decode_step_split(*args, pk, r, c, refit=False)
    torch.cuda.synchronize()
    assert p_none is None and r_none is None and c_none is None
    assert torch.equal(o_fused, o_split) and torch.equal(o_split, o_first)
    assert torch.equal(X_all, X_first)
    # the inputs are untouched when the outputs are separate tensors
    np.testing.assert_array_equal(pk.cpu().numpy(), st["packed"])
