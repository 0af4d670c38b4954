"""GPU parity of the prefill chunk (reconstruct once, C full-precision gated Delta updates on
the register-resident tile, fit and pack the boundary state once) against the oracle: every
token's readout within 1e-3 relative, the boundary state under the decode step's criteria;
one token identical to the fused decode step."""
import numpy as np
import pytest

import oracle
from recurrent_state_quantization_gated_b200 import synth
from tests.helpers import compare_decode, dev, host_half, with_pivots

pytestmark = pytest.mark.gpu


def _chunk(wl, C, t0=0):
    steps = [synth.tokens(wl, t0 + t) for t in range(C)]
    return {name: np.ascontiguousarray(np.stack([s[name] for s in steps])) for name in steps[0]}


def _dev_tokens(toks):
    import torch
    return dict(q=dev(toks["q"], torch.bfloat16), k=dev(toks["k"], torch.bfloat16), v=dev(toks["v"], torch.bfloat16),
                beta=dev(toks["beta"]), gate=dev(toks["gate"]))


def _setup(d, B, H, widths, gpc, seed, pivots=0):
    wl = synth.workload(2 if gpc else 1, B=B, H=H, d=d, seed=seed)
    S0 = synth.initial_state(wl)
    bits = with_pivots(synth.random_bits(H, d, choices=widths, seed=seed + 3), pivots, seed + 5)
    w = synth.random_weights(H, d, seed=seed + 4)
    r, c = oracle.fit_scales(S0, w, bits)
    return wl, bits, w, oracle.pack_state(S0, bits, r, c), r, c


@pytest.mark.parametrize("d,B,H,widths,gpc,C,pivots", [
    (64, 2, 2, (4, 8), False, 2, 0),
    (128, 3, 5, (2, 4, 6, 8), False, 7, 0),
    (128, 2, 7, (4, 6, 8), True, 16, 0),     # channel gates
    (64, 3, 3, (2, 4, 6, 8), True, 33, 0),
    (128, 2, 5, (4, 6, 8), True, 9, 11),     # FP16 pivot rows
])
def test_prefill_chunk_matches_oracle(d, B, H, widths, gpc, C, pivots):
    import torch
    from recurrent_state_quantization_gated_b200 import api
    wl, bits, w, packed, r, c = _setup(d, B, H, widths, gpc, seed=d + H + C, pivots=pivots)
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    toks = _chunk(wl, C)
    td = _dev_tokens(toks)
    pk, rr, cc = dev(packed), dev(r, torch.float16), dev(c, torch.float16)
    p_g, r_g, c_g, o_g = api.stepq_prefill_chunk(td["q"], td["k"], td["v"], td["beta"], td["gate"], dev(bits),
                                                 dev(w), dev(head_off), bps, pk, rr, cc, pk, rr, cc)   # in place
    torch.cuda.synchronize()
    p_r, r_r, c_r, o_r = oracle.prefill_chunk(toks, bits, w, packed, r, c)
    og, orf = o_g.cpu().numpy(), o_r
    for t in range(C):
        compare_o = np.abs(og[t] - orf[t]).max(axis=-1) / np.maximum(np.abs(orf[t]).max(axis=-1), 1e-30)
        assert compare_o.max() <= 1e-3, (t, compare_o.max())
    compare_decode((p_g.cpu().numpy(), host_half(r_g), host_half(c_g), og[-1]), (p_r, r_r, c_r, o_r[-1]), bits, d, B)


def test_one_token_chunk_is_the_decode_step():
    import torch
    from recurrent_state_quantization_gated_b200 import api
    d, B, H = 128, 3, 4
    wl, bits, w, packed, r, c = _setup(d, B, H, (2, 4, 6, 8), False, seed=41)
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    toks = _chunk(wl, 1, t0=3)
    td = _dev_tokens(toks)
    args = (dev(bits), dev(w), dev(head_off), bps, dev(packed), dev(r, torch.float16), dev(c, torch.float16))
    a = api.stepq_prefill_chunk(td["q"], td["k"], td["v"], td["beta"], td["gate"], *args)
    b = api.stepq_decode_step(td["q"][0], td["k"][0], td["v"][0], td["beta"][0], td["gate"][0], *args)
    torch.cuda.synchronize()
    for x, y in zip(a[:3], b[:3]):
        assert torch.equal(x, y)
    assert torch.equal(a[3][0], b[3])
