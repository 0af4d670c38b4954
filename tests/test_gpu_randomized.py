"""Seeded randomized parity cases for the fused decode step and both prefill forms against the
oracle: head width, batch, head count, the candidate widths, gate mode, FP16 pivot rows and the
chunk length are drawn per case (a fixed list of seeds, so every run checks the same cases), and
each case is held to the decode criteria of tests/helpers.py. The cases reach shapes the
hand-picked tests do not: odd head counts, single-width maps next to mixed ones, pivot rows at
random places, and chunk lengths up to 64 for the tensor-core form."""
import numpy as np
import pytest

import oracle
from recurrent_state_quantization_gated_b200 import synth
from tests.helpers import compare_decode, dev, host_half, oracle_chunk_state, oracle_updated_state, tokens_dev, with_pivots

pytestmark = pytest.mark.gpu

WIDTH_SETS = [(2,), (4,), (6,), (8,), (4, 8), (2, 4, 8), (4, 6, 8), (2, 4, 6, 8), (6, 16)]


def _draw(seed):
    rng = np.random.default_rng(1000 + seed)
    d = int(rng.choice([64, 128]))
    B = int(rng.integers(1, 4))
    H = int(rng.integers(1, 9))
    widths = WIDTH_SETS[int(rng.integers(len(WIDTH_SETS)))]
    gpc = bool(rng.integers(2))
    pivots = int(rng.integers(0, 2)) * int(rng.integers(1, max(2, H * d // 16)))
    return d, B, H, widths, gpc, pivots


def _state(d, B, H, widths, gpc, pivots, seed):
    wl = synth.workload(2 if gpc else 1, B=B, H=H, d=d, seed=seed)
    S0 = synth.initial_state(wl)
    bits = with_pivots(synth.random_bits(H, d, choices=widths, seed=seed + 3), pivots, seed + 5)
    w = synth.random_weights(H, d, seed=seed + 4)
    r, c = oracle.fit_scales(S0, w, bits)
    return wl, bits, w, oracle.pack_state(S0, bits, r, c), r, c


@pytest.mark.parametrize("seed", range(32))
def test_randomized_decode_steps(seed):
    import torch
    from recurrent_state_quantization_gated_b200 import api
    d, B, H, widths, gpc, pivots = _draw(seed)
    wl, bits, w, packed, r, c = _state(d, B, H, widths, gpc, pivots, 50 + seed)
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    label = f"randomized decode d={d} B={B} H={H} widths={widths} gates={'channel' if gpc else 'head'} pivots={pivots}"
    for t in range(3):
        tok = synth.tokens(wl, t)
        td = tokens_dev(tok)
        out = api.stepq_decode_step(td["q"], td["k"], td["v"], td["beta"], td["gate"], dev(bits), dev(w),
                                    dev(head_off), bps, dev(packed), dev(r, torch.float16), dev(c, torch.float16))
        torch.cuda.synchronize()
        p_g, r_g, c_g, o_g = out
        ref = oracle.decode_step(tok, bits, w, packed, r, c)
        X_ref = oracle_updated_state(tok, bits, packed, r, c)
        compare_decode((p_g.cpu().numpy(), host_half(r_g), host_half(c_g), o_g.cpu().numpy()), ref, bits, d, B,
                       X_ref=X_ref, label=label, w=w)
        packed, r, c = ref[:3]
    assert api.stepq_read_device_flags() == 0


@pytest.mark.parametrize("seed", range(24))
def test_randomized_prefill_chunks(seed):
    """Both forms where the tensor-core form applies (d = 128), the library's choice elsewhere."""
    import torch
    from recurrent_state_quantization_gated_b200 import api
    d, B, H, widths, gpc, pivots = _draw(100 + seed)
    C = int(np.random.default_rng(2000 + seed).integers(1, 65))
    wl, bits, w, packed, r, c = _state(d, B, H, widths, gpc, pivots, 150 + seed)
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    steps = [synth.tokens(wl, t) for t in range(C)]
    toks = {n: np.ascontiguousarray(np.stack([x[n] for x in steps])) for n in steps[0]}
    td = dict(q=dev(toks["q"], torch.bfloat16), k=dev(toks["k"], torch.bfloat16), v=dev(toks["v"], torch.bfloat16),
              beta=dev(toks["beta"]), gate=dev(toks["gate"]))
    ref = oracle.prefill_chunk(toks, bits, w, packed, r, c)
    X_ref = oracle_chunk_state(toks, bits, packed, r, c)
    for form in (["wy", "seq"] if d == 128 else [None]):
        out = api.stepq_prefill_chunk(td["q"], td["k"], td["v"], td["beta"], td["gate"], dev(bits), dev(w),
                                      dev(head_off), bps, dev(packed), dev(r, torch.float16), dev(c, torch.float16),
                                      form=form)
        torch.cuda.synchronize()
        p_g, r_g, c_g, o_g = out
        og = o_g.cpu().numpy()
        for t in range(C):
            err = np.abs(og[t] - ref[3][t]).max(axis=-1) / np.maximum(np.abs(ref[3][t]).max(axis=-1), 1e-30)
            assert err.max() <= 1e-3, (form, t, err.max())
        label = (f"randomized prefill C={C} form={form} d={d} B={B} H={H} widths={widths} "
                 f"gates={'channel' if gpc else 'head'} pivots={pivots}")
        compare_decode((p_g.cpu().numpy(), host_half(r_g), host_half(c_g), og[-1]), (ref[0], ref[1], ref[2], ref[3][-1]),
                       bits, d, B, X_ref=X_ref, label=label, w=w)
    assert api.stepq_read_device_flags() == 0
