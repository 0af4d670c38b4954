"""GPU parity of the prefill chunk (reconstruct once, C full-precision gated Delta updates, fit
and pack the boundary state once) against the oracle, in both forms: the sequential form on the
register-resident tile and the chunked WY form on the tensor cores (scalar and channel gates).
Every token's readout within 1e-3 relative, the boundary state under the decode step's criteria;
one token of the sequential form identical to the fused decode step; the two forms agree with
each other to a few 1e-6."""
import numpy as np
import pytest

import oracle
from recurrent_state_quantization_gated_b200 import synth
from tests.helpers import compare_decode, dev, host_half, oracle_chunk_state, with_pivots

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
    compare_decode((p_g.cpu().numpy(), host_half(r_g), host_half(c_g), og[-1]), (p_r, r_r, c_r, o_r[-1]), bits, d, B,
                   X_ref=oracle_chunk_state(toks, bits, packed, r, c), label=f"prefill chunk C={C} d={d} H={H}", w=w)


def test_one_token_chunk_is_the_decode_step():
    import torch
    from recurrent_state_quantization_gated_b200 import api
    d, B, H = 128, 3, 4
    wl, bits, w, packed, r, c = _setup(d, B, H, (2, 4, 6, 8), False, seed=41)
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    toks = _chunk(wl, 1, t0=3)
    td = _dev_tokens(toks)
    args = (dev(bits), dev(w), dev(head_off), bps, dev(packed), dev(r, torch.float16), dev(c, torch.float16))
    a = api.stepq_prefill_chunk(td["q"], td["k"], td["v"], td["beta"], td["gate"], *args, form="seq")
    b = api.stepq_decode_step(td["q"][0], td["k"][0], td["v"][0], td["beta"][0], td["gate"][0], *args)
    torch.cuda.synchronize()
    for x, y in zip(a[:3], b[:3]):
        assert torch.equal(x, y)
    assert torch.equal(a[3][0], b[3])


def _run(api, td, bits, w, head_off, bps, packed, r, c, form, in_place=True):
    import torch
    pk, rr, cc = dev(packed), dev(r, torch.float16), dev(c, torch.float16)
    outs = (pk, rr, cc) if in_place else (None, None, None)
    res = api.stepq_prefill_chunk(td["q"], td["k"], td["v"], td["beta"], td["gate"], dev(bits), dev(w),
                                  dev(head_off), bps, pk, rr, cc, *outs, form=form)
    torch.cuda.synchronize()
    return tuple(x.cpu().numpy() if x.dtype != torch.float16 else host_half(x) for x in res)


def _check_against_oracle(res, toks, bits, w, packed, r, c, d, B, C, form="wy"):
    p_r, r_r, c_r, o_r = oracle.prefill_chunk(toks, bits, w, packed, r, c)
    p_g, r_g, c_g, og = res
    for t in range(C):
        err = np.abs(og[t] - o_r[t]).max(axis=-1) / np.maximum(np.abs(o_r[t]).max(axis=-1), 1e-30)
        assert err.max() <= 1e-3, (t, err.max())
    return compare_decode((p_g, r_g, c_g, og[-1]), (p_r, r_r, c_r, o_r[-1]), bits, d, B,
                          X_ref=oracle_chunk_state(toks, bits, packed, r, c),
                          label=f"prefill chunk C={C} ({'tensor-core' if form == 'wy' else 'sequential'} form)",
                          w=w)


@pytest.mark.parametrize("B,H,widths,C,in_place", [
    (3, 5, (2, 4, 6, 8), 64, True),
    (2, 7, (4, 6, 8), 17, False),     # a ragged chunk (padded to 64 inside)
    (2, 3, (2, 4, 6, 8), 1, True),
    (2, 2, (8,), 64, True),           # every row 8-bit
    (2, 2, (2,), 40, True),           # every row 2-bit
    (8, 40, (4, 6, 8), 33, True),     # 320 tiles: more tiles than SMs, the next codes prefetched
    (4, 16, (8,), 64, True),          # 8-bit rows, 8192 columns: the column-scale rate is tight here
])
def test_tensor_core_prefill_matches_oracle(B, H, widths, C, in_place):
    from recurrent_state_quantization_gated_b200 import api
    d = 128
    wl, bits, w, packed, r, c = _setup(d, B, H, widths, False, seed=7 * B + H + C)
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    toks = _chunk(wl, C)
    res = _run(api, _dev_tokens(toks), bits, w, head_off, bps, packed, r, c, "wy", in_place)
    _check_against_oracle(res, toks, bits, w, packed, r, c, d, B, C)
    assert api.stepq_read_device_flags() == 0


@pytest.mark.parametrize("B,H,widths,C", [
    (3, 5, (2, 4, 6, 8), 64),
    (2, 7, (4, 6, 8), 17),            # a ragged chunk
    (2, 3, (2, 4, 6, 8), 1),
    (8, 40, (4, 6, 8), 33),           # 320 tiles: more tiles than SMs
    (4, 16, (8,), 64),                # 8-bit rows: the column-scale rate is tight here
])
def test_tensor_core_prefill_with_channel_gates_matches_oracle(B, H, widths, C):
    """Channel gates (one gate per key channel and token, the KDA workload's gates) through the
    tensor-core form: the gate-weighted pair products through the reference hierarchy, the
    gate-scaled operands in three bf16 parts."""
    from recurrent_state_quantization_gated_b200 import api
    d = 128
    wl, bits, w, packed, r, c = _setup(d, B, H, widths, True, seed=5 * B + H + C)
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    toks = _chunk(wl, C)
    assert toks["gate"].shape == (C, B, H, d)
    res = _run(api, _dev_tokens(toks), bits, w, head_off, bps, packed, r, c, "wy")
    _check_against_oracle(res, toks, bits, w, packed, r, c, d, B, C)
    assert api.stepq_read_device_flags() == 0


@pytest.mark.parametrize("gpc,B,H,widths,C,n_piv", [
    (True, 2, 5, (4, 6, 8), 9, 11),       # a few pivot rows among mixed widths, channel gates
    (False, 3, 4, (2, 4, 6, 8), 64, 7),   # scalar gates
    (True, 2, 3, (4, 8), 33, 40),         # pivot rows in every 16-row group of some heads
])
def test_tensor_core_prefill_with_pivot_rows_matches_oracle(gpc, B, H, widths, C, n_piv):
    """FP16 pivot rows through the tensor-core form: Z_ij = v_ij / c_j in two bf16 parts for the
    products, the boundary state's pivot rows from the stored binary16 values."""
    from recurrent_state_quantization_gated_b200 import api
    d = 128
    wl, bits, w, packed, r, c = _setup(d, B, H, widths, gpc, seed=3 * B + H + C, pivots=n_piv)
    assert (bits == 16).sum() == n_piv
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    toks = _chunk(wl, C)
    res = _run(api, _dev_tokens(toks), bits, w, head_off, bps, packed, r, c, "wy")
    _check_against_oracle(res, toks, bits, w, packed, r, c, d, B, C)
    assert api.stepq_read_device_flags() == 0


def test_tensor_core_prefill_with_a_pivot_head():
    """A head whose rows are all FP16 pivots (Qwen-style pivot head) beside integer heads."""
    from recurrent_state_quantization_gated_b200 import api
    d, B, H, C = 128, 2, 3, 64
    wl, bits, w, packed, r, c = _setup(d, B, H, (4, 6, 8), False, seed=83)
    bits = bits.copy()
    bits[1] = 16
    r, c = oracle.fit_scales(synth.initial_state(wl), w, bits)
    packed = oracle.pack_state(synth.initial_state(wl), bits, r, c)
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    toks = _chunk(wl, C)
    res = _run(api, _dev_tokens(toks), bits, w, head_off, bps, packed, r, c, "wy")
    _check_against_oracle(res, toks, bits, w, packed, r, c, d, B, C)


@pytest.mark.parametrize("form", ["wy", "seq"])
def test_prefill_with_steep_channel_gates(form):
    """Channel gates down to 0.01, exact zeros (three in one channel within 16 tokens, a whole
    channel of zeros, and ones): gate products of a channel run far below fp32's range inside the
    chunk, where a factorisation through one reference per 16-token block would overflow (the
    tensor-core form) and one running product per key row would be floored (the sequential
    form, which renormalises a row's product below 2^-32)."""
    from recurrent_state_quantization_gated_b200 import api
    d, B, H, C = 128, 2, 3, 64
    wl, bits, w, packed, r, c = _setup(d, B, H, (4, 6, 8), True, seed=79)
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    toks = _chunk(wl, C)
    rng = np.random.default_rng(6)
    g = rng.uniform(0.01, 1.0, toks["gate"].shape).astype(np.float32)
    g[[3, 7, 12], 0, 1, 5] = 0.0
    g[:, 1, 2, 9] = 0.0
    g[:, 0, 0, 17] = 1.0
    toks["gate"] = g
    res = _run(api, _dev_tokens(toks), bits, w, head_off, bps, packed, r, c, form)
    _check_against_oracle(res, toks, bits, w, packed, r, c, d, B, C, form)


def test_tensor_core_and_sequential_forms_agree_under_channel_gates():
    from recurrent_state_quantization_gated_b200 import api
    d, B, H, C = 128, 4, 8, 64
    wl, bits, w, packed, r, c = _setup(d, B, H, (2, 4, 6, 8), True, seed=93)
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    td = _dev_tokens(_chunk(wl, C))
    pw, rw, cw, ow = _run(api, td, bits, w, head_off, bps, packed, r, c, "wy")
    ps, rs, cs, os_ = _run(api, td, bits, w, head_off, bps, packed, r, c, "seq")
    err = np.abs(ow - os_).max(axis=-1) / np.maximum(np.abs(os_).max(axis=-1), 1e-30)
    assert err.max() <= 2e-5, err.max()
    compare_decode((pw, rw, cw, ow[-1]), (ps, rs, cs, os_[-1]), bits, d, B)


def test_tensor_core_prefill_with_fast_decaying_gates():
    """Gates drawn in [0.2, 1] per token (and one exact zero): the gate products fall below
    fp32's range inside the chunk; ratios of them stay exact (log domain)."""
    from recurrent_state_quantization_gated_b200 import api
    d, B, H, C = 128, 2, 3, 64
    wl, bits, w, packed, r, c = _setup(d, B, H, (4, 6, 8), False, seed=77)
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    toks = _chunk(wl, C)
    rng = np.random.default_rng(5)
    toks["gate"] = rng.uniform(0.2, 1.0, toks["gate"].shape).astype(np.float32)
    toks["gate"][10, 0, 1] = 0.0
    res = _run(api, _dev_tokens(toks), bits, w, head_off, bps, packed, r, c, "wy")
    _check_against_oracle(res, toks, bits, w, packed, r, c, d, B, C)


def test_tensor_core_and_sequential_forms_agree():
    """Same inputs through both forms: readouts within 2e-5 (max-normalised per tile) of each
    other; scales within one binary16 ulp; codes equal up to one step on at most 0.1 %."""
    from recurrent_state_quantization_gated_b200 import api
    d, B, H, C = 128, 4, 8, 64
    wl, bits, w, packed, r, c = _setup(d, B, H, (2, 4, 6, 8), False, seed=91)
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    td = _dev_tokens(_chunk(wl, C))
    pw, rw, cw, ow = _run(api, td, bits, w, head_off, bps, packed, r, c, "wy")
    ps, rs, cs, os_ = _run(api, td, bits, w, head_off, bps, packed, r, c, "seq")
    err = np.abs(ow - os_).max(axis=-1) / np.maximum(np.abs(os_).max(axis=-1), 1e-30)
    assert err.max() <= 2e-5, err.max()
    compare_decode((pw, rw, cw, ow[-1]), (ps, rs, cs, os_[-1]), bits, d, B)


def test_tensor_core_prefill_full_size_sampled():
    """The benchmark's prefill workload (GDN shape: 64 sequences x 32 heads, d = 128, 64-token
    chunk) in one launch; the oracle checks four sampled sequences (every head of each)."""
    import torch
    from recurrent_state_quantization_gated_b200 import api
    wl = synth.workload(1)
    d, B, H, C = wl.d, wl.B, wl.H, 64
    S0 = synth.initial_state(wl)
    bits = synth.random_bits(H, d, choices=(4, 6, 8), seed=3)
    w = synth.random_weights(H, d, seed=4)
    seqs = [0, 21, 42, B - 1]
    r, c = oracle.fit_scales(S0, w, bits)
    packed = oracle.pack_state(S0, bits, r, c)
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    toks = _chunk(wl, C)
    p_g, r_g, c_g, o_g = _run(api, _dev_tokens(toks), bits, w, head_off, bps, packed, r, c, "wy")
    sub = {n: np.ascontiguousarray(a[:, seqs]) for n, a in toks.items()}
    p_s = np.concatenate([packed[b * bps:(b + 1) * bps] for b in seqs])
    res = (np.concatenate([p_g[b * bps:(b + 1) * bps] for b in seqs]), r_g[seqs], c_g[seqs], o_g[:, seqs])
    _check_against_oracle(res, sub, bits, w, p_s, r[seqs], c[seqs], d, len(seqs), C)


def test_tensor_core_prefill_full_size_kda_sampled():
    """The KDA prefill workload (256 sequences x 32 heads, d = 128, channel gates, FP16 pivot rows,
    64-token chunk) in one launch of the tensor-core form; the oracle checks four sampled
    sequences (every head of each)."""
    from recurrent_state_quantization_gated_b200 import api
    wl = synth.workload(2)
    d, B, H, C = wl.d, wl.B, wl.H, 64
    S0 = synth.initial_state(wl)
    bits = with_pivots(synth.random_bits(H, d, choices=(4, 6, 8), seed=8), wl.n_pivots, 10)
    w = synth.random_weights(H, d, seed=9)
    seqs = [0, 85, 170, B - 1]
    r, c = oracle.fit_scales(S0, w, bits)
    packed = oracle.pack_state(S0, bits, r, c)
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    toks = _chunk(wl, C)
    p_g, r_g, c_g, o_g = _run(api, _dev_tokens(toks), bits, w, head_off, bps, packed, r, c, "wy")
    sub = {n: np.ascontiguousarray(a[:, seqs]) for n, a in toks.items()}
    p_s = np.concatenate([packed[b * bps:(b + 1) * bps] for b in seqs])
    res = (np.concatenate([p_g[b * bps:(b + 1) * bps] for b in seqs]), r_g[seqs], c_g[seqs], o_g[:, seqs])
    _check_against_oracle(res, sub, bits, w, p_s, r[seqs], c[seqs], d, len(seqs), C)


def test_sequential_prefill_code_paths_agree():
    """The sequential prefill form's two code organisations (stepq_dims.mixed) give the same bits
    on a map with channel gates, pivot rows and rows of mixed widths."""
    import torch
    from recurrent_state_quantization_gated_b200 import api
    d, B, H, C = 128, 2, 5, 9
    wl, bits, w, packed, r, c = _setup(d, B, H, (4, 6, 8), True, seed=61, pivots=7)
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    td = _dev_tokens(_chunk(wl, C))
    args = (td["q"], td["k"], td["v"], td["beta"], td["gate"], dev(bits), dev(w), dev(head_off), bps, dev(packed),
            dev(r, torch.float16), dev(c, torch.float16))
    a = api.stepq_prefill_chunk(*args, form="seq", mixed=0)
    b = api.stepq_prefill_chunk(*args, form="seq", mixed=1)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)
