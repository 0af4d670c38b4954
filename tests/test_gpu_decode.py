"""GPU parity of the fused quantized decode step against the oracle. The oracle runs its own
rollout; at every step the GPU starts from the oracle's packed state and scales (teacher
forcing), so differences never accumulate: readouts within 1e-3 relative; row scales within
one binary16 ulp; requantised codes within one step, on at most 0.1% of all integer entries when
the oracle's own updated state is quantised at the GPU's scales, and on at most 0.1% of the
entries where both sides chose the same scales; plus the tiny workload exactly as specified
(half-4/half-8 map, all 16 steps), in-place updates, every bit width, both gate modes, ragged
tile counts and degenerate inputs."""
import numpy as np
import pytest

import oracle
from recurrent_state_quantization_gated_b200 import synth
from tests.helpers import compare_decode, dev, host_half, oracle_updated_state, tokens_dev, with_pivots

pytestmark = pytest.mark.gpu


def _setup(d, B, H, widths, gate_per_channel, seed, host=True, pivots=0):
    """Workload, bits, w, layout and the oracle's initial packed state (host arrays, or
    device tensors with host=False). pivots: key rows made FP16 pivots (width 16)."""
    import torch
    from recurrent_state_quantization_gated_b200 import api
    wl = synth.workload(2 if gate_per_channel else 1, B=B, H=H, d=d, seed=seed)
    S0 = synth.initial_state(wl)
    bits = with_pivots(synth.random_bits(H, d, choices=widths, seed=seed + 3), pivots, seed + 5)
    w = synth.random_weights(H, d, seed=seed + 4)
    r, c = oracle.fit_scales(S0, w, bits)
    packed = oracle.pack_state(S0, bits, r, c)
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    state = dict(packed=packed, r=r, c=c)
    if not host:
        state = dict(packed=dev(packed), r=dev(r, torch.float16), c=dev(c, torch.float16))
    return wl, bits, w, head_off, bps, state


def _check_step(api, wl, bits, w, head_off, bps, st, t, in_place, label=""):
    """Step t on both sides from the oracle's state st (host arrays packed, r, c); returns the
    oracle's next state and the mismatch rates."""
    import torch
    tok = synth.tokens(wl, t)
    td = tokens_dev(tok)
    pk, r, c = dev(st["packed"]), dev(st["r"], torch.float16), dev(st["c"], torch.float16)
    if in_place:
        out = api.stepq_decode_step(td["q"], td["k"], td["v"], td["beta"], td["gate"], dev(bits), dev(w),
                                    dev(head_off), bps, pk, r, c, pk, r, c)
    else:
        out = api.stepq_decode_step(td["q"], td["k"], td["v"], td["beta"], td["gate"], dev(bits), dev(w),
                                    dev(head_off), bps, pk, r, c)
    torch.cuda.synchronize()
    p_g, r_g, c_g, o_g = out
    ref = oracle.decode_step(tok, bits, w, st["packed"], st["r"], st["c"])
    X_ref = oracle_updated_state(tok, bits, st["packed"], st["r"], st["c"])
    rates = compare_decode((p_g.cpu().numpy(), host_half(r_g), host_half(c_g), o_g.cpu().numpy()), ref, bits,
                           wl.d, wl.B, X_ref=X_ref, label=label, w=w)
    return dict(packed=ref[0], r=ref[1], c=ref[2]), rates


@pytest.mark.parametrize("d,B,H,widths,gpc,pivots", [
    (64, 2, 2, (4, 8), False, 0),          # the tiny workload's shape
    (128, 3, 5, (2, 4, 6, 8), False, 0),   # every width, 15 tiles
    (128, 2, 7, (4, 6, 8), True, 0),       # channel gates
    (64, 3, 3, (2, 4, 6, 8), True, 0),
    (128, 1, 1, (6,), False, 0),           # a single tile
    (128, 3, 40, (4, 6, 8), False, 0),     # more heads than the kernel's per-head table cache
    (64, 2, 70, (2, 4, 8), True, 0),
    (128, 3, 6, (4, 6, 8), True, 13),      # FP16 pivot rows among the integer rows (KDA)
    (64, 2, 5, (2, 4, 6, 8), False, 21),
    (128, 2, 3, (16,), False, 0),          # whole pivot heads (every row FP16)
    (128, 2, 4, (6, 16), False, 0),        # mixed, pivot rows in width-uniform and mixed warps
])
def test_decode_teacher_forced(d, B, H, widths, gpc, pivots):
    from recurrent_state_quantization_gated_b200 import api
    wl, bits, w, head_off, bps, st = _setup(d, B, H, widths, gpc, seed=d + B + H, pivots=pivots)
    rates = []
    label = f"teacher-forced d={d} B={B} H={H} widths={widths} gates={'channel' if gpc else 'head'} pivots={pivots}"
    for t in range(6):
        st, r = _check_step(api, wl, bits, w, head_off, bps, st, t, in_place=(t % 2 == 0), label=label)
        rates.append(r)
    assert max(r["at_gpu_scales"] for r in rates) <= 1e-3   # every integer code, every step
    assert np.mean([r["r_mismatch"] for r in rates]) < 1e-2 and np.mean([r["c_mismatch"] for r in rates]) < 1e-2
    assert max(r["raw"] for r in rates) <= 1e-3              # against the oracle's own codes and scales


def test_tiny_workload_as_specified():
    """The tiny oracle workload exactly as specified: B=2, H=2, d=64, the seeded half-4 /
    half-8 map of each head, row impact from its calibration stream, all T=16 decode steps,
    teacher-forced, every step checked (codes at the GPU's scales on every integer entry)."""
    import torch
    from recurrent_state_quantization_gated_b200 import api
    wl = synth.workload(0)
    assert (wl.B, wl.H, wl.d, wl.T) == (2, 2, 64, 16)
    bits = synth.half_bits(wl)
    assert ((bits == 4).sum(axis=1) == wl.d // 2).all() and ((bits == 8).sum(axis=1) == wl.d // 2).all()
    w = oracle.row_impact(synth.calib_tokens(wl))
    S0 = synth.initial_state(wl)
    r, c = oracle.fit_scales(S0, w, bits)
    st = dict(packed=oracle.pack_state(S0, bits, r, c), r=r, c=c)
    head_off, bps, _ = api.stepq_packed_layout(bits, wl.d, wl.B)
    rates = []
    for t in range(wl.T):
        st, rt = _check_step(api, wl, bits, w, head_off, bps, st, t, in_place=(t % 2 == 1),
                             label="tiny_b2_h2_d64_t16 (half-4/half-8, 16 steps)")
        rates.append(rt)
    assert max(r["at_gpu_scales"] for r in rates) <= 1e-3


def test_decode_many_tiles_ragged():
    """More tiles than persistent CTAs, and a count that leaves a ragged last wave."""
    from recurrent_state_quantization_gated_b200 import api
    wl, bits, w, head_off, bps, st = _setup(128, 61, 11, (4, 6, 8), False, seed=9)
    _check_step(api, wl, bits, w, head_off, bps, st, 0, in_place=True)


def test_in_place_equals_out_of_place():
    import torch
    from recurrent_state_quantization_gated_b200 import api
    wl, bits, w, head_off, bps, st = _setup(128, 4, 6, (2, 4, 6, 8), True, seed=21, host=False)
    td = tokens_dev(synth.tokens(wl, 3))
    a = api.stepq_decode_step(td["q"], td["k"], td["v"], td["beta"], td["gate"], dev(bits), dev(w), dev(head_off),
                              bps, st["packed"], st["r"], st["c"])
    pk, r, c = st["packed"].clone(), st["r"].clone(), st["c"].clone()
    b = api.stepq_decode_step(td["q"], td["k"], td["v"], td["beta"], td["gate"], dev(bits), dev(w), dev(head_off),
                              bps, pk, r, c, pk, r, c)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_decode_degenerate_inputs():
    """beta = 0 and g = 1 leave the reconstructed state unchanged before the refit: o = S_hat^T q;
    an all-zero state stays zero with floor scales."""
    import torch
    from recurrent_state_quantization_gated_b200 import api
    d, B, H = 128, 2, 3
    wl, bits, w, head_off, bps, st = _setup(d, B, H, (2, 4, 6, 8), False, seed=5, host=False)
    tok = synth.tokens(wl, 0)
    tok["beta"][:] = 0.0
    tok["gate"][:] = 1.0
    td = tokens_dev(tok)
    S_hat = api.stepq_unpack_state(st["packed"], dev(bits), dev(head_off), bps, st["r"], st["c"])
    _, _, _, o = api.stepq_decode_step(td["q"], td["k"], td["v"], td["beta"], td["gate"], dev(bits), dev(w),
                                       dev(head_off), bps, st["packed"], st["r"], st["c"])
    q = torch.from_numpy(synth.bf16_bits_to_f32(tok["q"])).cuda().double()
    ref = torch.einsum("bhij,bhi->bhj", S_hat.double(), q)
    torch.testing.assert_close(o.double(), ref, rtol=1e-5, atol=1e-6)
    # zero state
    z = torch.zeros_like(S_hat)
    r0, c0 = api.stepq_fit_scales(z, dev(w), dev(bits))
    pz = api.stepq_pack_state(z, dev(bits), dev(head_off), bps, r0, c0)
    tok["v"][:] = 0
    td = tokens_dev(tok)
    pk, r1, c1, o1 = api.stepq_decode_step(td["q"], td["k"], td["v"], td["beta"], td["gate"], dev(bits), dev(w),
                                           dev(head_off), bps, pz, r0, c0)
    torch.cuda.synchronize()
    assert not pk.any() and not o1.any()
    floor = np.float16(2.0 ** -14).view(np.uint16)
    r_zero, c_zero = oracle.fit_scales(np.zeros((B, H, d, d), np.float32), w, bits)   # r = fp16(2^-14 / w)
    np.testing.assert_array_equal(host_half(r1), r_zero)
    assert (host_half(c1) == floor).all() and (c_zero == floor).all()


def test_device_error_word_is_clear_after_decodes():
    from recurrent_state_quantization_gated_b200 import api
    wl, bits, w, head_off, bps, st = _setup(128, 3, 4, (4, 8), False, seed=2, host=False)
    td = tokens_dev(synth.tokens(wl, 0))
    api.stepq_decode_step(td["q"], td["k"], td["v"], td["beta"], td["gate"], dev(bits), dev(w), dev(head_off), bps,
                          st["packed"], st["r"], st["c"])
    assert api.stepq_read_device_flags() == 0


def test_undeclared_pivot_rows_raise_the_device_flag():
    """A bit map with FP16 pivot rows decoded with dims.pivots = 0: the kernel keeps every
    access inside the tile and raises bit 1 of the device error word."""
    import torch
    from recurrent_state_quantization_gated_b200 import api
    wl, bits, w, head_off, bps, st = _setup(128, 2, 3, (4, 16), False, seed=12, host=False)
    assert (bits == 16).any()
    td = tokens_dev(synth.tokens(wl, 0))
    assert api.stepq_read_device_flags() == 0
    api.stepq_decode_step(td["q"], td["k"], td["v"], td["beta"], td["gate"], dev(bits), dev(w), dev(head_off), bps,
                          st["packed"], st["r"], st["c"], pivots=0)
    torch.cuda.synchronize()
    assert api.stepq_read_device_flags() == 2
    api.stepq_decode_step(td["q"], td["k"], td["v"], td["beta"], td["gate"], dev(bits), dev(w), dev(head_off), bps,
                          st["packed"], st["r"], st["c"], pivots=1)
    torch.cuda.synchronize()
    assert api.stepq_read_device_flags() == 0


@pytest.mark.parametrize("pivots", [0, 6])
def test_mixed_and_width_specialised_paths_agree(pivots):
    """The decode step's two code organisations (stepq_dims.mixed: one path for every row width,
    or width-specialised paths per warp) give the same bits on the same inputs; half the heads
    here have one width per head, half mix widths across rows."""
    import torch
    from recurrent_state_quantization_gated_b200 import api
    d, B, H = 128, 3, 6
    wl = synth.workload(1, B=B, H=H, d=d, seed=17)
    S0 = synth.initial_state(wl)
    bits = synth.random_bits(H, d, choices=(2, 4, 6, 8), seed=5)
    bits[: H // 2] = bits[: H // 2, :1]                      # heads 0-2: one width each
    bits = with_pivots(bits, pivots, 7)
    w = synth.random_weights(H, d, seed=6)
    r, c = oracle.fit_scales(S0, w, bits)
    packed = oracle.pack_state(S0, bits, r, c)
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    td = tokens_dev(synth.tokens(wl, 2))
    args = (td["q"], td["k"], td["v"], td["beta"], td["gate"], dev(bits), dev(w), dev(head_off), bps,
            dev(packed), dev(r, torch.float16), dev(c, torch.float16))
    a = api.stepq_decode_step(*args, mixed=0)
    b = api.stepq_decode_step(*args, mixed=1, widths=0)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("widths,pivots", [((2, 4, 8), 0), ((4, 6, 8), 0), ((4, 6, 8), 9), ((4, 8), 0)])
def test_declared_width_sets_agree_with_the_generic_path(widths, pivots):
    """A mixed launch whose bit map holds only {2, 4, 8} or only {4, 6, 8} (the 4-bit and
    6-bit row allocations) runs per-row code for those widths alone; its results are the bits of
    the generic per-row path (widths undeclared)."""
    import torch
    from recurrent_state_quantization_gated_b200 import api
    d, B, H = 128, 3, 5
    wl = synth.workload(1, B=B, H=H, d=d, seed=31)
    S0 = synth.initial_state(wl)
    bits = with_pivots(synth.random_bits(H, d, choices=widths, seed=8), pivots, 9)
    w = synth.random_weights(H, d, seed=6)
    r, c = oracle.fit_scales(S0, w, bits)
    packed = oracle.pack_state(S0, bits, r, c)
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    td = tokens_dev(synth.tokens(wl, 1))
    args = (td["q"], td["k"], td["v"], td["beta"], td["gate"], dev(bits), dev(w), dev(head_off), bps,
            dev(packed), dev(r, torch.float16), dev(c, torch.float16))
    mask = api.width_mask(bits)
    a = api.stepq_decode_step(*args, mixed=1, widths=0)
    b = api.stepq_decode_step(*args, mixed=1, widths=mask)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    assert api.stepq_read_device_flags() == 0


def test_a_wait_that_runs_out_is_reported_and_the_context_stays_usable():
    """The kernels' bounded waits (tile copies, tensor-core rounds) give up after their limit,
    raise bit 0 of the device error word and return: a wait that nothing completes reports bit 0
    after its limit, and the next decode step runs normally with the error word clear."""
    import time

    import torch
    from recurrent_state_quantization_gated_b200 import api
    assert api.stepq_read_device_flags() == 0
    t0 = time.perf_counter()
    api.stepq_selftest_wait(50_000_000)                     # 50 ms
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 >= 0.04
    assert api.stepq_read_device_flags() == 1
    wl = synth.workload(1, B=2, H=3, d=128, seed=23)
    S0 = synth.initial_state(wl)
    bits = synth.random_bits(wl.H, wl.d, choices=(4, 6, 8), seed=2)
    w = synth.random_weights(wl.H, wl.d, seed=3)
    r, c = oracle.fit_scales(S0, w, bits)
    packed = oracle.pack_state(S0, bits, r, c)
    head_off, bps, _ = api.stepq_packed_layout(bits, wl.d, wl.B)
    tok = synth.tokens(wl, 0)
    td = tokens_dev(tok)
    p_g, r_g, c_g, o_g = api.stepq_decode_step(td["q"], td["k"], td["v"], td["beta"], td["gate"], dev(bits), dev(w),
                                               dev(head_off), bps, dev(packed), dev(r, torch.float16),
                                               dev(c, torch.float16))
    torch.cuda.synchronize()
    ref = oracle.decode_step(tok, bits, w, packed, r, c)
    compare_decode((p_g.cpu().numpy(), host_half(r_g), host_half(c_g), o_g.cpu().numpy()), ref, bits, wl.d, wl.B)
    assert api.stepq_read_device_flags() == 0


def test_a_mixed_launch_without_declared_widths_can_be_captured_in_a_graph():
    """Inside CUDA-graph capture the binding cannot read the bit map back, so a mixed launch whose
    widths are not declared runs the generic per-row code; its results equal the declared launch's."""
    import torch
    from recurrent_state_quantization_gated_b200 import api
    d, B, H = 128, 2, 4
    wl = synth.workload(1, B=B, H=H, d=d, seed=41)
    S0 = synth.initial_state(wl)
    bits = synth.random_bits(H, d, choices=(2, 4, 8), seed=12)
    w = synth.random_weights(H, d, seed=13)
    r, c = oracle.fit_scales(S0, w, bits)
    packed = oracle.pack_state(S0, bits, r, c)
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    td = tokens_dev(synth.tokens(wl, 0))
    bits_d, w_d, ho_d = dev(bits), dev(w), dev(head_off)
    ref = api.stepq_decode_step(td["q"], td["k"], td["v"], td["beta"], td["gate"], bits_d, w_d, ho_d, bps, dev(packed),
                                dev(r, torch.float16), dev(c, torch.float16), pivots=0, mixed=1,
                                widths=api.width_mask(bits))
    pk, rr, cc = dev(packed), dev(r, torch.float16), dev(c, torch.float16)
    out = (torch.empty_like(pk), torch.empty_like(rr), torch.empty_like(cc),
           torch.empty((B, H, d), dtype=torch.float32, device="cuda"))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        api.stepq_decode_step(td["q"], td["k"], td["v"], td["beta"], td["gate"], bits_d, w_d, ho_d, bps, pk, rr, cc,
                              *out, pivots=0, mixed=1)
    g.replay()
    torch.cuda.synchronize()
    for x, y in zip(ref, out):
        assert torch.equal(x, y)
