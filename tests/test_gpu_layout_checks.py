"""Head-offset tables the kernels cannot trust. The C ABI sees only pointers, so every kernel that
addresses the packed state checks each tile's head range itself: the range must be 16-byte
aligned, ascending, inside the sequence (bytes_per_seq) and hold the tile's bytes under the bit
map. A tile that fails is skipped -- nothing of it is read or written -- and bit 2 of the device
error word is raised. These tests call the C ABI directly (the Python binding refuses such
tables on the host first) with tables chosen so that every access stays inside the buffers even
if a check were missing: a head whose bit map was widened past its range, and a bytes_per_seq
shorter than the table, over buffers sized for the true layout."""
import ctypes

import numpy as np
import pytest

import oracle
from recurrent_state_quantization_gated_b200 import synth
from tests.helpers import dev, host_half, tokens_dev

pytestmark = pytest.mark.gpu

BAD_LAYOUT = 4


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _case(widths=(4, 6, 8), d=128, B=3, H=4, seed=3):
    import torch
    from recurrent_state_quantization_gated_b200 import api
    wl = synth.workload(1, B=B, H=H, d=d, seed=seed)
    S0 = synth.initial_state(wl)
    bits = synth.random_bits(H, d, choices=widths, seed=seed + 1)
    w = synth.random_weights(H, d, seed=seed + 2)
    r, c = oracle.fit_scales(S0, w, bits)
    packed = oracle.pack_state(S0, bits, r, c)
    head_off, bps, _ = api.stepq_packed_layout(bits, d, B)
    return wl, bits, w, head_off, bps, packed, r, c


def _decode_raw(fn, wl, bits_dev, w, head_off_dev, bps, packed, r, c, chunk=None, toks=None):
    """One call of a decode-shaped entry point through the C ABI; returns the outputs."""
    import torch
    from recurrent_state_quantization_gated_b200 import _lib
    td = toks if toks is not None else tokens_dev(synth.tokens(wl, 0))
    pk_in, r_in, c_in = dev(packed), dev(r, torch.float16), dev(c, torch.float16)
    pk_out, r_out, c_out = pk_in.clone(), r_in.clone(), c_in.clone()
    oshape = (chunk,) + tuple(td["q"].shape[-3:]) if chunk else tuple(td["q"].shape)
    o = torch.full(oshape, 7.0, dtype=torch.float32, device="cuda")
    dims = _lib.Dims(wl.B, wl.H, wl.d, wl.d, 0, 0, 1)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    args = [_p(td["q"]), _p(td["k"]), _p(td["v"]), _p(td["beta"]), _p(td["gate"]), _p(bits_dev), _p(w),
            _p(head_off_dev), ctypes.c_int64(bps), _p(pk_in), _p(r_in), _p(c_in), _p(pk_out), _p(r_out), _p(c_out),
            _p(o), stream]
    lib = _lib.lib()
    rc = getattr(lib, fn)(dims, *( [ctypes.c_int(chunk)] if chunk else []), *args)
    torch.cuda.synchronize()
    assert rc == 0, lib.stepq_last_error()
    return pk_out, r_out, c_out, o


def test_decode_skips_a_head_whose_range_cannot_hold_its_tile():
    import torch
    from recurrent_state_quantization_gated_b200 import api
    wl, bits, w, head_off, bps, packed, r, c = _case()
    wide = bits.copy()
    wide[0] = 8                                   # head 0 now needs more bytes than its range has
    assert oracle.tile_bytes(wide[0], wl.d) > head_off[1] - head_off[0]
    assert api.stepq_read_device_flags() == 0
    good = _decode_raw("stepq_decode_step", wl, dev(bits), dev(w), dev(head_off), bps, packed, r, c)
    assert api.stepq_read_device_flags() == 0
    bad = _decode_raw("stepq_decode_step", wl, dev(wide), dev(w), dev(head_off), bps, packed, r, c)
    assert api.stepq_read_device_flags() == BAD_LAYOUT
    pk_g, r_g, c_g, o_g = good
    pk_b, r_b, c_b, o_b = bad
    # head 0 of every sequence: nothing written (outputs keep their initial contents)
    pk_in = dev(packed)
    for b in range(wl.B):
        s0 = b * bps + head_off[0]
        assert torch.equal(pk_b[s0:s0 + head_off[1]], pk_in[s0:s0 + head_off[1]])
    assert (o_b[:, 0] == 7.0).all()
    assert torch.equal(r_b[:, 0], dev(r, torch.float16)[:, 0]) and torch.equal(c_b[:, 0], dev(c, torch.float16)[:, 0])
    # the other heads decode as with the right bit map
    for b in range(wl.B):
        s1 = b * bps + head_off[1]
        assert torch.equal(pk_b[s1:(b + 1) * bps], pk_g[s1:(b + 1) * bps])
    assert torch.equal(o_b[:, 1:], o_g[:, 1:]) and torch.equal(r_b[:, 1:], r_g[:, 1:])


def test_decode_with_a_short_bytes_per_seq_raises_the_flag():
    from recurrent_state_quantization_gated_b200 import api
    wl, bits, w, head_off, bps, packed, r, c = _case()
    assert api.stepq_read_device_flags() == 0
    _decode_raw("stepq_decode_step", wl, dev(bits), dev(w), dev(head_off), bps - 16, packed, r, c)
    assert api.stepq_read_device_flags() == BAD_LAYOUT
    _decode_raw("stepq_decode_step", wl, dev(bits), dev(w), dev(head_off), bps, packed, r, c)
    assert api.stepq_read_device_flags() == 0


def test_tensor_core_prefill_skips_a_bad_head():
    import torch
    from recurrent_state_quantization_gated_b200 import api
    wl, bits, w, head_off, bps, packed, r, c = _case(widths=(4, 6), B=2, H=3)
    C = 8
    steps = [synth.tokens(wl, t) for t in range(C)]
    toks = {n: np.ascontiguousarray(np.stack([x[n] for x in steps])) for n in steps[0]}
    td = tokens_dev(toks)
    wide = bits.copy()
    wide[1] = 8
    assert api.stepq_read_device_flags() == 0
    pk_b, r_b, c_b, o_b = _decode_raw("stepq_prefill_chunk_wy", wl, dev(wide), dev(w), dev(head_off), bps, packed, r,
                                      c, chunk=C, toks=td)
    assert api.stepq_read_device_flags() == BAD_LAYOUT
    assert (o_b[:, :, 1] == 7.0).all() and (o_b[:, :, 0] != 7.0).any()
    pk_in = dev(packed)
    for b in range(wl.B):
        s = b * bps + head_off[1]
        assert torch.equal(pk_b[s:b * bps + head_off[2]], pk_in[s:b * bps + head_off[2]])


def test_pack_and_unpack_skip_a_bad_head():
    import torch
    from recurrent_state_quantization_gated_b200 import _lib, api
    wl, bits, w, head_off, bps, packed, r, c = _case(B=2, H=3)
    wide = bits.copy()
    wide[2] = 8                                   # the last head: its range ends at bytes_per_seq
    S = dev(synth.initial_state(wl))
    rr, cc = dev(r, torch.float16), dev(c, torch.float16)
    dims = _lib.Dims(wl.B, wl.H, wl.d, wl.d, 0, 0, 0)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    out = torch.full((wl.B * bps,), 0xAB, dtype=torch.uint8, device="cuda")
    assert api.stepq_read_device_flags() == 0
    rc = _lib.lib().stepq_pack_state(dims, _p(S), _p(dev(wide)), _p(dev(head_off)), ctypes.c_int64(bps), _p(rr),
                                     _p(cc), _p(out), stream)
    torch.cuda.synchronize()
    assert rc == 0 and api.stepq_read_device_flags() == BAD_LAYOUT
    for b in range(wl.B):
        assert (out[b * bps + head_off[2]:(b + 1) * bps] == 0xAB).all()
        assert (out[b * bps:b * bps + head_off[2]] != 0xAB).any()
    S_out = torch.full_like(S, 3.0)
    rc = _lib.lib().stepq_unpack_state(dims, _p(dev(packed)), _p(dev(wide)), _p(dev(head_off)), ctypes.c_int64(bps),
                                       _p(rr), _p(cc), _p(S_out), stream)
    torch.cuda.synchronize()
    assert rc == 0 and api.stepq_read_device_flags() == BAD_LAYOUT
    assert (S_out[:, 2] == 3.0).all() and (S_out[:, :2] != 3.0).any()
