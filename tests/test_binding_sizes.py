"""The Python binding checks every buffer's size against the call's dimensions before it reaches
the C ABI, which sees only pointers: a buffer short by one along its last axis is refused with
its name, on the host, before any launch. Runs on the CPU: with every size right, the same CPU tensors get as far
as the device check."""
import pytest
import torch

from recurrent_state_quantization_gated_b200 import api

B, H, d, C, T, W = 2, 3, 64, 4, 5, 8
BPS = H * d * d * 6 // 8                     # bytes per sequence at 6 bits per value
bf, f32, f16, u8, i64, i8, f64 = (torch.bfloat16, torch.float32, torch.float16, torch.uint8, torch.int64,
                                  torch.int8, torch.float64)


def z(dtype, *shape):
    return torch.zeros(shape, dtype=dtype)


def HEAD_OFF():
    """The packed layout's head offsets of a uniform 6-bit map: P_h = d/8 * 6 * d bytes per head."""
    return torch.arange(H, dtype=i64) * (BPS // H)


def _state_args():
    return dict(bits=z(u8, H, d) + 6, w=z(f32, H, d), head_off=HEAD_OFF(), bytes_per_seq=BPS,
                packed_in=z(u8, B * BPS), r_in=z(f16, B, H, d), c_in=z(f16, B, H, d),
                packed_out=z(u8, B * BPS), r_out=z(f16, B, H, d), c_out=z(f16, B, H, d))


CASES = {
    "decode_step": (api.stepq_decode_step,
                    lambda: dict(q=z(bf, B, H, d), k=z(bf, B, H, d), v=z(bf, B, H, d), beta=z(f32, B, H),
                                 gate=z(f32, B, H, d), **_state_args(), o=z(f32, B, H, d), pivots=0, mixed=0)),
    "decode_step_split": (api.stepq_decode_step_split,
                          lambda: dict(q=z(bf, B, H, d), k=z(bf, B, H, d), v=z(bf, B, H, d), beta=z(f32, B, H),
                                       gate=z(f32, B, H), **_state_args(), o=z(f32, B, H, d),
                                       x_ws=z(f32, B, H, d, d), side_stream=object(), pivots=0)),
    "prefill_chunk": (api.stepq_prefill_chunk,
                      lambda: dict(q=z(bf, C, B, H, d), k=z(bf, C, B, H, d), v=z(bf, C, B, H, d),
                                   beta=z(f32, C, B, H), gate=z(f32, C, B, H), **_state_args(),
                                   o=z(f32, C, B, H, d), pivots=0, mixed=0)),
    "decode_step_fp32": (api.stepq_decode_step_fp32,
                         lambda: dict(q=z(bf, B, H, d), k=z(bf, B, H, d), v=z(bf, B, H, d), beta=z(f32, B, H),
                                      gate=z(f32, B, H), S_in=z(f32, B, H, d, d), S_out=z(f32, B, H, d, d),
                                      o=z(f32, B, H, d))),
    "decode_step_int8": (api.stepq_decode_step_int8,
                         lambda: dict(q=z(bf, B, H, d), k=z(bf, B, H, d), v=z(bf, B, H, d), beta=z(f32, B, H),
                                      gate=z(f32, B, H), codes_in=z(i8, B, H, d, d), s_in=z(f16, B, H, d),
                                      codes_out=z(i8, B, H, d, d), s_out=z(f16, B, H, d), o=z(f32, B, H, d))),
    "leap_step": (api.stepq_leap_step,
                  lambda: dict(window=W, t=0, q=z(bf, B, H, d), k=z(bf, B, H, d), v=z(bf, B, H, d),
                               beta=z(f32, B, H), gate=z(f32, B, H), codes=z(i8, B, H, d, d), s=z(f16, B, H, d),
                               kbuf=z(bf, W, B, H, d), ubuf=z(f32, W, B, H, d), lbuf=z(f32, W, B, H),
                               o=z(f32, B, H, d))),
    "fit_scales": (api.stepq_fit_scales,
                   lambda: dict(S=z(f32, B, H, d, d), w=z(f32, H, d), bits=z(u8, H, d), r=z(f16, B, H, d),
                                c=z(f16, B, H, d))),
    "pack_state": (api.stepq_pack_state,
                   lambda: dict(S=z(f32, B, H, d, d), bits=z(u8, H, d) + 6, head_off=HEAD_OFF(), bytes_per_seq=BPS,
                                r=z(f16, B, H, d), c=z(f16, B, H, d), packed=z(u8, B * BPS))),
    "unpack_state": (api.stepq_unpack_state,
                     lambda: dict(packed=z(u8, B * BPS), bits=z(u8, H, d) + 6, head_off=HEAD_OFF(), bytes_per_seq=BPS,
                                  r=z(f16, B, H, d), c=z(f16, B, H, d), S_out=z(f32, B, H, d, d))),
    "int8_quantize_state": (api.stepq_int8_quantize_state,
                            lambda: dict(S=z(f32, B, H, d, d), codes=z(i8, B, H, d, d), s=z(f16, B, H, d))),
    "row_impact": (api.stepq_row_impact,
                   lambda: dict(q=z(bf, T, B, H, d), k=z(bf, T, B, H, d), beta=z(f32, T, B, H),
                                gate=z(f32, T, B, H, d), w_out=z(f32, H, d))),
    "calib_distortion": (api.stepq_calib_distortion,
                         lambda: dict(S=z(f32, B, H, d, d), w=z(f32, H, d), b=6, d_row=z(f64, H, d),
                                      d_head=z(f64, H), scratch=z(f64, B, H, d))),
    "calib_distortion_bits": (api.stepq_calib_distortion_bits,
                              lambda: dict(S=z(f32, B, H, d, d), w=z(f32, H, d), bits=z(u8, H, d) + 6,
                                           d_row=z(f64, H, d), d_head=z(f64, H), scratch=z(f64, B, H, d))),
    "calib_distortion_static": (api.stepq_calib_distortion_static,
                                lambda: dict(S=z(f32, B, H, d, d), w=z(f32, H, d), b=6, d_row=z(f64, H, d),
                                             d_head=z(f64, H))),
}

# the tensor whose first axes give the call its dimensions is not checked against itself (a
# state S [B][H][d][d] is: its last axis must match)
SHAPE_SOURCE = {"q", "r"}


@pytest.mark.parametrize("name", sorted(CASES))
def test_every_short_buffer_is_refused_by_name(name):
    fn, make = CASES[name]
    with pytest.raises(ValueError, match="must be a CUDA tensor"):     # every size right
        fn(**make())
    checked = 0
    for key, val in make().items():
        if not isinstance(val, torch.Tensor) or key in SHAPE_SOURCE:
            continue
        if name == "unpack_state" and key == "r":
            continue
        args = make()
        short = torch.zeros(*val.shape[:-1], val.shape[-1] - 1, dtype=val.dtype)   # same rank, last axis short
        args[key] = short
        with pytest.raises(ValueError, match=rf"^{key}: {short.numel()} elements, the call needs {val.numel()}$"):
            fn(**args)
        checked += 1
    assert checked >= 2


@pytest.mark.parametrize("name", ["decode_step", "decode_step_split", "prefill_chunk", "pack_state", "unpack_state"])
def test_a_layout_that_does_not_match_the_bit_map_is_refused(name):
    """head_off / bytes_per_seq are checked against the bit map's packed layout on the host before
    the call reaches the C ABI (a wrong table would move the kernels' accesses; the kernels also
    check every tile's range themselves)."""
    fn, make = CASES[name]
    args = make()
    args["head_off"] = HEAD_OFF().flip(0)
    with pytest.raises(ValueError, match="do not match the bit map's packed layout"):
        fn(**args)
    args = make()
    args["bytes_per_seq"] = BPS - 16
    for key in ("packed", "packed_in", "packed_out"):
        if key in args:
            args[key] = z(u8, B * BPS)
    with pytest.raises(ValueError, match="do not match the bit map's packed layout"):
        fn(**args)
