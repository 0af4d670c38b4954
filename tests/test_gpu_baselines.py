"""GPU parity of the comparison state formats (STEPQuant §5.1): the FP32 state and the uniform
rowwise-absmax INT8 state, against the oracle."""
import numpy as np
import pytest

import oracle
from recurrent_state_quantization_gated_b200 import synth
from tests.helpers import assert_codes_close, assert_outputs_close, dev, host_half, tokens_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d,B,H,gpc", [(64, 2, 2, False), (128, 3, 5, True), (128, 17, 9, False)])
def test_fp32_decode(d, B, H, gpc):
    import torch
    from recurrent_state_quantization_gated_b200 import api
    wl = synth.workload(2 if gpc else 1, B=B, H=H, d=d)
    S = synth.initial_state(wl)
    for t in range(4):                  # the GPU starts every step from the oracle's state
        tok = synth.tokens(wl, t)
        td = tokens_dev(tok)
        S_ref, o_ref = oracle.decode_step_fp32(tok, S)
        Sd = dev(S)
        S_new, o = api.stepq_decode_step_fp32(td["q"], td["k"], td["v"], td["beta"], td["gate"], Sd,
                                              Sd if t % 2 else None)
        torch.cuda.synchronize()
        np.testing.assert_allclose(S_new.cpu().numpy(), S_ref, rtol=2e-5, atol=2e-6 * np.abs(S_ref).max())
        assert_outputs_close(o.cpu().numpy(), o_ref, rtol=1e-5)
        S = S_ref


@pytest.mark.parametrize("d,B,H,gpc", [(64, 2, 2, False), (128, 4, 6, True), (128, 21, 3, False)])
def test_int8_quantize_and_decode(d, B, H, gpc):
    import torch
    from recurrent_state_quantization_gated_b200 import api
    wl = synth.workload(2 if gpc else 1, B=B, H=H, d=d)
    S = synth.initial_state(wl)
    codes_ref, s_ref = oracle.int8_quantise_state(S)
    codes, s = api.stepq_int8_quantize_state(dev(S))
    np.testing.assert_array_equal(codes.cpu().numpy(), codes_ref)
    np.testing.assert_array_equal(host_half(s), s_ref)
    c_in, s_in = codes_ref, s_ref
    for t in range(4):                  # the GPU starts every step from the oracle's state
        tok = synth.tokens(wl, t)
        td = tokens_dev(tok)
        c_ref, s_out_ref, o_ref = oracle.decode_step_int8(tok, c_in, s_in)
        codes, s = dev(c_in), dev(s_in, torch.float16)
        codes, s, o = api.stepq_decode_step_int8(td["q"], td["k"], td["v"], td["beta"], td["gate"], codes, s,
                                                 codes, s)
        torch.cuda.synchronize()
        assert_outputs_close(o.cpu().numpy(), o_ref)
        assert_codes_close(codes.cpu().numpy(), c_ref)
        assert np.abs(host_half(s).astype(np.int32) - s_out_ref.astype(np.int32)).max() <= 1
        c_in, s_in = c_ref, s_out_ref
