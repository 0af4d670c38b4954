"""The packed token layout of the runtime (q | k | v | beta | gate in one byte buffer, each part
16-byte aligned) that lets one host-to-device copy carry a step's inputs: the typed views read
back exactly the host arrays, for decode steps, prefill chunks and channel gates."""
import numpy as np
import pytest
import torch

from recurrent_state_quantization_gated_b200 import runtime, synth


def _chunk(wl, C):
    steps = [synth.tokens(wl, t) for t in range(C)]
    return {n: np.ascontiguousarray(np.stack([s[n] for s in steps])) for n in steps[0]}


@pytest.mark.parametrize("make", [
    lambda: synth.tokens(synth.workload(0), 5),                       # one step, d = 64
    lambda: synth.tokens(synth.workload(2, B=3, H=5), 1),             # channel gates [B][H][d]
    lambda: _chunk(synth.workload(1, B=2, H=3), 7),                   # a prefill chunk
])
def test_views_of_the_packed_buffer_equal_the_host_arrays(make):
    tok = make()
    buf = torch.from_numpy(runtime.pack_tokens(tok))
    views = runtime.token_views(buf, tok)
    ref = runtime.to_device_tokens(tok, device="cpu")
    for name in runtime.TOKEN_FIELDS:
        assert views[name].dtype == ref[name].dtype and views[name].shape == ref[name].shape
        assert torch.equal(views[name], ref[name])
        assert (views[name].data_ptr() - buf.data_ptr()) % 16 == 0


def test_wrong_buffer_size_is_refused():
    tok = synth.tokens(synth.workload(0), 0)
    buf = torch.from_numpy(runtime.pack_tokens(tok))
    with pytest.raises(ValueError):
        runtime.token_views(buf[:-16], tok)
