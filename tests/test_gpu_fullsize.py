"""Parity at the decode workloads' full sizes, in the launch configuration the benchmark times
(one launch over every tile of the batch, state updated in place). The GPU steps the whole
batch; the oracle checks a sample of sequences (every head of each) started from the same
packed bytes. Then the 256-step rollout drift of the quantized state against the FP32 state on
the drift workload (heads split between g = 0.999 and g = 0.9, Student-t values): the GPU's
drift must be within 1% of the oracle's.

Bit maps and row weights come from the oracle's offline calibration on the first sequences'
initial states (same distributions as the full batch)."""
import numpy as np
import pytest

import oracle
from recurrent_state_quantization_gated_b200 import synth
from tests.helpers import compare_decode, dev, half_ulps, host_half, oracle_updated_state

pytestmark = pytest.mark.gpu


def _calibrated(wl, n_samples=8):
    seqs = range(min(n_samples, wl.B))
    S0 = synth.initial_state(wl, seqs)
    cal = synth.calib_tokens(wl, seqs)
    bits, w = oracle.calibrate(wl.alloc, wl.candidates, wl.nominal_bits, S0, cal,
                               n_pivots=wl.n_pivots)
    # each FP16 pivot row counts 8 bits of the integer budget and 8 on top (App. D)
    assert bits.astype(np.int64).sum() == wl.nominal_bits * bits.size + 8 * int((bits == 16).sum())
    return bits, w


def _subset(tok, seqs):
    return {name: np.ascontiguousarray(a[seqs]) for name, a in tok.items()}


def _seq_bytes(packed, seqs, bps):
    return np.concatenate([packed[b * bps:(b + 1) * bps] for b in seqs])


def _start_from_oracle(wl, bits, w, S0, seqs):
    """GPU state of the whole batch (fit + pack on the GPU), with the sampled sequences then
    overwritten by the oracle's packed bytes and scales; the GPU's own fit of those sequences
    is checked first (scales within one ulp; its pack of the oracle's scales bit-exact)."""
    import torch
    from recurrent_state_quantization_gated_b200 import api, runtime
    layout = runtime.Layout.build(bits, wl.d)
    st = runtime.QuantizedState.from_fp32(dev(S0), layout, dev(w))
    S_s = np.ascontiguousarray(S0[seqs])
    r_ref, c_ref = oracle.fit_scales(S_s, w, bits)
    p_ref = oracle.pack_state(S_s, bits, r_ref, c_ref)
    assert half_ulps(host_half(st.r)[seqs], r_ref).max() <= 1
    assert half_ulps(host_half(st.c)[seqs], c_ref).max() <= 1
    p_gpu = api.stepq_pack_state(dev(S_s), layout.bits_dev, layout.head_off_dev, layout.bytes_per_seq,
                                 dev(r_ref, torch.float16), dev(c_ref, torch.float16))
    np.testing.assert_array_equal(p_gpu.cpu().numpy(), p_ref)
    bps = layout.bytes_per_seq
    for n, b in enumerate(seqs):
        st.packed[b * bps:(b + 1) * bps].copy_(torch.from_numpy(p_ref[n * bps:(n + 1) * bps]))
        st.r[b].copy_(dev(r_ref[n], torch.float16))
        st.c[b].copy_(dev(c_ref[n], torch.float16))
    return st, (p_ref, r_ref, c_ref)


@pytest.mark.parametrize("index", [1, 2, 3, 4])
def test_full_size_step_on_sampled_sequences(index):
    """gdn 64x32, kda 256x32 (channel gates), gdn4 1024x16 ({2,4,8} bits), drift 128x32 (heads at
    g = 0.999 / 0.9, Student-t values), d = 128; every integer code of the sampled sequences
    checked at the GPU's scales."""
    import torch
    from recurrent_state_quantization_gated_b200 import runtime
    wl = synth.workload(index)
    bits, w = _calibrated(wl)
    S0 = synth.initial_state(wl)
    seqs = sorted({0, wl.B // 3, (2 * wl.B) // 3, wl.B - 1})
    st, (p_ref, r_ref, c_ref) = _start_from_oracle(wl, bits, w, S0, seqs)
    for t in range(2):
        tok = synth.tokens(wl, t)
        o = st.step(**runtime.to_device_tokens(tok))
        torch.cuda.synchronize()
        ts = _subset(tok, seqs)
        ref = oracle.decode_step(ts, bits, w, p_ref, r_ref, c_ref)
        X_ref = oracle_updated_state(ts, bits, p_ref, r_ref, c_ref)
        gpu = (_seq_bytes(st.packed.cpu().numpy(), seqs, st.layout.bytes_per_seq), host_half(st.r)[seqs],
               host_half(st.c)[seqs], o.cpu().numpy()[seqs])
        compare_decode(gpu, ref, bits, wl.d, len(seqs), X_ref=X_ref, label=f"full size {wl.name}, sampled sequences",
                       w=w)
        # the next step starts both sides from the oracle's state again
        p_ref, r_ref, c_ref = ref[:3]
        bps = st.layout.bytes_per_seq
        for n, b in enumerate(seqs):
            st.packed[b * bps:(b + 1) * bps].copy_(torch.from_numpy(p_ref[n * bps:(n + 1) * bps]))
            st.r[b].copy_(dev(r_ref[n], torch.float16))
            st.c[b].copy_(dev(c_ref[n], torch.float16))


def test_rollout_drift_matches_oracle():
    """drift(t) = ||O_q(t) - O_fp32(t)||_F / ||O_fp32(t)||_F over 64 sampled tiles (2 sequences
    x 32 heads), averaged over t = 1..256, each side against its own FP32 rollout; both sides
    run free (no teacher forcing). |drift_gpu - drift_oracle| <= 1% of drift_oracle."""
    import torch
    from recurrent_state_quantization_gated_b200 import api, runtime
    wl = synth.workload(4)
    T = 256
    bits, w = _calibrated(wl, n_samples=16)
    S0 = synth.initial_state(wl)
    seqs = [0, wl.B - 1]
    st, (p, r, c) = _start_from_oracle(wl, bits, w, S0, seqs)
    S_fp = dev(S0)
    S_ref = np.ascontiguousarray(S0[seqs])
    dg, do = [], []
    for t in range(T):
        tok = synth.tokens(wl, t)
        td = runtime.to_device_tokens(tok)
        o_q = st.step(**td)
        S_fp, o_f = api.stepq_decode_step_fp32(td["q"], td["k"], td["v"], td["beta"], td["gate"], S_fp, S_fp)
        torch.cuda.synchronize()
        og, ofg = o_q.cpu().numpy()[seqs].astype(np.float64), o_f.cpu().numpy()[seqs].astype(np.float64)
        ts = _subset(tok, seqs)
        p, r, c, oq_ref = oracle.decode_step(ts, bits, w, p, r, c)
        S_ref, of_ref = oracle.decode_step_fp32(ts, S_ref)
        dg.append(np.linalg.norm(og - ofg) / np.linalg.norm(ofg))
        do.append(np.linalg.norm(oq_ref.astype(np.float64) - of_ref) / np.linalg.norm(of_ref))
    drift_gpu, drift_oracle = float(np.mean(dg)), float(np.mean(do))
    assert drift_oracle > 0
    assert abs(drift_gpu - drift_oracle) <= 0.01 * drift_oracle, (drift_gpu, drift_oracle)
