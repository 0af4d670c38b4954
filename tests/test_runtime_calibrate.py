"""Host logic of the library's offline calibration (runtime.calibrate), on the CPU.

The GPU statistics that runtime.calibrate reads (row impact, candidate distortions) are replaced
here by the oracle's values, so what is checked is its host part: the mean log retention of the
calibration gates and the lifetimes over the horizon (App. A.3), the lifetime-weighted objective
(§3.2), pivot ranking and the (16 - 8) budget accounting (App. C.2, App. D), and the host
allocation library (multiple-choice DP, Lagrangian with repair) — all against the oracle's own
calibration. The GPU statistics themselves are compared with the oracle by the GPU tests."""
import numpy as np
import pytest
import torch

import oracle
from recurrent_state_quantization_gated_b200 import runtime, synth


@pytest.fixture
def oracle_statistics(monkeypatch):
    api = runtime.api

    def row_impact(q, k, beta, gate):
        return torch.from_numpy(oracle.row_impact(dict(q=q, k=k, beta=beta, gate=gate)))

    def distortion(S, w, b):
        dr, dh = oracle.calib_distortion(S.numpy(), w.numpy(), int(b))
        return torch.from_numpy(dr), torch.from_numpy(dh)

    def distortion_bits(S, w, bits):
        dr, dh = oracle.calib_distortion_bits(S.numpy(), w.numpy(), bits.numpy())
        return torch.from_numpy(dr), torch.from_numpy(dh)

    monkeypatch.setattr(api, "stepq_row_impact", row_impact)
    monkeypatch.setattr(api, "stepq_calib_distortion", distortion)
    monkeypatch.setattr(api, "stepq_calib_distortion_bits", distortion_bits)


@pytest.mark.parametrize("idx,over,pivots", [
    (1, dict(B=3, H=6, d=64), 0),                 # head units, DP
    (1, dict(B=3, H=6, d=64), 2),                 # head units with two FP16 pivot heads
    (2, dict(B=3, H=2, d=64), 0),                 # key-row units under channel gates, Lagrangian
    (2, dict(B=3, H=2, d=64), 5),                 # key rows with five FP16 pivot rows
])
def test_runtime_calibration_matches_the_oracle(oracle_statistics, idx, over, pivots):
    wl = synth.workload(idx, **over)
    S0 = synth.initial_state(wl)
    cal = synth.calib_tokens(wl)
    bits_ref, w_ref = oracle.calibrate(wl.alloc, wl.candidates, wl.nominal_bits, S0, cal, n_pivots=pivots)
    bits, w = runtime.calibrate(wl.alloc, wl.candidates, wl.nominal_bits, torch.from_numpy(S0), cal,
                                n_pivots=pivots)
    np.testing.assert_array_equal(w.numpy(), w_ref)
    np.testing.assert_array_equal(bits, bits_ref)
    n16 = int((bits == 16).sum())
    assert n16 == pivots * (1 if wl.alloc == "lagrange_row" else wl.d)
    assert bits.astype(np.int64).sum() == wl.nominal_bits * bits.size + 8 * n16


@pytest.mark.parametrize("horizon", [1, 7, 2048])
def test_runtime_lifetime_closed_form_equals_the_oracle_sum(horizon):
    ell = np.log(np.array([0.5, 0.9, 0.999, 0.99999, 1.0]))
    np.testing.assert_allclose(runtime.lifetime(ell, horizon), oracle.lifetime(ell, horizon), rtol=1e-12)
    gate = np.random.default_rng(0).uniform(0.3, 1.0, size=(9, 4, 3, 5)).astype(np.float32)
    np.testing.assert_allclose(runtime.mean_log_retention(gate), oracle.mean_log_retention(gate), rtol=1e-15)
    np.testing.assert_allclose(runtime.mean_log_retention(torch.from_numpy(gate)),
                               oracle.mean_log_retention(gate), rtol=1e-15)


def test_lifetime_weights_are_bit_identical_to_the_oracles():
    """The runtime's lifetime weights L_u (App. A.3) equal the oracle's bit for bit over gates
    from 0 to 1 (both sum the series term by term), so the lifetime-weighted costs J the two
    allocators compare are the same numbers."""
    import oracle
    rng = np.random.default_rng(11)
    g = np.concatenate([[1.0, 0.999, 0.9, 1e-30], rng.uniform(0.0, 1.0, 4000), 1.0 - rng.exponential(1e-3, 96)])
    ell = np.log(np.clip(g, 1e-30, 1.0))
    np.testing.assert_array_equal(runtime.lifetime(ell), oracle.lifetime(ell))
