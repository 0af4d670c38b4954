"""The benchmark's reference arm (the oracle on the host cores): each distinct step's inputs are
drawn once, whatever the number of steps, so that a long run's wall time is the oracle's."""
import os
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_draws_each_distinct_step_once(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    from recurrent_state_quantization_gated_b200 import synth
    calls = []
    real = synth.tokens

    def counted(wl, t, calib=False, seqs=None):
        if not calib:                                       # the decode inputs, not the calibration stream
            calls.append(t)
        return real(wl, t, calib=calib, seqs=seqs)

    monkeypatch.setattr(synth, "tokens", counted)
    wl = synth.workload(0)
    args = types.SimpleNamespace(steps=3 * wl.T + 5, warmup=2)
    ref = bench.run_reference(args, wl, budget_s=5.0)
    timed = [t for t in calls[1:]]                          # calls[0]: the rate probe
    assert len(timed) == len(set(timed)) == min(wl.T, args.steps + args.warmup)
    assert ref["value"] > 0 and f"{args.steps} timed steps" in ref["sample"]
