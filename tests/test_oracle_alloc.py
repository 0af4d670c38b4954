"""Pins of the oracle's lifetime-aware bit allocation (STEPQuant §3.2, App. C.2): the
multiple-choice DP against brute force, the Lagrangian allocation against the breakpoint
solutions of min_b J_u(b) + lambda b, exact budgets, the repair move, and lifetime monotonicity;
and of the calibration statistics (App. A.3, B.3, C.1)."""
import itertools

import numpy as np
import pytest

import oracle
from recurrent_state_quantization_gated_b200 import synth


def _brute(J, cand, budget):
    n, nc = J.shape
    best, arg = None, None
    for ks in itertools.product(range(nc), repeat=n):          # lexicographic order
        if sum(cand[k] for k in ks) != budget:
            continue
        cost = sum(J[u, k] for u, k in enumerate(ks))
        if best is None or cost < best:
            best, arg = cost, ks
    return best, None if arg is None else np.array([cand[k] for k in arg], dtype=np.uint8)


@pytest.mark.parametrize("seed", range(6))
def test_dp_equals_brute_force(seed):
    rng = np.random.default_rng(seed)
    cand = [4, 6, 8] if seed % 2 else [2, 4, 6, 8]
    n = 7 if len(cand) == 3 else 6
    J = rng.exponential(size=(n, len(cand))) * rng.exponential(size=(n, 1))
    for mean_bits in (cand[0], 5, 6, cand[-1]):
        budget = n * mean_bits
        cost, ref = _brute(J, cand, budget)
        if ref is None:                                   # no assignment reaches this budget
            with pytest.raises(ValueError):
                oracle.allocate_bits(J, cand, budget, mode=1)
            continue
        got = oracle.allocate_bits(J, cand, budget, mode=1)
        assert int(got.astype(int).sum()) == budget
        got_cost = sum(J[u, cand.index(int(b))] for u, b in enumerate(got))
        assert abs(got_cost - cost) <= 1e-12 * cost


def test_dp_tie_break_is_lexicographic_on_exact_costs():
    """With integer objectives every sum is exact; among equal optima the DP returns the
    lexicographically smallest assignment (brute force in lexicographic order keeps the first)."""
    rng = np.random.default_rng(42)
    cand = [4, 6, 8]
    for _ in range(20):
        J = rng.integers(0, 4, size=(6, 3)).astype(np.float64)
        cost, ref = _brute(J, cand, 36)
        np.testing.assert_array_equal(oracle.allocate_bits(J, cand, 36, mode=1), ref)


def test_dp_infeasible_budget_raises():
    with pytest.raises(ValueError):
        oracle.allocate_bits(np.ones((3, 3)), [4, 6, 8], 3 * 4 + 1, mode=1)


def _decreasing_convex_J(rng, n, cand):
    """Per-unit objectives that fall with the width: L_u * d(b) with d ~ 4^(-b) noise."""
    L = rng.exponential(size=(n, 1)) * 10
    d = np.array([4.0 ** (-b) for b in cand])[None, :] * rng.uniform(0.5, 2.0, size=(n, len(cand)))
    d = np.sort(d, axis=1)[:, ::-1]
    return L * d


@pytest.mark.parametrize("cand", [[4, 6, 8], [2, 4, 6, 8], [2, 4, 8]])
def test_lagrange_matches_breakpoint_solutions(cand):
    rng = np.random.default_rng(len(cand))
    n = 40
    J = _decreasing_convex_J(rng, n, cand)
    c = np.array(cand, dtype=np.float64)
    checked = 0
    for lam in np.exp(np.linspace(-25, 2, 200)):
        vals = J + lam * c[None, :]
        srt = np.sort(vals, axis=1)
        if np.any(srt[:, 1] - srt[:, 0] < 1e-9 * np.abs(srt[:, 0])):
            continue                                  # skip lambdas with a tie
        sol = c[np.argmin(vals, axis=1)].astype(np.uint8)
        budget = int(sol.astype(int).sum())
        got = oracle.allocate_bits(J, cand, budget, mode=0)
        np.testing.assert_array_equal(got, sol)
        checked += 1
    assert checked > 20


@pytest.mark.parametrize("cand,mean_bits", [([4, 6, 8], 6), ([2, 4, 8], 4), ([2, 4, 6, 8], 4), ([4, 6, 8], 5)])
def test_lagrange_meets_budget_exactly(cand, mean_bits):
    rng = np.random.default_rng(mean_bits)
    for n in (1, 2, 17, 300):
        if (n * mean_bits) % 2:                          # even widths cannot reach an odd budget
            with pytest.raises(ValueError):
                oracle.allocate_bits(_decreasing_convex_J(rng, n, cand), cand, n * mean_bits, mode=0)
            continue
        J = _decreasing_convex_J(rng, n, cand)
        got = oracle.allocate_bits(J, cand, n * mean_bits, mode=0)
        assert int(got.astype(int).sum()) == n * mean_bits
        assert set(np.unique(got)).issubset(set(cand))


def test_lagrange_repair_takes_the_cheapest_exact_move_from_the_hull_state():
    """Every unit's middle width lies above the chord of its two ends, so it is off the lower
    hull and the hull moves are 4 -> 8 only, taken steepest (J_4 - J_8) first. With a budget of
    4n + 4m + 2 bits the greedy phase stops with the m steepest units at 8 bits and 2 bits left
    over, a state known here without the oracle. The repair must then be the cheapest move to the
    exact budget among single changes (a unit 4 -> 6) and (up, down) pairs (4 -> 8 with
    8 -> 6), found by enumerating every such change of that state; over the seeds both kinds win."""
    cand = [4, 6, 8]
    n, m = 10, 4
    kinds = set()
    for seed in range(12):
        rng = np.random.default_rng(100 + seed)
        J4 = rng.uniform(5, 10, n)
        G = rng.uniform(1, 4, n)
        J8 = J4 - G
        J6 = (J4 + J8) / 2 + rng.exponential(0.15, n) * G        # above the chord: off the hull
        J = np.stack([J4, J6, J8], axis=1)
        budget = 4 * n + 4 * m + 2
        before = np.full(n, 4)
        before[np.argsort(-G)[:m]] = 8
        cost = lambda a: sum(J[u, cand.index(int(b))] for u, b in enumerate(a))
        best, arg, kind = None, None, None
        for u in range(n):                                        # single changes
            for bu in cand:
                t = before.copy(); t[u] = bu
                if t.sum() == budget and (best is None or cost(t) < best):
                    best, arg, kind = cost(t), t, "single"
        for u in range(n):                                        # (up, down) pairs
            for v in range(n):
                if u == v:
                    continue
                for bu in cand:
                    for bv in cand:
                        t = before.copy(); t[u] = bu; t[v] = bv
                        if bu > before[u] and bv < before[v] and t.sum() == budget and cost(t) < best:
                            best, arg, kind = cost(t), t, "pair"
        np.testing.assert_array_equal(oracle.allocate_bits(J, cand, budget, mode=0), arg)
        kinds.add(kind)
    assert kinds == {"single", "pair"}


def test_longer_lived_units_never_get_fewer_bits():
    rng = np.random.default_rng(9)
    cand = [4, 6, 8]
    groups, per = 8, 6
    d = np.sort(rng.exponential(size=(groups, 3)) * np.array([16.0, 1.0, 1 / 16]), axis=1)[:, ::-1]
    d = np.repeat(d, per, axis=0)
    gate = rng.uniform(0.5, 0.999, size=groups * per)
    J = oracle.objective(d, np.log(gate))
    for mode in (0, 1):
        bits = oracle.allocate_bits(J, cand, groups * per * 6, mode=mode)
        for g0 in range(groups):
            sl = slice(g0 * per, (g0 + 1) * per)
            order = np.argsort(gate[sl])
            assert np.all(np.diff(bits[sl][order].astype(int)) >= 0)


def test_row_impact_matches_explicit_transition():
    """omega_i = mean (A_t^T q_t)_i^2 with A_t = (I - beta k k^T) D_t built as a matrix;
    w_i = omega_i^(1/8) normalised to mean 1 per head (App. B.3)."""
    wl = synth.workload(2, B=3, H=2, d=64)
    cal = synth.calib_tokens(wl)
    w = oracle.row_impact(cal)
    T, B, H, d = cal["q"].shape
    for h in range(H):
        om = np.zeros(d)
        for t in range(T):
            for b in range(B):
                q = synth.bf16_bits_to_f32(cal["q"][t, b, h]).astype(np.float64)
                k = synth.bf16_bits_to_f32(cal["k"][t, b, h]).astype(np.float64)
                A = (np.eye(d) - cal["beta"][t, b, h] * np.outer(k, k)) @ np.diag(cal["gate"][t, b, h].astype(np.float64))
                om += (A.T @ q) ** 2
        om /= T * B
        om = np.maximum(om, 1e-12 * om.max())
        ref = om ** 0.125
        np.testing.assert_allclose(w[h], ref / ref.mean(), rtol=1e-6)


def test_distortion_definitions():
    """Eq. 17 and Eq. 18: d_head = (1/d_k) sum_i w_i^2 d_row_i; the MSE falls with the width;
    d_row equals the per-row MSE of fit -> pack -> unpack."""
    S = synth.random_tile_state(3, 2, 64, seed=30)
    w = synth.random_weights(2, 64, seed=31)
    prev = None
    for b in (2, 4, 6, 8):
        dr, dh = oracle.calib_distortion(S, w, b)
        np.testing.assert_allclose(dh, (w.astype(np.float64) ** 2 * dr).mean(axis=1), rtol=1e-12)
        if prev is not None:
            assert np.all(dh < prev)
        prev = dh
        if b == 6:
            bits = np.full(64, 6, dtype=np.uint8)
            acc = np.zeros(64)
            for s in range(3):
                X = S[s, 1]
                r, c = oracle.fit_tile(X, w[1], bits)
                Xh = oracle.unpack_tile(oracle.pack_tile(X, bits, r, c), bits, r, c, 64)
                acc += ((Xh.astype(np.float64) - X) ** 2).sum(axis=1)
            np.testing.assert_allclose(dr[1], acc / (3 * 64), rtol=1e-12)


def test_row_impact_floors_a_channel_that_no_query_or_key_reaches():
    """A key channel whose query and key entries are zero in every step has omega_i = 0; the
    floor 1e-12 max_i omega_i keeps its impact factor positive (App. B.3 keeps the numerical
    floor), so r_i = m_i / w_i stays finite."""
    wl = synth.workload(2, B=2, H=2, d=64)
    cal = synth.calib_tokens(wl)
    cal["q"][..., 0, 5] = 0
    cal["k"][..., 0, 5] = 0
    w = oracle.row_impact(cal)
    T, B, H, d = cal["q"].shape
    om = np.zeros(d)
    for t in range(T):
        for b in range(B):
            q = synth.bf16_bits_to_f32(cal["q"][t, b, 0]).astype(np.float64)
            k = synth.bf16_bits_to_f32(cal["k"][t, b, 0]).astype(np.float64)
            A = (np.eye(d) - cal["beta"][t, b, 0] * np.outer(k, k)) @ np.diag(
                np.broadcast_to(cal["gate"][t, b, 0], (d,)).astype(np.float64))
            om += (A.T @ q) ** 2
    om /= T * B
    assert om[5] == 0.0
    ref = np.maximum(om, 1e-12 * om.max()) ** 0.125
    np.testing.assert_allclose(w[0], ref / ref.mean(), rtol=1e-6)
    assert 0.0 < w[0, 5] < w[0].max() * 0.1


@pytest.mark.parametrize("g", [0.5, 0.9, 0.999, 1.0])
def test_lifetime_is_the_squared_error_a_decaying_unit_keeps(g):
    """App. A.3: L_u sums exp(2 j ell_u) over the horizon. Run the oracle's own recurrence with
    beta = 0 (pure retention) on an error injected once into one key row, and add up the squared
    error norm over the horizon: the total per unit injected is L_u at ell = log g."""
    horizon, dk, dv = 40, 6, 5
    rng = np.random.default_rng(11)
    E = np.zeros((dk, dv))
    E[2] = rng.normal(size=dv)
    e0 = float((E ** 2).sum())
    gate = np.full(dk, 0.3)
    gate[2] = g
    zero_v = np.zeros(dv)
    total = 0.0
    for _ in range(horizon):
        total += float((E ** 2).sum())
        E, _ = oracle.delta_update(E, rng.normal(size=dk), rng.normal(size=dk), zero_v, 0.0, gate)
    L = oracle.lifetime(np.log(g), horizon=horizon)
    np.testing.assert_allclose(total / e0, L, rtol=1e-12)
    if g == 1.0:
        assert L == horizon


def test_mean_log_retention_is_the_log_of_the_geometric_mean_gate():
    """ell_u = E_cal[log r_{t,u}]: a unit whose gate alternates between a and b over the stream
    retains exp(j ell) = (a b)^(j/2) over an even number j of steps, as §3.2's product approximation
    states; head gates give one value per head, channel gates one per key channel."""
    a, b = 0.8, 0.98
    T, B, H = 6, 3, 2
    gate = np.empty((T, B, H))
    gate[0::2], gate[1::2] = a, b
    gate[:, :, 1] = 0.9
    ell = oracle.mean_log_retention(gate)
    assert ell.shape == (H,)
    np.testing.assert_allclose(np.exp(4 * ell[0]), (a * b) ** 2, rtol=1e-14)
    np.testing.assert_allclose(np.exp(ell[1]), 0.9, rtol=1e-14)
    ch = np.broadcast_to(gate[..., None], (T, B, H, 4)).copy()
    ch[..., 3] = 0.5
    ell_c = oracle.mean_log_retention(ch)
    assert ell_c.shape == (H, 4)
    np.testing.assert_allclose(ell_c[:, :3], np.repeat(ell[:, None], 3, axis=1), rtol=1e-14)
    np.testing.assert_allclose(ell_c[:, 3], np.log(0.5), rtol=1e-14)
