"""Pins of the oracle's gated Delta-rule recurrence against what STEPQuant §2.1, §3.1 and
App. A/B fix: the affine unrolling, the Delta-feedback contraction identity, the row-confined
read-error identity, linearity in the carried error, and closed-form special cases."""
import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(1234)


def _inputs(dk, dv, T, channel=False, rng=RNG):
    S0 = rng.normal(size=(dk, dv))
    steps = []
    for _ in range(T):
        q = rng.normal(size=dk); q /= np.linalg.norm(q)
        k = rng.normal(size=dk); k /= np.linalg.norm(k)
        v = rng.normal(size=dv)
        beta = float(1 / (1 + np.exp(-rng.normal())))
        g = rng.uniform(0.8, 1.0, size=dk) if channel else float(rng.uniform(0.8, 1.0))
        steps.append((q, k, v, beta, g))
    return S0, steps


def _A(k, beta, g):
    dk = len(k)
    D = np.diag(np.broadcast_to(np.asarray(g, dtype=float), (dk,)))
    return (np.eye(dk) - beta * np.outer(k, k)) @ D


@pytest.mark.parametrize("channel", [False, True])
def test_recurrence_matches_affine_unrolling(channel):
    """S_T = Phi_{T,0} S_0 + sum_r Phi_{T,r} B_r with Phi_{t,r} = A_t ... A_{r+1} (§2.1, App. A.2)."""
    dk, dv, T = 12, 9, 7
    S0, steps = _inputs(dk, dv, T, channel)
    S = S0.copy()
    outs = []
    for (q, k, v, beta, g) in steps:
        S, o = oracle.delta_update(S, q, k, v, beta, g)
        outs.append(o)
    As = [_A(k, beta, g) for (q, k, v, beta, g) in steps]
    Bs = [beta * np.outer(k, v) for (q, k, v, beta, g) in steps]

    def phi(t, r):  # A_t ... A_{r+1}, 1-based step indices
        P = np.eye(dk)
        for s in range(r + 1, t + 1):
            P = As[s - 1] @ P
        return P

    for t in range(1, T + 1):
        St = phi(t, 0) @ S0 + sum(phi(t, r) @ Bs[r - 1] for r in range(1, t + 1))
        if t == T:
            np.testing.assert_allclose(S, St, rtol=1e-12, atol=1e-12)
        q = steps[t - 1][0]
        np.testing.assert_allclose(outs[t - 1], St.T @ q, rtol=1e-11, atol=1e-12)


def test_delta_feedback_contraction_identity():
    """||a (I - b k k^T) E||_F^2 = a^2 [||E||^2 - b (2 - b ||k||^2) ||k^T E||^2] (App. B.1)."""
    rng = np.random.default_rng(7)
    for _ in range(20):
        dk, dv = 16, 11
        E = rng.normal(size=(dk, dv))
        k = rng.normal(size=dk) * rng.uniform(0.2, 1.5)
        a = rng.uniform(0.5, 1.0)
        b = rng.uniform(0.0, 1.0)
        X, _ = oracle.delta_update(E, np.zeros(dk), k, np.zeros(dv), b, a)
        lhs = np.sum(X * X)
        kE = k @ E
        rhs = a * a * (np.sum(E * E) - b * (2 - b * (k @ k)) * (kE @ kE))
        assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(rhs))


def test_row_confined_read_error_is_g_squared():
    """A unit perturbation confined to key row i changes the next read by exactly
    g_i^2 in squared norm, g = A^T q (App. B.3); g_i = d_i [q_i - beta k_i (k.q)] (App. C.1)."""
    rng = np.random.default_rng(11)
    dk, dv = 10, 7
    S = rng.normal(size=(dk, dv))
    q = rng.normal(size=dk); k = rng.normal(size=dk); k /= np.linalg.norm(k)
    v = rng.normal(size=dv)
    beta = 0.6
    d = rng.uniform(0.7, 1.0, size=dk)
    _, o_ref = oracle.delta_update(S, q, k, v, beta, d)
    g_closed = d * (q - beta * k * (k @ q))
    g_matrix = _A(k, beta, d).T @ q
    np.testing.assert_allclose(g_closed, g_matrix, rtol=1e-13, atol=1e-14)
    for i in range(dk):
        e = rng.normal(size=dv); e /= np.linalg.norm(e)
        E = np.zeros((dk, dv)); E[i] = e
        _, o = oracle.delta_update(S + E, q, k, v, beta, d)
        assert abs(np.sum((o - o_ref) ** 2) - g_matrix[i] ** 2) <= 1e-12


def test_carried_error_propagates_linearly():
    """(S + E)' - S' = A_t E, so the read error is E^T A_t^T q_t (Prop. 1, §3.1)."""
    rng = np.random.default_rng(5)
    dk, dv = 9, 13
    S = rng.normal(size=(dk, dv)); E = 1e-3 * rng.normal(size=(dk, dv))
    q = rng.normal(size=dk); k = rng.normal(size=dk); k /= np.linalg.norm(k)
    v = rng.normal(size=dv); beta = 0.37; g = 0.93
    X1, o1 = oracle.delta_update(S + E, q, k, v, beta, g)
    X0, o0 = oracle.delta_update(S, q, k, v, beta, g)
    A = _A(k, beta, g)
    np.testing.assert_allclose(X1 - X0, A @ E, rtol=1e-9, atol=1e-15)
    np.testing.assert_allclose(o1 - o0, E.T @ A.T @ q, rtol=1e-9, atol=1e-15)


def test_beta_zero_unit_gate_keeps_state():
    rng = np.random.default_rng(3)
    S = rng.normal(size=(8, 8)); q = rng.normal(size=8); k = rng.normal(size=8); v = rng.normal(size=8)
    X, o = oracle.delta_update(S, q, k, v, 0.0, 1.0)
    np.testing.assert_array_equal(X, S)
    np.testing.assert_allclose(o, S.T @ q, rtol=1e-14)


def test_unit_beta_unit_key_overwrites_association():
    """With g = 1, beta = 1 and ||k|| = 1 the Delta rule stores v exactly: S'^T k = v."""
    rng = np.random.default_rng(4)
    S = rng.normal(size=(16, 12)); k = rng.normal(size=16); k /= np.linalg.norm(k)
    v = rng.normal(size=12)
    X, _ = oracle.delta_update(S, np.zeros(16), k, v, 1.0, 1.0)
    np.testing.assert_allclose(X.T @ k, v, rtol=1e-12, atol=1e-12)


def test_scalar_gate_equals_uniform_channel_gate():
    rng = np.random.default_rng(6)
    S = rng.normal(size=(8, 8)); q = rng.normal(size=8); k = rng.normal(size=8); v = rng.normal(size=8)
    X1, o1 = oracle.delta_update(S, q, k, v, 0.4, 0.9)
    X2, o2 = oracle.delta_update(S, q, k, v, 0.4, np.full(8, 0.9))
    np.testing.assert_array_equal(X1, X2)
    np.testing.assert_array_equal(o1, o2)
