"""The chunked WY/UT rearrangement that the tensor-core prefill kernel evaluates, written out in
float64 and checked against the oracle's per-token recurrence (§2.1: S_t = g_t S_{t-1} + k_t u_t^T,
u_t = beta_t (v_t - g_t S_{t-1}^T k_t), o_t = S_t^T q_t). With gamma_t the running gate product:
  L_ts = beta_t (gamma_t/gamma_s) k_t.k_s (s < t),  T = (I + L)^-1,
  U = T diag(beta) V - T diag(beta gamma) K S0,
  O = diag(gamma) Q S0 + (gamma_t/gamma_s on and below the diagonal, o Q K^T) U,
  S_C = gamma_C S0 + (diag(gamma_C/gamma) K)^T U.
The gate ratios are taken as 2^(l_t - l_s) from the running log2 of the gates (l_t = sum of
log2 g), as the kernel forms them; the 16 x 16 block inversion of T is checked against a plain
inverse."""
import numpy as np
import pytest

import oracle
from recurrent_state_quantization_gated_b200 import synth


def _block_inverse(L):
    """(I + L)^-1 for strictly lower L, 64 x 64: 16 x 16 diagonal blocks by substitution, then
    T_ij = -sum_{k=j}^{i-1} G_ik T_kj with G_ik = T_ii L_ik, by distance i - j."""
    n = L.shape[0]
    T = np.zeros_like(L)
    for o in range(0, n, 16):
        for c in range(16):
            x = np.zeros(16)
            x[c] = 1.0
            for r in range(c + 1, 16):
                x[r] = -L[o + r, o:o + r] @ x[:r]
            T[o:o + 16, o + c] = x
    nb = n // 16
    blk = lambda M, i, j: M[16 * i:16 * i + 16, 16 * j:16 * j + 16]
    G = {(i, k): blk(T, i, i) @ blk(L, i, k) for i in range(nb) for k in range(i)}
    for lv in range(1, nb):
        for j in range(nb - lv):
            i = j + lv
            T[16 * i:16 * i + 16, 16 * j:16 * j + 16] = -sum(G[i, k] @ blk(T, k, j) for k in range(j, i))
    return T


def _chunk(wl, C, gates=None):
    steps = [synth.tokens(wl, t) for t in range(C)]
    toks = {n: np.ascontiguousarray(np.stack([s[n] for s in steps])) for n in steps[0]}
    if gates is not None:
        toks["gate"] = gates.astype(np.float32)
    return toks


@pytest.mark.parametrize("C,gate_lo", [(64, None), (17, None), (1, None), (64, 0.2)])
def test_wy_form_equals_the_recurrence(C, gate_lo):
    wl = synth.workload(1, B=1, H=2, d=64, seed=C)
    S0 = synth.initial_state(wl).astype(np.float64)
    gates = None
    if gate_lo is not None:
        gates = np.random.default_rng(1).uniform(gate_lo, 1.0, (C, wl.B, wl.H))
        gates[C // 2, 0, 1] = 0.0                      # an exact zero gate (counted as 2^-64)
    toks = _chunk(wl, C, gates)
    for h in range(wl.H):
        K = synth.bf16_bits_to_f32(toks["k"][:, 0, h]).astype(np.float64)
        Q = synth.bf16_bits_to_f32(toks["q"][:, 0, h]).astype(np.float64)
        V = synth.bf16_bits_to_f32(toks["v"][:, 0, h]).astype(np.float64)
        beta = toks["beta"][:, 0, h].astype(np.float64)
        g = np.maximum(toks["gate"][:, 0, h].astype(np.float64), 2.0 ** -64)
        # the recurrence, token by token (the oracle's delta update)
        S, O_ref = S0[0, h], np.zeros((C, wl.d))
        for t in range(C):
            S, O_ref[t] = oracle.delta_update(S, Q[t], K[t], V[t], beta[t], g[t])
        # the chunk form, padded to 64 tokens with k = q = v = 0, beta = 0, g = 1
        n = 64
        pad = lambda A, fill=0.0: np.concatenate([A, np.full((n - C,) + A.shape[1:], fill)])
        Kp, Qp, Vp, bp, gp = pad(K), pad(Q), pad(V), pad(beta), pad(g, 1.0)
        l = np.cumsum(np.log2(gp))
        R = np.exp2(l[:, None] - l[None, :])
        gam = np.exp2(l)
        L = np.tril(bp[:, None] * R * (Kp @ Kp.T), -1)
        T = _block_inverse(L)
        np.testing.assert_allclose(T, np.linalg.inv(np.eye(n) + L), rtol=0, atol=1e-9)
        U = T @ np.diag(bp) @ Vp - T @ np.diag(bp * gam) @ Kp @ S0[0, h]
        O = np.diag(gam) @ Qp @ S0[0, h] + (np.tril(R) * (Qp @ Kp.T)) @ U
        SC = gam[-1] * S0[0, h] + (np.diag(gam[-1] / gam) @ Kp).T @ U
        scale = np.abs(O_ref).max()
        np.testing.assert_allclose(O[:C], O_ref, rtol=0, atol=1e-9 * scale)
        np.testing.assert_allclose(SC, S, rtol=0, atol=1e-9 * np.abs(S).max())


def _split_pair_products(A, B, l, blk=16):
    """M_ts = sum_i A_ti B_si 2^(l_ti - l_si) for s <= t, as plain products of scaled operands.
    Every factor stays at most 1 off the diagonal blocks: the pair (t-block a, s-block b < a)
    takes the reference r = l at the last token of block b, so A is scaled by 2^(l_t - r) <= 1 and
    B by 2^(r - l_s) <= 1. Inside a diagonal block the reference is the block's first token (B is
    scaled by 2^(r - l_s) >= 1, bounded by the decay over fewer than blk tokens)."""
    n = A.shape[0]
    M = np.zeros((n, n))
    for a in range(n // blk):
        ta = slice(a * blk, (a + 1) * blk)
        for b in range(a + 1):
            sb = slice(b * blk, (b + 1) * blk)
            r = l[b * blk + blk - 1] if b < a else l[a * blk]
            if b < a:
                assert (l[ta] - r <= 0).all() and (r - l[sb] <= 0).all()
            M[ta, sb] = (A[ta] * np.exp2(l[ta] - r)) @ (B[sb] * np.exp2(r - l[sb])).T
    return np.tril(M)


@pytest.mark.parametrize("C,gate_lo", [(64, None), (23, None), (64, 0.3)])
def test_channel_gate_wy_form_equals_the_recurrence(C, gate_lo):
    """The same rearrangement under channel gates (KDA: D_t = diag(g_t), one gate per key
    channel), as a tensor-core form for channel gates would evaluate it. With l_t the running
    log2 of the gate products per channel (a vector), and every pair ratio 2^(l_t - l_s) folded
    into the operands through a per-block reference (_split_pair_products):
      L_ts = beta_t sum_i k_ti k_si 2^(l_ti - l_si) (s < t),  T = (I + L)^-1,
      U = T diag(beta) V - T diag(beta) (K o 2^l) S0,
      O = (Q o 2^l) S0 + tril(sum_i q_ti k_si 2^(l_ti - l_si)) U,
      S_C = diag(2^(l_C)) S0 + (K o 2^(l_C - l))^T U.
    The operands scaled this way are no longer exact in bf16, unlike the scalar-gate form's K, Q."""
    wl = synth.workload(2, B=1, H=2, d=64, seed=C)
    S0 = synth.initial_state(wl).astype(np.float64)
    gates = None
    if gate_lo is not None:
        gates = np.random.default_rng(2).uniform(gate_lo, 1.0, (C, wl.B, wl.H, wl.d))
        gates[C // 3, 0, 1, 5] = 0.0                   # an exact zero gate (counted as 2^-64)
    toks = _chunk(wl, C, gates)
    for h in range(wl.H):
        K = synth.bf16_bits_to_f32(toks["k"][:, 0, h]).astype(np.float64)
        Q = synth.bf16_bits_to_f32(toks["q"][:, 0, h]).astype(np.float64)
        V = synth.bf16_bits_to_f32(toks["v"][:, 0, h]).astype(np.float64)
        beta = toks["beta"][:, 0, h].astype(np.float64)
        g = np.maximum(toks["gate"][:, 0, h].astype(np.float64), 2.0 ** -64)      # [C][d]
        S, O_ref = S0[0, h], np.zeros((C, wl.d))
        for t in range(C):
            S, O_ref[t] = oracle.delta_update(S, Q[t], K[t], V[t], beta[t], g[t])
        n = 64
        pad = lambda A, fill=0.0: np.concatenate([A, np.full((n - C,) + A.shape[1:], fill)])
        Kp, Qp, Vp, bp, gp = pad(K), pad(Q), pad(V), pad(beta), pad(g, 1.0)
        l = np.cumsum(np.log2(gp), axis=0)                                          # [n][d]
        # the pair products by their definition, for comparison with the split form
        direct = np.einsum("ti,si,tsi->ts", Kp, Kp, np.exp2(l[:, None, :] - l[None, :, :]))
        KK = _split_pair_products(Kp, Kp, l)
        np.testing.assert_allclose(np.tril(KK, -1), np.tril(direct, -1), rtol=0,
                                   atol=1e-12 * np.abs(direct).max())
        L = np.tril(bp[:, None] * KK, -1)
        T = _block_inverse(L)
        U = T @ (bp[:, None] * Vp) - T @ ((bp[:, None] * Kp * np.exp2(l)) @ S0[0, h])
        O = (Qp * np.exp2(l)) @ S0[0, h] + _split_pair_products(Qp, Kp, l) @ U
        SC = np.exp2(l[-1])[:, None] * S0[0, h] + (Kp * np.exp2(l[-1] - l)).T @ U
        np.testing.assert_allclose(O[:C], O_ref, rtol=0, atol=1e-9 * np.abs(O_ref).max())
        np.testing.assert_allclose(SC, S, rtol=0, atol=1e-9 * np.abs(S).max())
