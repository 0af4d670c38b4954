"""Shared helpers of the GPU parity tests: moving seeded host inputs to the device and comparing
the CUDA library's results with the oracle's under the stated tolerances."""
import numpy as np

import oracle


def dev(a, dtype=None):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:                    # bf16 / fp16 bit patterns
        t = torch.from_numpy(a.view(np.int16)).cuda()
        return t.view(dtype) if dtype is not None else t
    return torch.from_numpy(a).cuda()


def host_half(t):
    """fp16 torch tensor -> uint16 bit patterns (numpy)."""
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def tokens_dev(tok):
    import torch
    return dict(q=dev(tok["q"], torch.bfloat16), k=dev(tok["k"], torch.bfloat16), v=dev(tok["v"], torch.bfloat16),
                beta=dev(tok["beta"]), gate=dev(tok["gate"]))


def tile_codes(packed, bits, d, B):
    """All codes [B][H][d][d] of a packed state (oracle's unpacker)."""
    head_off, bps = oracle.layout(bits, d)
    H = bits.shape[0]
    out = np.zeros((B, H, d, d), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            n = oracle.tile_bytes(bits[h], d)
            off = b * bps + head_off[h]
            out[b, h] = oracle.unpack_codes(packed[off:off + n], bits[h], d)
    return out


def with_pivots(bits, n, seed):
    """A copy of the bit map with n seeded key rows made FP16 pivots (width 16)."""
    rng = np.random.default_rng(seed)
    out = bits.copy()
    flat = out.reshape(-1)
    flat[rng.choice(flat.size, size=n, replace=False)] = 16
    return out


def half_ulps(a, b):
    """Distance in binary16 units in the last place between two arrays of positive fp16 bits."""
    return np.abs(a.astype(np.int32) - b.astype(np.int32))


def assert_outputs_close(o_gpu, o_ref, rtol=1e-3):
    """Per-tile relative L2 error and max-normalised elementwise error, both <= rtol."""
    og = o_gpu.reshape(-1, o_gpu.shape[-1]).astype(np.float64)
    orf = o_ref.reshape(-1, o_ref.shape[-1]).astype(np.float64)
    num = np.linalg.norm(og - orf, axis=1)
    den = np.maximum(np.linalg.norm(orf, axis=1), 1e-30)
    assert np.max(num / den) <= rtol, f"per-tile L2 rel err {np.max(num / den):.3e}"
    scale = np.maximum(np.abs(orf).max(axis=1, keepdims=True), 1e-30)
    assert np.max(np.abs(og - orf) / scale) <= rtol


def assert_codes_close(c_gpu, c_ref, max_frac=1e-3):
    diff = np.abs(c_gpu.astype(np.int64) - c_ref.astype(np.int64))
    assert diff.max() <= 1, f"codes differ by {diff.max()}"
    frac = (diff > 0).mean()
    assert frac <= max_frac, f"{frac:.2e} of codes differ by one step"
    return frac


# Mismatch rates of every decode comparison in this process, printed in the run's summary
# (tests/conftest.py) so that the measured rates sit beside the pass/fail record.
RATES = []


def oracle_updated_state(tok, bits, packed, r, c):
    """The oracle's updated state X of every tile before requantisation, fp32 [B][H][dk][dv]: the
    packed state reconstructed by the oracle, one gated Delta update in float64 (§2.1), rounded
    to fp32 -- the X that the oracle's own decode step fits and quantises (Table C2)."""
    from recurrent_state_quantization_gated_b200 import synth
    S = oracle.unpack_state(packed, bits, r, c)
    B, H, dk, dv = S.shape
    q = synth.bf16_bits_to_f32(tok["q"]).astype(np.float64)
    k = synth.bf16_bits_to_f32(tok["k"]).astype(np.float64)
    v = synth.bf16_bits_to_f32(tok["v"]).astype(np.float64)
    beta, gate = np.asarray(tok["beta"]), np.asarray(tok["gate"])
    X = np.empty_like(S)
    for b in range(B):
        for h in range(H):
            Xt, _ = oracle.delta_update(S[b, h], q[b, h], k[b, h], v[b, h], float(beta[b, h]), gate[b, h])
            X[b, h] = Xt.astype(np.float32)
    return X


def oracle_chunk_state(toks, bits, packed, r, c):
    """As ``oracle_updated_state`` for a prefill chunk: tokens with a leading token axis applied
    in float64 one after another without requantisation in between, the boundary state rounded
    to fp32 (App. F.1)."""
    from recurrent_state_quantization_gated_b200 import synth
    S = oracle.unpack_state(packed, bits, r, c).astype(np.float64)
    C = toks["q"].shape[0]
    B, H = S.shape[:2]
    for t in range(C):
        q = synth.bf16_bits_to_f32(toks["q"][t]).astype(np.float64)
        k = synth.bf16_bits_to_f32(toks["k"][t]).astype(np.float64)
        v = synth.bf16_bits_to_f32(toks["v"][t]).astype(np.float64)
        for b in range(B):
            for h in range(H):
                S[b, h], _ = oracle.delta_update(S[b, h], q[b, h], k[b, h], v[b, h], float(toks["beta"][t][b, h]),
                                                 toks["gate"][t][b, h])
    return S.astype(np.float32)


def quantise_with_scales(X, bits, r, c):
    """Codes [B][H][dk][dv] of X at the given binary16 scales r [B][H][dk], c [B][H][dv] (the
    oracle's quantiser; FP16 pivot rows give their binary16 bits)."""
    B, H = X.shape[:2]
    out = np.zeros(X.shape, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            out[b, h] = oracle.quantise_tile(X[b, h], bits[h], r[b, h], c[b, h])
    return out


def flip_explains(X, w, bits, r, j, c_want, tol=2e-3, max_flips=6):
    """Whether binary16 column scale c_want of column j is, within one binary16 ulp, the
    fixed-code least-squares update (App. C.1) of the oracle's codes at (r, c0) with some of the
    column's entries that lie within ``tol`` of a rounding boundary (X/(r 2^(8-b) c0) a
    half-integer) rounded to the other side: the codes such an entry gets depend on the last
    bits of X, and the update moves with them."""
    _, det = oracle.fit_columns(X, w, bits, r, detail=True)
    z0, c0 = det["z0"], det["c0"]
    rf = oracle.half_to_float(r).astype(np.float64) * 2.0 ** (8 - bits.astype(np.float64))
    qb = (1 << (bits.astype(np.int64) - 1)) - 1
    y = X[:, j].astype(np.float64) / rf / float(c0[j])
    alt = z0[:, j] + np.where(y >= z0[:, j], 1, -1)
    cand = np.flatnonzero((bits != 16) & (np.abs(np.abs(y) % 1.0 - 0.5) < tol) & (np.abs(alt) <= qb))
    if cand.size == 0 or cand.size > max_flips:
        return False
    for m in range(1, 1 << cand.size):
        z = z0.copy()
        rows = cand[[k for k in range(cand.size) if m >> k & 1]]
        z[rows, j] = alt[rows]
        c, _ = oracle.ls_columns(X, w, bits, r, z, c0)
        if abs(int(c[j]) - int(c_want)) <= 1:
            return True
    return False


def compare_decode(gpu, ref, bits, d, B, X_ref=None, max_frac=1e-3, label="", w=None):
    """Compares one decode step's results, (packed, r, c, o) as host arrays from both sides,
    started from the same packed state.

    o within 1e-3 relative; r within one binary16 ulp of the oracle's. A row scale one ulp apart
    moves that row's intermediate codes, which enter every column's least-squares sums of the
    tile (App. C.1), so the tile's column scales and codes may follow it. The reference for c and
    the codes is therefore the oracle's own result where the row scales agree and, in a tile
    where some row scale is one ulp apart (given ``X_ref`` and the row-impact factors ``w``
    [H][dk]), the oracle's column fit of X_ref at the GPU's row scales with X_ref quantised at
    (GPU's r, that c); without them the reference is the oracle's own result everywhere and
    the column scales of such tiles are not compared. Against that reference, at most 1 % of
    the column scales differ, or one, and each that differs by more than one binary16 ulp must
    be the least-squares update of the reference's intermediate codes with some entries of its
    column that sit on a rounding boundary rounded the other way (``flip_explains``: such an
    entry's code depends on the last bits of X, and in a column whose sums a few entries
    dominate it moves the update by several %, and with it the final codes of that column);
    without ``X_ref`` and ``w``, c within 10 % instead. Codes (every integer entry of every
    tile):

    * with ``X_ref`` (the oracle's updated state, ``oracle_updated_state``): X_ref quantised by
      the oracle's quantiser at the GPU's own scales must give the GPU's codes within one step,
      with at most ``max_frac`` of them one step off -- the bound that isolates the kernel's
      quantisation from the choice of scales -- and the entries whose row and column scales
      agree with the reference's must match the reference codes within one step, at most
      ``max_frac`` of them one step off;
    * without ``X_ref``: every integer entry within one step of the reference codes, at most
      ``max_frac`` of them and of the entries whose scales agree one step off.

    Returns a dict of rates (``raw_own``: the share of integer codes that differ from the
    oracle's own codes, reported only), also appended to ``RATES``."""
    p_g, r_g, c_g, o_g = gpu
    p_r, r_r, c_r, o_r = ref
    assert_outputs_close(o_g, o_r)
    assert half_ulps(r_g, r_r).max() <= 1, "row factors are continuous in X: one ulp at most"
    codes_g = tile_codes(p_g, bits, d, B)
    codes_r = tile_codes(p_r, bits, d, B)
    # The reference scales and codes: the oracle's own, or at the GPU's row scales where they differ.
    r_same = (r_g == r_r).all(axis=-1)
    r_ref, c_ref, codes_ref, held = r_r.copy(), c_r.copy(), codes_r.copy(), r_same.copy()   # held: c compared
    if X_ref is not None and w is not None:
        for b, h in zip(*np.nonzero(~r_same)):
            Xt = np.asarray(X_ref[b, h], dtype=np.float32)
            r_ref[b, h] = r_g[b, h]
            c_ref[b, h] = oracle.fit_columns(Xt, w[h], bits[h], r_g[b, h])
            codes_ref[b, h] = oracle.quantise_tile(Xt, bits[h], r_ref[b, h], c_ref[b, h])
        held[:] = True
    if X_ref is not None and w is not None:
        # every column scale more than one ulp from the reference is the least-squares update of
        # the reference's intermediate codes with some entries on a rounding boundary rounded
        # the other way
        for b, h, j in zip(*np.nonzero(half_ulps(c_g, c_ref) > 1)):
            assert flip_explains(np.asarray(X_ref[b, h], dtype=np.float32), w[h], bits[h], r_ref[b, h], j,
                                 c_g[b, h, j]), \
                f"column scale {j} of tile ({b}, {h}) is no least-squares update of the reference codes " \
                f"with boundary entries flipped"
    else:
        cf_g = c_g.view(np.float16).astype(np.float64)[held]
        cf_f = c_ref.view(np.float16).astype(np.float64)[held]
        if cf_g.size:
            gap = np.max(np.abs(cf_g / cf_f - 1))
            assert gap < 0.1, f"a column scale {gap:.1%} away from the reference column fit"
    moved = (c_g != c_ref)[held]
    c_mis = float(moved.mean()) if moved.size else 0.0
    # a flip is a per-column event: one column of a one-tile case is 1.6 % of its 64
    assert moved.sum() <= max(1, int(1e-2 * moved.size)), \
        f"{c_mis:.2e} of column scales differ from the reference column fit ({int(moved.sum())} columns)"
    piv = np.broadcast_to((bits == 16)[None, :, :, None], codes_g.shape)
    if piv.any():
        # FP16 pivot entries: binary16 values within one unit in the last place, or, for a value
        # far below the largest entry of its tile, within 2^-20 of that largest magnitude: the
        # entry is an fp32 sum of terms of the tile's magnitude (the update's pseudo-values and
        # keys), whose rounding, a few fp32 ulps of that magnitude, exceeds a binary16 ulp once
        # the value is that much smaller.
        vg_all = codes_g.astype(np.uint16).view(np.float16).astype(np.float64)
        vr_all = codes_r.astype(np.uint16).view(np.float16).astype(np.float64)
        S_r = oracle.unpack_state(p_r, bits, r_r, c_r)
        tile_max = np.abs(S_r).max(axis=(-2, -1), keepdims=True)
        vg, vr = vg_all[piv], vr_all[piv]
        floor = np.broadcast_to(tile_max, codes_g.shape)[piv] * 2.0 ** -20
        ulp = np.spacing(np.maximum(np.abs(vg), np.abs(vr)).astype(np.float16)).astype(np.float64)
        assert (np.abs(vg - vr) <= np.maximum(ulp, floor)).all(), "pivot values differ by more than one binary16 ulp"
    integer = ~piv
    diff = np.where(piv, 0, np.abs(codes_g.astype(np.int64) - codes_ref))
    same = (r_g == r_ref)[..., :, None] & (c_g == c_ref)[..., None, :] & integer
    if X_ref is None:
        assert diff.max() <= 1, f"codes differ by {diff.max()}"
    else:
        # Where a column scale differs from the reference, the final codes of that column follow
        # it: held to X_ref quantised at the GPU's own scales below.
        assert diff[same].max(initial=0) <= 1, f"codes with equal scales differ by {diff[same].max(initial=0)}"
    own = np.where(piv, 0, np.abs(codes_g.astype(np.int64) - codes_r))
    rates = dict(label=label, equal_scales=None, raw=None, r_mismatch=float((r_g != r_r).mean()),
                 c_mismatch=float((c_g != c_r).mean()), at_gpu_scales=None, n_codes=int(integer.sum()),
                 raw_own=float((own[integer] > 0).mean() if integer.any() else 0.0))
    if X_ref is not None:
        codes_x = quantise_with_scales(X_ref, bits, r_g, c_g)
        dx = np.abs(codes_g.astype(np.int64) - codes_x)[integer]
        assert dx.max(initial=0) <= 1, f"codes at the GPU's scales differ by {dx.max()}"
        fx = (dx > 0).mean() if dx.size else 0.0
        rates["at_gpu_scales"] = float(fx)
        assert fx <= max_frac, f"{fx:.2e} of all integer codes differ from the oracle's X at the GPU's scales"
    frac_same = (diff[same] > 0).mean() if same.any() else 0.0
    rates["equal_scales"] = float(frac_same)
    rates["raw"] = float((diff[integer] > 0).mean() if integer.any() else 0.0)
    assert frac_same <= max_frac, f"{frac_same:.2e} of codes with equal scales differ by one step"
    if X_ref is None:   # with X_ref every code is bounded at the GPU's own scales instead
        assert rates["raw"] <= max_frac, f"{rates['raw']:.2e} of the integer codes differ from the reference codes"
    RATES.append(rates)
    return rates
