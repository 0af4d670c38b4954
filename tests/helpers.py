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


def compare_decode(gpu, ref, bits, d, B, max_frac=1e-3):
    """Compares one decode step's results, (packed, r, c, o) as host arrays from both sides,
    started from the same packed state.

    o within 1e-3 relative; r within one binary16 ulp; c equal except where an entry of the
    updated state sits on a rounding boundary of the intermediate codes, which moves the
    least-squares column update by a few ulps (at most 10% apart, on under 1% of columns).
    Codes: never more than one step apart; where the row and column scales of both sides
    agree, at most ``max_frac`` of them differ. Returns the mismatch rates (codes where the
    scales agree, r, c, all codes)."""
    p_g, r_g, c_g, o_g = gpu
    p_r, r_r, c_r, o_r = ref
    assert_outputs_close(o_g, o_r)
    assert half_ulps(r_g, r_r).max() <= 1, "row factors are continuous in X: one ulp at most"
    cf_g = c_g.view(np.float16).astype(np.float64)
    cf_r = c_r.view(np.float16).astype(np.float64)
    assert np.max(np.abs(cf_g / cf_r - 1)) < 0.1
    c_mis = (c_g != c_r).mean()
    assert c_mis < 1e-2, f"{c_mis:.2e} of column scales differ"
    codes_g = tile_codes(p_g, bits, d, B)
    codes_r = tile_codes(p_r, bits, d, B)
    piv = np.broadcast_to((bits == 16)[None, :, :, None], codes_g.shape)
    if piv.any():   # FP16 pivot entries: binary16 values within one unit in the last place
        vg = codes_g[piv].astype(np.uint16).view(np.float16).astype(np.float64)
        vr = codes_r[piv].astype(np.uint16).view(np.float16).astype(np.float64)
        ulp = np.spacing(np.maximum(np.abs(vg), np.abs(vr)).astype(np.float16)).astype(np.float64)
        assert (np.abs(vg - vr) <= ulp).all(), "pivot values differ by more than one binary16 ulp"
    diff = np.where(piv, 0, np.abs(codes_g.astype(np.int64) - codes_r))
    assert diff.max() <= 1, f"codes differ by {diff.max()}"
    same = (r_g == r_r)[..., :, None] & (c_g == c_r)[..., None, :] & ~piv
    frac = (diff[same] > 0).mean() if same.any() else 0.0
    assert frac <= max_frac, f"{frac:.2e} of codes with equal scales differ by one step"
    return frac, (r_g != r_r).mean(), c_mis, (diff > 0).mean()
