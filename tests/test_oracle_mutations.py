"""Planted mistakes in the oracle, each of which some pin must catch.

The oracle is only as trustworthy as its pins. This test copies the oracle (its C source and
its Python wrapper), the pin tests and the input generators into a scratch tree, plants ONE
plausible mistake in the copy (a dropped term, a flipped sign, a transposed operand or index, a
changed rounding or tie-break, an off-by-one constant, a step taken in the wrong order), and runs
the pins against it. Every planted mistake must make at least one pin fail; the unmodified copy
must pass. The mistakes live only in the scratch copies, on the CPU; the oracle itself is never
changed. Each edit names text that occurs exactly once in the file it edits, so the list stays
in step with the source.

Where a plausible mistake gives the same results as the correct code on every input the method
can meet, it is not listed here (for example, sign-extending a code of -2^(b-1), which the
symmetric quantiser never writes).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parent.parent
TESTS = ROOT / "tests"
PKG = "recurrent_state_quantization_gated_b200"
SCRATCH = ROOT / "_build" / "oracle_mutants"
C_SRC = "oracle/stepq_oracle.c"
PY_SRC = "oracle/__init__.py"

# The pins: every oracle test module, and the chunk-form algebra checked against the oracle's
# per-token recurrence.
PIN_FILES = sorted(p.name for p in TESTS.glob("test_oracle_*.py") if p.name != Path(__file__).name)
PIN_FILES.append("test_chunk_algebra.py")


@dataclass(frozen=True)
class Mutant:
    name: str
    path: str
    edits: tuple            # ((old, new), ...), each old text occurring once in path


def _m(name, path, *edits):
    return Mutant(name, path, tuple(edits))


MUTANTS = [
    # gated Delta rule (§2.1): X = D S + beta k (v - (D S)^T k)^T, o = X^T q
    _m("gate dropped from the decay", C_SRC,
       ("X[i * dv + j] = gate[i] * S[i * dv + j];", "X[i * dv + j] = S[i * dv + j];")),
    _m("delta sign flipped", C_SRC,
       ("k[i] * (beta * (v[j] - p[j]))", "k[i] * (beta * (v[j] + p[j]))")),
    _m("beta dropped from the write", C_SRC,
       ("k[i] * (beta * (v[j] - p[j]))", "k[i] * (v[j] - p[j])")),
    _m("prediction read from the ungated state", C_SRC,
       ("p[j] += k[i] * X[i * dv + j];", "p[j] += k[i] * S[i * dv + j];")),
    _m("prediction read through a transposed state", C_SRC,
       ("p[j] += k[i] * X[i * dv + j];", "p[j] += k[i] * X[j * dk + i];")),
    _m("readout taken before the update", C_SRC,
       ("acc += q[i] * X[i * dv + j];", "acc += q[i] * S[i * dv + j];")),
    _m("readout with the key instead of the query", C_SRC,
       ("acc += q[i] * X[i * dv + j];", "acc += k[i] * X[i * dv + j];")),
    _m("readout through a transposed state", C_SRC,
       ("acc += q[i] * X[i * dv + j];", "acc += q[i] * X[j * dk + i];")),
    _m("gate applied after the update instead of before it", C_SRC,
       ("X[i * dv + j] = gate[i] * S[i * dv + j];", "X[i * dv + j] = S[i * dv + j];"),
       ("X[i * dv + j] += k[i] * (beta * (v[j] - p[j]));",
        "X[i * dv + j] = gate[i] * (X[i * dv + j] + k[i] * (beta * (v[j] - p[j])));")),
    _m("channel gate replaced by its first entry", C_SRC,
       ("t->g[i] = gate_per_channel ? (double)gate[i] : (double)gate[0];", "t->g[i] = (double)gate[0];")),
    # quantiser and dequantiser (§2.2)
    _m("codes rounded toward zero", C_SRC,
       ("float n = rintf(t);", "float n = truncf(t);")),
    _m("negative codes clamped at -2^(b-1)", C_SRC,
       ("if (n < -qb) n = -qb;", "if (n < -qb - 1.0f) n = -qb - 1.0f;")),
    _m("quantiser rounds ties away from zero", C_SRC,
       ("float n = rintf(t);", "float n = roundf(t);")),
    _m("INT8 baseline rounds ties away from zero", C_SRC,
       ("float n = rintf(X[i * dv + j] * is);", "float n = roundf(X[i * dv + j] * is);")),
    _m("codebook step z dropped in the dequantiser", C_SRC,
       ("return rc * (float)(q * znorm_of(b));", "return rc * (float)q;")),
    # packed layout
    _m("4-bit nibbles in plain order", C_SRC,
       ("static const int pos[4] = {0, 2, 1, 3};", "static const int pos[4] = {0, 1, 2, 3};")),
    _m("6-bit planes swapped (pack and unpack agree)", C_SRC,
       ("uint8_t* lo_plane = row;\n        uint8_t* hi_plane = row + dv / 2;",
        "uint8_t* lo_plane = row + dv / 4;\n        uint8_t* hi_plane = row;"),
       ("get_bits(row, field_bit(j, 4), 4) | (get_bits(row + dv / 2, field_bit(j, 2), 2) << 4)",
        "get_bits(row + dv / 4, field_bit(j, 4), 4) | (get_bits(row, field_bit(j, 2), 2) << 4)")),
    _m("packed codes lose their sign bit", C_SRC,
       ("(unsigned)q[j] & ((1u << b) - 1u)", "(unsigned)q[j] & ((1u << (b - 1)) - 1u)")),
    _m("6-bit high plane joined one bit low", C_SRC,
       ("field_bit(j, 2), 2) << 4)", "field_bit(j, 2), 2) << 3)")),
    _m("rows laid out in reverse key order", C_SRC,
       ("        for (int i = 0; i < dk; ++i)\n            if (is_pivot(bits[i]) == pass) {",
        "        for (int i = dk - 1; i >= 0; --i)\n            if (is_pivot(bits[i]) == pass) {")),
    _m("pivot rows stored before the integer rows", C_SRC,
       ("if (is_pivot(bits[i]) == pass) {", "if (is_pivot(bits[i]) != pass) {")),
    _m("state unpack ignores the head offset", C_SRC,
       ("orc_unpack_tile(dk, dv, packed + b * bytes_per_seq + head_off[h], bits",
        "orc_unpack_tile(dk, dv, packed + b * bytes_per_seq, bits")),
    # binary16 conversions
    _m("scales truncated instead of rounded to nearest even", C_SRC,
       ("double sig = nearbyint(ldexp(m, 11)); /* 11 significant bits, ties to even    */",
        "double sig = floor(ldexp(m, 11));")),
    _m("pivot values overflow to infinity", C_SRC,
       ("if (x > HALF_MAX) return (uint16_t)(sign | 0x7BFFu);",
        "if (x > HALF_MAX) return (uint16_t)(sign | 0x7C00u);")),
    _m("binary16 subnormals decoded one exponent low", C_SRC,
       ("if (e == 0) v = ldexp((double)m, -24);", "if (e == 0) v = ldexp((double)m, -25);")),
    # key-row-aware dual-axis fit (§4.3, App. C.1)
    _m("row factor is a sum, not a mean", C_SRC,
       ("        m /= dv;\n", "")),
    _m("row factor takes the row maximum", C_SRC,
       ("for (int j = 0; j < dv; ++j) m += fabs((double)X[i * dv + j]);",
        "for (int j = 0; j < dv; ++j) m = fmax(m, fabs((double)X[i * dv + j]));")),
    _m("pivot rows join the shared column init as 8-bit rows", C_SRC,
       ("if (is_pivot(b)) continue;\n            float a = 1.0f", "if (is_pivot(b)) b = 8;\n            float a = 1.0f")),
    _m("row factor floor dropped", C_SRC,
       ("        if (m < HALF_MIN_NORMAL) m = HALF_MIN_NORMAL;\n", "")),
    _m("column init floor dropped", C_SRC,
       ("c0[j] = mx < (float)HALF_MIN_NORMAL ? (float)HALF_MIN_NORMAL : mx;", "c0[j] = mx;")),
    _m("row impact multiplies the row factor", C_SRC,
       ("r_out[i] = orc_scale_to_half(m / (double)w[i]);", "r_out[i] = orc_scale_to_half(m * (double)w[i]);")),
    _m("no-clip column init ignores the codebook step", C_SRC,
       ("float a = 1.0f / (rf[i] * (float)(znorm_of(b) * qmax_of(b)));",
        "float a = 1.0f / (rf[i] * (float)qmax_of(b));")),
    _m("least-squares weights not squared", C_SRC,
       ("double ww = (double)w[i] * (double)w[i];", "double ww = (double)w[i];")),
    _m("least-squares model drops the codebook step", C_SRC,
       ("double v = (double)orc_half_to_float(r[i]) * znorm_of(bits[i]) * z[i * dv + j];",
        "double v = (double)orc_half_to_float(r[i]) * z[i * dv + j];")),
    _m("least-squares update skipped", C_SRC,
       ("c_out[j] = orc_scale_to_half(c1);", "c_out[j] = orc_scale_to_half((double)cfall[j]);")),
    _m("zero-denominator column loses its start scale", C_SRC,
       ("double c1 = den > 0.0 ? num / den : (double)cfall[j];", "double c1 = den > 0.0 ? num / den : 0.0;")),
    _m("column fit ignores the given row scales", C_SRC,
       ("for (int i = 0; i < dk; ++i) rf[i] = orc_half_to_float(r[i]);", "for (int i = 0; i < dk; ++i) rf[i] = 1.0f;")),
    # the persistent decode step (Table C2) and the prefill boundary (App. F.1)
    _m("decode refits the previous state", C_SRC,
       ("    for (int e = 0; e < dk * dv; ++e) S32[e] = (float)t.X[e];\n"
        "    orc_fit_tile(dk, dv, S32, w, bits, r_out, c_out);",
        "    orc_fit_tile(dk, dv, S32, w, bits, r_out, c_out);")),
    _m("decode batch fits every head with the first head's impact", C_SRC,
       ("gate_per_channel, bits + (int64_t)h * dk, w + (int64_t)h * dk,", "gate_per_channel, bits + (int64_t)h * dk, w,")),
    _m("decode packs with the previous scales", C_SRC,
       ("orc_pack_tile(dk, dv, S32, bits, r_out, c_out, packed_out);",
        "orc_pack_tile(dk, dv, S32, bits, r_in, c_in, packed_out);")),
    _m("prefill chunk never advances its state", C_SRC,
       ("memcpy(t.S, t.X, sizeof(double) * dk * dv);            /* full precision in between */", "")),
    _m("prefill readouts all written to the first token's slot", C_SRC,
       ("o[tc * dv + j] = (float)t.o[j];\n            memcpy(t.S, t.X, sizeof(double) * dk * dv);            /* full precision in between */",
        "o[tl * dv + j] = (float)t.o[j];\n            memcpy(t.S, t.X, sizeof(double) * dk * dv);            /* full precision in between */")),
    _m("prefill boundary fit with the first head's impact", C_SRC,
       ("orc_fit_tile(dk, dv, S32, w + (int64_t)h * dk, bh,", "orc_fit_tile(dk, dv, S32, w, bh,")),
    # per-window 8-bit state and the INT8 baseline (§5.1)
    _m("window never advances its state", C_SRC,
       ("memcpy(t.S, t.X, sizeof(double) * dk * dv);            /* no quantisation inside the window */", "")),
    _m("window requantised after every token", C_SRC,
       ("memcpy(t.S, t.X, sizeof(double) * dk * dv);            /* no quantisation inside the window */",
        "for (int e = 0; e < dk * dv; ++e) S32[e] = (float)t.X[e];\n"
        "            orc_int8_quantise_tile(dk, dv, S32, codes_out + tl * dk * dv, s_out + tl * dk);\n"
        "            for (int i = 0; i < dk; ++i)\n"
        "                for (int j = 0; j < dv; ++j)\n"
        "                    t.S[i * dv + j] = (double)(orc_half_to_float(s_out[tl * dk + i]) *\n"
        "                                               (float)codes_out[(tl * dk + i) * dv + j]);")),
    _m("window reads the first tile's scales for every tile", C_SRC,
       ("float si = orc_half_to_float(s_in[tl * dk + i]);", "float si = orc_half_to_float(s_in[i]);")),
    _m("INT8 scale divides by 128", C_SRC,
       ("s[i] = orc_scale_to_half((double)mx / 127.0);", "s[i] = orc_scale_to_half((double)mx / 128.0);")),
    # calibration statistics (App. A.3, B.3)
    _m("row impact with the Delta feedback sign flipped", C_SRC,
       ("(orc_bf16_to_float(qq[i]) - (double)beta[tile]", "(orc_bf16_to_float(qq[i]) + (double)beta[tile]")),
    _m("row impact feedback with q.q in place of k.q", C_SRC,
       ("kq += (double)orc_bf16_to_float(kk[i]) * orc_bf16_to_float(qq[i]);",
        "kq += (double)orc_bf16_to_float(qq[i]) * orc_bf16_to_float(qq[i]);")),
    _m("row impact without the gate", C_SRC,
       ("double g = d * (orc_bf16_to_float(qq[i])", "double g = (orc_bf16_to_float(qq[i])")),
    _m("row impact fourth root instead of eighth", C_SRC,
       ("oh[i] = pow(oh[i], 0.125);", "oh[i] = pow(oh[i], 0.25);")),
    _m("row impact not normalised per head", C_SRC,
       ("(float)(mean > 0.0 ? oh[i] / mean : 1.0);", "(float)oh[i];")),
    _m("row impact floor dropped", C_SRC,
       ("if (oh[i] < 1e-12 * mx) oh[i] = 1e-12 * mx;", "")),
    _m("distortion fits every head with the first head's impact", C_SRC,
       ("const float* wh = w + (int64_t)h * dk;", "const float* wh = w;")),
    _m("head distortion weights not squared", C_SRC,
       ("dh += (double)wh[i] * (double)wh[i] * row;", "dh += (double)wh[i] * row;")),
    _m("row distortion not divided by the row length", C_SRC,
       ("d_row[(int64_t)h * dk + i] /= (double)B * dv;", "d_row[(int64_t)h * dk + i] /= (double)B;")),
    # allocation (§3.2, App. C.2)
    _m("DP budget relaxed to at most", C_SRC,
       ("G[(int64_t)n * W + s] = (s == 0) ? 0.0 : INFINITY;", "G[(int64_t)n * W + s] = 0.0;")),
    _m("DP ties go to the widest candidate", C_SRC,
       ("for (int kk = 0; kk < nc && chosen < 0; ++kk) {", "for (int kk = 0; kk < nc; ++kk) {")),
    _m("Lagrangian walks the upper hull", C_SRC,
       ("if (s1 >= s2) --m; else break;", "if (s1 <= s2) --m; else break;")),
    _m("Lagrangian takes the flattest move first", C_SRC,
       ("if (best < 0 || slope < best_slope) { best = u; best_slope = slope; }",
        "if (best < 0 || slope > best_slope) { best = u; best_slope = slope; }")),
    _m("repair pairs count the down move as up", C_SRC,
       ("if (down <= 0 || up - down != rem) continue;", "if (down <= 0 || up + down != rem) continue;")),
    _m("repair takes the first single move, not the cheapest", C_SRC,
       ("if (!found || dj < bdj) { found = 1; bdj = dj; bu = u; bku = kk; bv = -1; }",
        "if (!found) { found = 1; bdj = dj; bu = u; bku = kk; bv = -1; }")),
    _m("decode wrapper passes channel gates as head gates", PY_SRC,
       ("gpc = int(gate.ndim == 3)", "gpc = 0")),
    _m("prefill wrapper passes channel gates as head gates", PY_SRC,
       ("gpc = int(gate.ndim == 4)\n    head_off, bps = layout(bits, dv)", "gpc = 0\n    head_off, bps = layout(bits, dv)")),
    _m("row impact wrapper passes channel gates as head gates", PY_SRC,
       ("int(gate.ndim == 4), _p(q)", "0, _p(q)")),
    _m("lifetime sums the retention, not the squared error", PY_SRC,
       ("total += np.exp(2.0 * j * ell)", "total += np.exp(j * ell)")),
    _m("lifetime sum starts one step late", PY_SRC,
       ("for j in range(int(horizon)):", "for j in range(1, int(horizon)):")),
    _m("mean log retention taken as the log of the mean gate", PY_SRC,
       ("return np.log(g).mean(axis=(0, 1))", "return np.log(g.mean(axis=(0, 1)))")),
    _m("objective without the lifetime", PY_SRC,
       ("return lifetime(ell, horizon)[:, None] * np.asarray(d, dtype=np.float64)",
        "return np.asarray(d, dtype=np.float64)")),
    _m("pivots ranked by ascending score", PY_SRC,
       ("return np.lexsort((np.arange(score.size), -score))", "return np.lexsort((np.arange(score.size), score))")),
    _m("row pivots charged 16 bits of the budget", PY_SRC,
       ("nominal_bits * n - 8 * n_pivots", "nominal_bits * n - 16 * n_pivots")),
    _m("head pivots charged nothing", PY_SRC,
       ("nominal_bits * H - 8 * n_pivots", "nominal_bits * H")),
]


def _slug(name: str) -> str:
    return "".join(ch if ch.isalnum() else "_" for ch in name.lower())[:60]


def _make_tree(dst: Path, mutant: Mutant | None) -> None:
    if dst.exists():
        shutil.rmtree(dst)
    dst.mkdir(parents=True)
    shutil.copytree(ROOT / "oracle", dst / "oracle", ignore=shutil.ignore_patterns("_build", "__pycache__"))
    (dst / PKG).mkdir()
    for f in ("__init__.py", "synth.py"):
        shutil.copy(ROOT / PKG / f, dst / PKG / f)
    (dst / "tests").mkdir()
    for f in PIN_FILES + ["conftest.py"]:
        shutil.copy(TESTS / f, dst / "tests" / f)
    shutil.copytree(TESTS / "golden", dst / "tests" / "golden")
    shutil.copy(ROOT / "pytest.ini", dst / "pytest.ini")
    if mutant is None:
        return
    target = dst / mutant.path
    text = target.read_text()
    for old, new in mutant.edits:
        assert text.count(old) == 1, f"{mutant.name}: edit text occurs {text.count(old)} times"
        text = text.replace(old, new)
    target.write_text(text)


def _run_pins(dst: Path):
    """(status, detail): status is 'pass', 'fail' (a pin failed), 'build' or 'error'."""
    env = dict(os.environ, OMP_NUM_THREADS="1", PYTHONDONTWRITEBYTECODE="1")
    env.pop("PYTHONPATH", None)
    b = subprocess.run([sys.executable, "-c", "import oracle; oracle.build()"], cwd=dst, env=env,
                       capture_output=True, text=True, timeout=300)
    if b.returncode != 0:
        return "build", b.stderr[-2000:]
    p = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "not gpu",
                        *[f"tests/{f}" for f in PIN_FILES]],
                       cwd=dst, env=env, capture_output=True, text=True, timeout=900)
    if p.returncode == 0:
        return "pass", ""
    failed = [ln for ln in p.stdout.splitlines() if ln.startswith("FAILED")]
    if p.returncode == 1 and failed:
        return "fail", failed[0]
    return "error", f"rc={p.returncode}\n{p.stdout[-2000:]}\n{p.stderr[-2000:]}"


def _case(mutant: Mutant | None):
    dst = SCRATCH / ("control" if mutant is None else _slug(mutant.name))
    _make_tree(dst, mutant)
    try:
        return _run_pins(dst)
    finally:
        shutil.rmtree(dst, ignore_errors=True)


def test_every_edit_names_one_place_in_the_source():
    names = [m.name for m in MUTANTS]
    assert len(set(names)) == len(names)
    assert len({_slug(n) for n in names}) == len(names)
    for m in MUTANTS:
        text = (ROOT / m.path).read_text()
        for old, _ in m.edits:
            assert text.count(old) == 1, f"{m.name!r}: {old!r} occurs {text.count(old)} times in {m.path}"


def test_every_planted_mistake_fails_a_pin():
    workers = max(1, min(8, (os.cpu_count() or 2)))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        results = list(ex.map(_case, [None] + MUTANTS))
    status, detail = results[0]
    assert status == "pass", f"the unmodified copy must pass its pins: {status}\n{detail}"
    bad = [(m.name, s, d) for m, (s, d) in zip(MUTANTS, results[1:]) if s != "fail"]
    assert not bad, "planted mistakes no pin caught:\n" + "\n".join(f"  {n}: {s} {d}" for n, s, d in bad)
