"""The pins must catch plausible mistakes in the oracle.

Each case below plants one mistake in a copy of the oracle's C source (on the
CPU, in a temporary directory), builds it, binds the oracle module to the
mutant, and runs the pins of test_oracle_pins.py. At least one pin must fail
for every mutant; the real oracle is re-bound afterwards.
"""
import inspect

import numpy as np
import pytest

import test_oracle_pins as pins

# (name, text in rq_oracle.c, replacement, occurrence index or None = all)
MUTANTS = [
    ("drop the E[x^2] weight", "L = L + ak * e;", "L = L + e;", None),
    ("ties go to the last index", "L < bestL", "L <= bestL", None),
    ("qmax = 2^(b-1)", "int qmax = (1 << (bits - 1)) - 1;", "int qmax = (1 << (bits - 1));", None),
    ("nibbles swapped", "if ((kk & 1) == 0) *byte = u;\n            else *byte = (uint8_t)(*byte | (u << 4));",
     "if ((kk & 1) == 1) *byte = u;\n            else *byte = (uint8_t)(*byte | (u << 4));", None),
    ("search on the unrounded scale", "float sf = orc_f16_to_f32(sh);\n        double L", "float sf = prod;\n        double L", None),
    ("truncate instead of rint", "float r = rintf(clampf(v, -(float)qmax, (float)qmax));",
     "float r = truncf(clampf(v, -(float)qmax, (float)qmax));", None),
    ("asym offset sign", "float M = (lo_i < 0.0f) ? -lo_i : 0.0f;", "float M = (lo_i < 0.0f) ? lo_i : 0.0f;", None),
    ("asym step over 2^b levels", "float S = (2.0f * r) / (float)levels;", "float S = (2.0f * r) / (float)(levels + 1);", None),
    ("5-bit plane bit order", "blk[144 + kk / 8] |= (uint8_t)(up << (kk % 8));", "blk[144 + kk / 8] |= (uint8_t)(up << (7 - kk % 8));", None),
    ("6-bit plane uses 1 bit per code", "blk[144 + kk / 4] |= (uint8_t)(up << (2 * (kk % 4)));", "blk[144 + kk / 4] |= (uint8_t)((up & 1) << (2 * (kk % 4)));", None),
    ("bit string off by one", "int bs = 6 * j + b, bm = 48 + 6 * j + b;", "int bs = 6 * j + b, bm = 47 + 6 * j + b;", None),
    ("fp16 ties away from zero", "(rem == halfway && (kept & 1u))", "(rem == halfway)", None),
    ("grid misses its top end", "step = step / (double)(n - 1);", "step = step / (double)n;", None),
    ("superblock min from the scales", "if (M_star[j] > mM) mM = M_star[j];", "if (S_star[j] > mM) mM = S_star[j];", None),
    ("product sums the wrong row of x", "const double *xm = xd + (size_t)m * K;", "const double *xm = xd;", None),
    ("int8 code offset 127", "codes[(size_t)n * K + kk] = (uint8_t)(qk + 128);",
     "codes[(size_t)n * K + kk] = (uint8_t)(qk + 127);", None),
    ("dequant drops the group index", "float s = orc_f16_to_f32(scales[(size_t)n * ng + k / G]);",
     "float s = orc_f16_to_f32(scales[(size_t)n * ng]);", None),
    ("sb dequant adds the min", "float p = (float)q * S;\n    return p - M;", "float p = (float)q * S;\n    return p + M;", None),
    ("absmax from the last element", "if (v > absmax) absmax = v;", "absmax = v;", None),
    ("6-bit symmetric plane bit order", "chunk[32 + j / 4] |= (uint8_t)((u >> 4) << (2 * (j % 4)));",
     "chunk[32 + j / 4] |= (uint8_t)((u >> 4) << (6 - 2 * (j % 4)));", None),
    ("6-bit symmetric code offset 31", "int u = qk + 32;", "int u = qk + 31;", None),
    ("6-bit symmetric low nibbles swapped", "if ((j & 1) == 0) chunk[j / 2] = (uint8_t)(u & 15);",
     "if ((j & 1) == 1) chunk[j / 2] = (uint8_t)(u & 15);", None),
    ("int8 g64 search on the first 16 weights", "orc_sym_group(row + (size_t)g * G, a ? a + (size_t)g * G : NULL, G, qmax,",
     "orc_sym_group(row + (size_t)g * G, a ? a + (size_t)g * G : NULL, G == 64 && bits == 8 ? 16 : G, qmax,", None),
    ("GPTQ update adds the error", "w[j] = w[j] - err * U[(size_t)k * K + j];", "w[j] = w[j] + err * U[(size_t)k * K + j];", None),
    ("GPTQ divides by the wrong diagonal", "double err = d / U[(size_t)k * K + k];", "double err = d / U[(size_t)k0 * K + k0];", None),
    ("GPTQ scale from the original weights", "for (int i = 0; i < G; i++) wg[i] = (float)w[k0 + i];",
     "for (int i = 0; i < G; i++) wg[i] = W[(size_t)n * K + k0 + i];", None),
    ("GPTQ keeps dead columns", "w[k] = dead[k] ? 0.0 : (double)W[(size_t)n * K + k];", "w[k] = (double)W[(size_t)n * K + k];", None),
    ("GPTQ code from the group search's codes", "int q = sym_code((float)w[k], sf, qmax);", "int q = qg[i];", None),
    ("GPTQ superblock header from the original weights", "for (int i = 0; i < 256; i++) wsb[i] = (float)w[k0 + i];",
     "for (int i = 0; i < 256; i++) wsb[i] = W[(size_t)n * K + k0 + i];", None),
    ("GPTQ superblock error without the min", "double err = (w[k] - (double)asym_deq(q, Sj, Mj)) / U[(size_t)k * K + k];",
     "double err = (w[k] - (double)((float)q * Sj)) / U[(size_t)k * K + k];", None),
    ("Hessian skips the last row", "for (int r = 0; r < R; r++) {\n                double xi", "for (int r = 0; r < R - 1; r++) {\n                double xi", None),
    ("E[x^2] sums |x| instead of x^2", "s = s + v * v;", "s = s + fabs(v);", None),
    ("E[x^2] skips the last row", "for (int r = 0; r < R; r++) {\n            double v", "for (int r = 0; r < R - 1; r++) {\n            double v", None),
    ("E[x^2] divides by rows - 1", "act_sq[k] = (float)(sum_sq[k] / (double)rows);", "act_sq[k] = (float)(sum_sq[k] / (double)(rows - 1));", None),
    ("E[x^2] drops the running sum", "double s = sum_sq[k];", "double s = 0.0;", None),
]


def _pin_calls():
    """Every pin of test_oracle_pins as a zero-argument callable of orc."""
    calls = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        params = list(inspect.signature(fn).parameters)
        marks = getattr(fn, "pytestmark", [])
        grids = [m.args for m in marks if m.name == "parametrize"]
        combos = [{}]
        for argnames, values in grids:
            names = [a.strip() for a in argnames.split(",")]
            new = []
            for c in combos:
                for v in values:
                    vv = v if len(names) > 1 else (v,)
                    new.append({**c, **dict(zip(names, vv))})
            combos = new
        for c in combos:
            if set(params) - {"orc"} <= set(c):
                calls.append((name, fn, c))
    return calls


@pytest.mark.parametrize("mut", range(len(MUTANTS)), ids=[m[0] for m in MUTANTS])
def test_a_pin_fails_for_every_planted_mistake(orc, tmp_path, mut):
    name, old, new, _ = MUTANTS[mut]
    src = orc.source_text()
    assert old in src, f"mutation site for '{name}' not found"
    so = str(tmp_path / "mutant.so")
    orc.compile_variant(src.replace(old, new), so)
    prev = orc.swap_library(so)
    failed = []
    try:
        for pname, fn, kw in _pin_calls():
            try:
                with np.errstate(all="ignore"):
                    fn(orc=orc, **kw)
            except (AssertionError, ValueError, IndexError, OverflowError, ZeroDivisionError):
                failed.append(pname)
                break
    finally:
        orc.swap_library(None)
        orc._lib = prev
    assert failed, f"no pin caught the planted mistake '{name}'"
