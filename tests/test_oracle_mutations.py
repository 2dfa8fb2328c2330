"""Plant plausible mistakes in a copy of the oracle and check that the pins catch each one.

The mistakes are the kinds the parakeet.cpp PR's own mutation testing planted (section
"Tests": a swapped or one-off pad, a scrambled batch axis), plus dropped masks, a dropped
ReLU, flipped taps and transposed operands.  Each mutant is compiled from a temporary copy
of the oracle's C source on the CPU; the committed oracle is never changed.
"""
import os
import shutil

import pytest

import oracle
from pinlib import pin_battery

MUTANTS = {
    "one-off pad": ("int64_t s = j - pad_left;", "int64_t s = j - pad_left + 1;"),
    "pre-mask dropped": ("if (s < 0 || s >= L) return 0.0;", "if (s < 0 || s >= T) return 0.0;"),
    "post-mask dropped": ("if (t < L) {", "if (t < T) {"),
    "dx taps flipped": ("const int64_t s = t + k - pad_left;", "const int64_t s = t - k + pad_left;"),
    "dx batch scrambled": ("dx[(b * T + s) * C + c] += dy[(b * T + t) * C + c]",
                           "dx[(b * T + s) * C + c] += dy[((B - 1 - b) * T + t) * C + c]"),
    "dw taps reversed": ("xpad_at(x, b, t + k, c, T, C, pad_left, L);\n",
                         "xpad_at(x, b, t + K - 1 - k, c, T, C, pad_left, L);\n"),
    "dbias unmasked": ("db += dz;", "db += dy[(b * T + t) * C + c];"),
    "relu dropped": ("double hv = a > 0.0 ? a : 0.0;", "double hv = a;"),
    "h mask off by one": ("if (i >= L2) hv = 0.0;", "if (i > L2) hv = 0.0;"),
    "out mask dropped": ("if (i >= L4) a = 0.0;", "if (i > T4) a = 0.0;"),
    "conv0 taps transposed": ("* w0[(p * 3 + q) * C + c];", "* w0[(q * 3 + p) * C + c];"),
    "h placed with symmetric offset": ("hpad[((i + Pt) * HF + (j + 1)) * C + c] = hv;",
                                       "hpad[((i + 1) * HF + (j + 1)) * C + c] = hv;"),
    "conv_dw1 freq taps flipped": ("hpad[((2 * i + p) * HF + (2 * j + q)) * C + c]",
                                   "hpad[((2 * i + p) * HF + (2 * j + 2 - q)) * C + c]"),
    "mel not masked": ("melpad[r * FP + f] = (t >= 0 && t < L &&", "melpad[r * FP + f] = (t >= 0 && t < T &&"),
    "stream cache not shifted": ("cache_out[(b * H + j) * C + c] = xcat[(L + j) * C + c];",
                                 "cache_out[(b * H + j) * C + c] = xcat[j * C + c];"),
    "stream output mask dropped": ("if (L > t) {", "if (T > t) {"),
    "stream taps reversed": ("acc += xcat[(t + k) * C + c] * w[k * C + c];",
                             "acc += xcat[(t + k) * C + c] * w[(K - 1 - k) * C + c];"),
    "subsample bwd relu derivative dropped": ("(r < L2 && z[(r * F2 + s) * C + c] > 0.0)", "(r < L2)"),
    "subsample bwd h mask dropped": ("(r < L2 && z[(r * F2 + s) * C + c] > 0.0)",
                                     "(z[(r * F2 + s) * C + c] > 0.0)"),
    "subsample bwd dout mask dropped": ("const double dm = (i < L4) ?", "const double dm = (i < T4) ?"),
    "subsample bwd dw1 taps transposed": ("dw1[(p * 3 + q) * C + c] += dm * hpad[at];",
                                          "dw1[(q * 3 + p) * C + c] += dm * hpad[at];"),
    "subsample bwd recomputed conv0 taps transposed": ("const double tap = w0[(p * 3 + q) * C + c];",
                                                       "const double tap = w0[(q * 3 + p) * C + c];"),
    "subsample bwd mel not masked": ("(ff >= 0 && ff < F && t >= 0 && t < L)", "(ff >= 0 && ff < F && t >= 0 && t < T)"),
    "conv2d taps transposed": ("w[(p * KF + q) * C + c];\n                    }\n                    y[", "w[(q * KT + p) * C + c];\n                    }\n                    y["),
    "conv2d dx stride dropped": ("const int64_t t = st * i + p - pt, f = sf * j + q - pf;",
                                 "const int64_t t = i + p - pt, f = sf * j + q - pf;"),
    "conv2d output mask dropped": ("                    if (i < Lo) {\n                        acc = bias ? bias[c] : 0.0;",
                                   "                    if (i < To) {\n                        acc = bias ? bias[c] : 0.0;"),
    "conv2d dbias unmasked rows": ("            for (int64_t i = 0; i < Lo; ++i)\n                for (int64_t j = 0; j < Fo; ++j) {\n                    const double g = dy[((b * To + i) * Fo + j) * C + c];\n                    gb += g;",
                                   "            for (int64_t i = 0; i < To; ++i)\n                for (int64_t j = 0; j < Fo; ++j) {\n                    const double g = dy[((b * To + i) * Fo + j) * C + c];\n                    gb += g;"),
    "kink budget sign of z ignored": ("if (fabs(zv) > delta + delta_rel * mag) continue;",
                                      "if (zv > delta + delta_rel * mag) continue;"),
    "kink budget row mask off by one": ("for (int64_t r = 0; r < T2 && r < L2; ++r)",
                                        "for (int64_t r = 0; r < T2 && r <= L2; ++r)"),
    "kink budget dout mask dropped": ("if (i >= T4 || i >= L4 || j >= F4) continue;",
                                      "if (i >= T4 || j >= F4) continue;"),
    "kink budget signed dh": ("kdb0[c] += fabs(dh);", "kdb0[c] += dh;"),
    "kink budget signed term magnitudes": ("mag += fabs(term);", "mag += term;"),
    "subsample bwd dh taps flipped": ("dhpad[at] += dm * w1[(p * 3 + q) * C + c];",
                                      "dhpad[at] += dm * w1[((2 - p) * 3 + q) * C + c];"),
}


@pytest.fixture(scope="module")
def source():
    with open(os.path.join(os.path.dirname(oracle.__file__), "dwconv_oracle.c")) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, source, tmp_path):
    old, new = MUTANTS[name]
    assert source.count(old) == 1, f"mutation site for {name!r} not unique in the oracle source"
    src = tmp_path / "mutant.c"
    src.write_text(source.replace(old, new))
    lib = oracle.build(force=True, src=str(src), out=str(tmp_path / "libmutant.so"))
    fails = pin_battery(oracle.Oracle(lib))
    assert fails, f"no pin caught the planted mistake {name!r}"
    shutil.rmtree(tmp_path, ignore_errors=True)
