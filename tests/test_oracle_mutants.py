"""The oracle's pins against planted mistakes.

Each case copies oracle/oracle.c, plants one plausible mistake (a comparison,
a rounding mode, a clamp, a scale, an index, a loop bound, a dropped or
misplaced term), builds the copy and runs tests/test_oracle_pins.py against
it in a subprocess.  Every such mutant must fail at least one pin; an
unmutated copy built the same way must pass them all."""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

MUTANTS = {
    # binary16 codec
    "half_decode_exponent_bias": ("v = ldexp((double)(1024 + f), e - 25);", "v = ldexp((double)(1024 + f), e - 24);"),
    "half_decode_subnormal_scale": ("v = ldexp((double)f, -24);", "v = ldexp((double)f, -25);"),
    "half_encode_ties_away": ("double m = nearbyint(ldexp(a, 10 - e));", "double m = round(ldexp(a, 10 - e));"),
    # outlier detection
    "threshold_ge": ("if (colmax[j] > alpha) idx[n++] = (int32_t)j;", "if (colmax[j] >= alpha) idx[n++] = (int32_t)j;"),
    "colmax_skips_first_row": ("    for (int64_t i = 0; i < M; ++i)\n        for (int64_t j = 0; j < K; ++j) {",
                               "    for (int64_t i = 1; i < M; ++i)\n        for (int64_t j = 0; j < K; ++j) {"),
    "outliers_descending": ("    for (int64_t j = 0; j < K; ++j)\n        if (colmax[j] > alpha)",
                            "    for (int64_t j = K - 1; j >= 0; --j)\n        if (colmax[j] > alpha)"),
    # vector-wise quantisation
    "scale_128": ("return 127.0f / absmax;", "return 128.0f / absmax;"),
    "scale_inverted": ("return 127.0f / absmax;", "return absmax / 127.0f;"),
    "round_half_away": ("float r = nearbyintf(p);", "float r = roundf(p);"),
    "clamp_to_minus_128": ("if (r < -127.0f) r = -127.0f;", "if (r < -128.0f) r = -128.0f;"),
    "row_absmax_over_outliers_too": ("            if (is_out[j]) continue;\n", ""),
    "outlier_codes_not_zeroed": ("q[i * K + j] = is_out[j] ? 0 : orc_quantize_value(x, ci);",
                                 "q[i * K + j] = orc_quantize_value(x, ci);"),
    "col_absmax_skips_last_row": (
        "        for (int64_t k = 0; k < K; ++k) {\n            float a = (float)fabs(orc_half_to_double(W[k * N + j]));",
        "        for (int64_t k = 0; k < K - 1; ++k) {\n            float a = (float)fabs(orc_half_to_double(W[k * N + j]));"),
    # contraction
    "matmul_skips_last_k": ("for (int64_t k = 0; k < K; ++k) {\n                int64_t a = qx[i * K + k];",
                            "for (int64_t k = 0; k < K - 1; ++k) {\n                int64_t a = qx[i * K + k];"),
    # dequantisation and the outlier product
    "dequant_multiplies": ("(double)acc[i * N + j] / s;", "(double)acc[i * N + j] * s;"),
    "dequant_forgets_c_w": ("double s = (double)cx[i] * (double)cw[j];", "double s = (double)cx[i];"),
    "outlier_term_dropped": ("row[j] += x * orc_half_to_double(W[k * N + j]);", "row[j] += 0.0 * x;"),
    "outlier_row_by_ordinal": ("row[j] += x * orc_half_to_double(W[k * N + j]);",
                               "row[j] += x * orc_half_to_double(W[o * N + j]);"),
    "bias_dropped": ("if (bias)  /* the layer's bias", "if (0 && bias)  /* the layer's bias"),
    "bias_after_rounding": (
        "Y[i * N + j] = orc_double_to_half(row[j]);",
        "Y[i * N + j] = bias ? orc_double_to_half(orc_half_to_double(orc_double_to_half(row[j] - "
        "orc_half_to_double(bias[j]))) + orc_half_to_double(bias[j])) : orc_double_to_half(row[j]);"),
    # memory-saving weight
    "rebuild_scale_wrong_way": ("float w = (float)q[k * N + j] * inv;", "float w = (float)q[k * N + j] * c[j];"),
}


def _run_pins(workdir: str, source: str):
    c = os.path.join(workdir, "oracle_copy.c")
    with open(c, "w", encoding="utf-8") as f:
        f.write(source)
    so = os.path.join(workdir, "liboracle_copy.so")
    subprocess.check_call(["gcc", *oracle.CFLAGS, c, "-o", so, "-lm"])
    env = dict(os.environ, INT8MM_ORACLE_LIB=so, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", PINS, "-x", "-q", "-p", "no:cacheprovider"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    return r.returncode, r.stdout[-3000:]


def _source():
    with open(oracle._SRC, encoding="utf-8") as f:
        return f.read()


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    """Build and run the unmutated copy and every mutant, several at a time."""
    src = _source()
    jobs = {"unmutated": src}
    for name, (old, new) in MUTANTS.items():
        assert src.count(old) == 1, f"mutation site of {name} not found exactly once"
        jobs[name] = src.replace(old, new)
    workers = max(1, min(8, (os.cpu_count() or 2) // 2))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        futs = {name: ex.submit(_run_pins, str(tmp_path_factory.mktemp(name)), text) for name, text in jobs.items()}
        return {name: f.result() for name, f in futs.items()}


def test_unmutated_copy_passes_the_pins(outcomes):
    code, out = outcomes["unmutated"]
    assert code == 0, out


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_a_planted_mistake(name, outcomes):
    code, out = outcomes[name]
    # 1: tests ran and at least one failed (a crash or a collection error is not a catch)
    assert code == 1, (name, code, out)
