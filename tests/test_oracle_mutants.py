"""The oracle's pins catch plausible mistakes.

Each case compiles a copy of the oracle's C source with one planted mistake (a
strict comparison, another rounding rule, a dropped term, a wrong sign or
index, a dropped row, a wrong constant), points the oracle wrapper at the
mutant through LLMINT8_ORACLE_LIB and runs tests/test_oracle.py against it:
some pin must fail.  The unmodified source, compiled the same way, must pass.
Mistakes are planted on the CPU only, in a temporary copy; the committed
oracle is untouched.

Left out because they cannot change any result (equivalent mutants): a strict
`> 65520` overflow bound in the fp16 conversion (the normal path rounds 65520
up to infinity as well) and a lower clamp of -128 (|x / s| <= 127 keeps every
code inside [-127, 127] before the clamp).
"""
import concurrent.futures
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_DIR = os.path.join(ROOT, "oracle")
SRC = os.path.join(ORACLE_DIR, "llmint8_oracle.c")

# name -> (text in the source, replacement); each text occurs exactly once.
MUTANTS = {
    # a1: the outlier test compares strictly
    "threshold_strict": ("if (fabsf(oracle_h2f(X[t * K + k])) >= tau) flag[k] = 1;",
                         "if (fabsf(oracle_h2f(X[t * K + k])) > tau) flag[k] = 1;"),
    # a1: only the first token is searched for outliers
    "detect_first_row_only": ("  for (int64_t t = 0; t < T; ++t)\n    for (int64_t k = 0; k < K; ++k)\n      if (fabsf",
                              "  for (int64_t t = 0; t < T && t < 1; ++t)\n    for (int64_t k = 0; k < K; ++k)\n      if (fabsf"),
    # a4: outlier list in descending order
    "compact_descending": ("  for (int64_t k = 0; k < K; ++k)\n    if (flag[k]) idx[n++] = (int32_t)k;",
                           "  for (int64_t k = K - 1; k >= 0; --k)\n    if (flag[k]) idx[n++] = (int32_t)k;"),
    # a0/a3: ties rounded away from zero, or truncated
    "round_half_away": ("float q = nearbyintf(r);", "float q = roundf(r);"),
    "round_truncate": ("float q = nearbyintf(r);", "float q = truncf(r);"),
    # a0/a3: clamp one short of the int8 range
    "clamp_126": ("if (q > 127.0f) q = 127.0f;", "if (q > 126.0f) q = 126.0f;"),
    # a0: scale from 2^(b-1) instead of 2^(b-1) - 1
    "weight_scale_128": ("    float s = amax / 127.0f;\n    sw[n] = s;", "    float s = amax / 128.0f;\n    sw[n] = s;"),
    # a0: signed maximum instead of the maximum magnitude
    "weight_amax_signed": ("      float a = fabsf(oracle_h2f(row[k]));\n      if (a > amax) amax = a;\n    }\n"
                           "    float s = amax / 127.0f;\n    sw[n] = s;",
                           "      float a = oracle_h2f(row[k]);\n      if (a > amax) amax = a;\n    }\n"
                           "    float s = amax / 127.0f;\n    sw[n] = s;"),
    # a2: the outlier columns still set the activation scale
    "act_scale_over_all_columns": ("      if (flag[k]) continue;\n", ""),
    # a3: outlier columns keep their int8 codes (counted twice)
    "outlier_codes_not_zeroed": ("Xq[t * K + k] = flag[k] ? 0 : oracle_quantize_value(",
                                 "Xq[t * K + k] = oracle_quantize_value("),
    # a5: the last column's term dropped
    "int8_gemm_drops_last_k": ("for (int64_t k = 0; k < K; ++k) s += (int64_t)a[k] * (int64_t)b[k];",
                               "for (int64_t k = 0; k + 1 < K; ++k) s += (int64_t)a[k] * (int64_t)b[k];"),
    # a5: no overflow report
    "int8_gemm_no_overflow_check": ("      if (s > INT32_MAX || s < INT32_MIN) overflow = 1;\n", ""),
    # a6: wrong sign, or the weight column indexed by position in the list
    "outlier_gemm_sign": ("        s += (double)oracle_h2f(X[t * K + k]) *", "        s -= (double)oracle_h2f(X[t * K + k]) *"),
    "outlier_gemm_wrong_index": ("(double)oracle_h2f(W[n * K + k]);", "(double)oracle_h2f(W[n * K + j]);"),
    # a7: a scale or the fp part dropped
    "dequant_drops_weight_scale": ("(double)acc[t * N + n] * (double)sx[t] * (double)sw[n];",
                                   "(double)acc[t * N + n] * (double)sx[t];"),
    "dequant_drops_outlier_part": ("      if (yo) v += yo[t * N + n];\n", ""),
    # fp16 conversions
    "d2h_ties_away": ("double q = nearbyint(ldexp(a, 10 - E));", "double q = round(ldexp(a, 10 - E));"),
    "d2h_overflow_bound": ("if (a >= 65520.0) return sign | 0x7c00;", "if (a >= 65504.0) return sign | 0x7c00;"),
    "h2f_subnormal_scale": ("v = ldexp((double)m, -24);", "v = ldexp((double)m, -25);"),
    "h2f_exponent_bias": ("v = ldexp((double)(1024 + m), e - 25);", "v = ldexp((double)(1024 + m), e - 24);"),
}


def _compile(root, name, text):
    from oracle import oracle as O
    d = root / name
    d.mkdir()
    src = d / "llmint8_oracle.c"
    src.write_text(text, encoding="utf-8")
    shutil.copy(os.path.join(ORACLE_DIR, "llmint8_oracle.h"), d / "llmint8_oracle.h")
    lib = d / "liboracle.so"
    subprocess.check_call(["gcc", *O.CFLAGS, "-o", str(lib), str(src), "-lm"])
    return str(lib)


def _run_pins(lib):
    env = dict(os.environ, LLMINT8_ORACLE_LIB=lib, OMP_NUM_THREADS="2")
    return subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle.py"),
                           "-x", "-q", "-p", "no:cacheprovider", "-m", "not gpu"],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    """name -> CompletedProcess of the pin run, the control ("") included; the
    runs go in parallel, one subprocess each."""
    root = tmp_path_factory.mktemp("oracle_mutants")
    with open(SRC, encoding="utf-8") as f:
        text = f.read()
    libs = {"": _compile(root, "control", text)}
    for name, (old, new) in MUTANTS.items():
        assert text.count(old) == 1, f"{name}: the planted text must occur exactly once"
        libs[name] = _compile(root, name, text.replace(old, new))
    workers = max(1, min(8, (os.cpu_count() or 2) // 2))
    with concurrent.futures.ThreadPoolExecutor(workers) as ex:
        futs = {name: ex.submit(_run_pins, lib) for name, lib in libs.items()}
        return {name: f.result() for name, f in futs.items()}


def test_unmodified_copy_passes(outcomes):
    r = outcomes[""]
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(outcomes, name):
    r = outcomes[name]
    # pytest exits 1 when a test failed (not 2-5: collection or usage errors)
    assert r.returncode == 1, f"{name} survived the pins:\n" + r.stdout[-2000:] + r.stderr[-2000:]
