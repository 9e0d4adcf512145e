"""The pins of the variant oracle catch plausible mistakes.

As tests/test_oracle_mutants.py does for the LLM.int8() oracle: each case
compiles a copy of next_oracle.c with one planted mistake (together with the
unmodified llmint8_oracle.c), points oracle_next at it through
LLMINT8_ORACLE_NEXT_LIB and runs tests/test_oracle_next.py: some pin must fail.
The unmodified copy, compiled the same way, must pass.  Mistakes are planted
on the CPU only, in a temporary copy.
"""
import concurrent.futures
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_DIR = os.path.join(ROOT, "oracle")
SRC = os.path.join(ORACLE_DIR, "next_oracle.c")

MUTANTS = {
    # SmoothQuant: the garbled product form of the factor
    "factor_product_form": ("s[k] = onext_pow(ax[k], alpha) / onext_pow(aw[k], beta);",
                            "s[k] = onext_pow(ax[k], alpha) * onext_pow(aw[k], beta);"),
    # SmoothQuant: the weight exponent not complemented
    "factor_exponent_alpha": ("const float beta = 1.0f - alpha;", "const float beta = alpha;"),
    # SmoothQuant: activations multiplied by s instead of divided
    "activations_times_s": ("float a = fabsf(oracle_h2f(X[t * K + k]) / s[k]);",
                            "float a = fabsf(oracle_h2f(X[t * K + k]) * s[k]);"),
    # SmoothQuant: a zero channel gets s = 0
    "zero_channel_zero": ("      s[k] = 1.0f;\n      continue;", "      s[k] = 0.0f;\n      continue;"),
    # FP8: ties away from zero
    "e4m3_ties_away": ("double q = nearbyint(ldexp(a, 3 - E));", "double q = round(ldexp(a, 3 - E));"),
    # FP8: exponent bias 8
    "e4m3_bias_8": ("v = ldexp((double)(8 + m), e - 10);", "v = ldexp((double)(8 + m), e - 11);"),
    # FP8: int8 scale
    "fp8_weight_scale_127": ("    float s = amax / 448.0f;\n    sw[n] = s;", "    float s = amax / 127.0f;\n    sw[n] = s;"),
    # FP8: the sign of zero dropped
    "e4m3_unsigned_zero": ("const uint8_t sign = signbit(x) ? 0x80 : 0;", "const uint8_t sign = (x < 0) ? 0x80 : 0;"),
    # FP8: the last product dropped
    "fp8_gemm_drops_last_k": ("for (int64_t k = 0; k < K; ++k) s += xd[t * K + k] * wd[n * K + k];",
                              "for (int64_t k = 0; k + 1 < K; ++k) s += xd[t * K + k] * wd[n * K + k];"),
    # stored columns: a miss uses the raw code without its scale
    "miss_without_scale": ("onext_reconstruct_weight(Wq[n * K + k], sw[n]);",
                           "onext_reconstruct_weight(Wq[n * K + k], 1.0f);"),
    # stored columns: truncating reconstruction
    "reconstruct_binary64": ("float p = s * (float)q;", "double p = (double)s * (double)q;"),
    # stored columns: misses not counted
    "miss_not_counted": ("    if (slot[idx[j]] < 0) ++miss;", "    if (slot[idx[j]] < -1) ++miss;"),
}


def run_pins(lib, tmp):
    env = dict(os.environ, LLMINT8_ORACLE_NEXT_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_next.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    return r.returncode


def build(tmp, name, text):
    d = tmp / name
    d.mkdir()
    for f in ("llmint8_oracle.c", "llmint8_oracle.h", "next_oracle.h"):
        shutil.copy(os.path.join(ORACLE_DIR, f), d / f)
    (d / "next_oracle.c").write_text(text, encoding="utf-8")
    from oracle import oracle as O
    lib = d / "lib.so"
    subprocess.check_call(["gcc", *O.CFLAGS, "-o", str(lib), str(d / "llmint8_oracle.c"), str(d / "next_oracle.c"),
                           "-lm"])
    return lib


def test_mutants_are_caught(tmp_path):
    src = open(SRC, encoding="utf-8").read()
    jobs = {"unmodified": src}
    for name, (old, new) in MUTANTS.items():
        assert src.count(old) == 1, name
        jobs[name] = src.replace(old, new)
    libs = {name: build(tmp_path, name, text) for name, text in jobs.items()}
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        rcs = dict(zip(libs, ex.map(lambda kv: run_pins(kv[1], tmp_path), libs.items())))
    assert rcs.pop("unmodified") == 0
    survivors = [n for n, rc in rcs.items() if rc == 0]
    assert not survivors, f"mutants not caught by any pin: {survivors}"
