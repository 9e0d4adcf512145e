"""The division-free code arithmetic of the kernels (csrc/quant.cuh), restated
in numpy on the CPU for every finite fp16 value under many scales, against the
oracle's codes from the IEEE quotient:

- int8: the product e = x * fl(1/s) rounded to an integer inside one fused
  multiply-add, and its distance d to that integer rounded once; wherever
  |d| < 1/2 - 2^-12 the kernel keeps that integer, and it must be the code
  rint_even(fl(x / s)).  Only about one element in 2000 may fall back.
- E4M3: a = fl(x * fl(1/s)); wherever fl(a (1 - 2^-20)) and fl(a (1 + 2^-20))
  convert to the same code, that code must be the code of fl(x / s).
- the threshold: for an fp16 x, |x| >= tau in binary32 exactly when
  |x| >= tau_h in fp16, tau_h the smallest fp16 not below tau.

These pin the arithmetic the kernels rely on; the GPU tests check the kernels
themselves bit for bit."""
import numpy as np
import pytest

from oracle import oracle_next as ON


def finite_halves():
    pos = np.arange(0, 0x7C00, dtype=np.uint16)
    return np.concatenate([pos, pos | 0x8000]).view(np.float16)


def scales_from(rng, n, lo=-14, hi=15):
    """fp16 row maxima: powers of two, near-powers, random values, edge values."""
    pw = [np.float16(2.0 ** k) for k in range(lo, hi)]
    near = [np.nextafter(np.float16(v), np.float16(0)) for v in pw] + [np.float16(127.0), np.float16(6.0),
                                                                        np.float16(0.37), np.float16(65504.0)]
    rnd = rng.uniform(2.0 ** -10, 6e4, size=n).astype(np.float16)
    out = np.array(pw + near + list(rnd), np.float16)
    return out[out > 0]


def test_int8_fused_rounding_matches_the_quotient():
    vals = finite_halves().astype(np.float32)
    rng = np.random.default_rng(11)
    near_total = checked = 0
    for amax in scales_from(rng, 60):
        a32 = np.float32(amax)
        s = np.float32(a32 / np.float32(127.0))
        inv = np.float32(np.float32(1.0) / s)
        x = vals[np.abs(vals) <= a32]                         # the regular elements of such a row
        e = x.astype(np.float64) * np.float64(inv)            # exact product (24 x 24 bits)
        r = np.rint(e)                                        # fl(e + 1.5 * 2^23) - 1.5 * 2^23, ties to even
        d = (e - r).astype(np.float32)                        # e - r exact in binary64, rounded once
        near = ~(np.abs(d) < np.float32(0.5 - 2.0 ** -12))
        oracle_code = np.clip(np.rint((x / s).astype(np.float32)), -127, 127)
        ok = ~near
        assert np.array_equal(r[ok], oracle_code[ok]), f"amax={amax}"
        assert np.abs(r[ok]).max() <= 127                     # no clamp needed on the fast path
        near_total += int(near.sum())
        checked += x.size
    assert near_total < checked / 500, (near_total, checked)


def test_e4m3_bracketing_matches_the_quotient():
    vals = finite_halves().astype(np.float32)
    rng = np.random.default_rng(12)
    down = np.float32(1.0 - 2.0 ** -20)
    up = np.float32(1.0 + 2.0 ** -20)
    differ_total = checked = 0
    for amax in scales_from(rng, 2, lo=-6, hi=12)[::3]:
        a32 = np.float32(amax)
        s = np.float32(a32 / np.float32(448.0))
        inv = np.float32(np.float32(1.0) / s)
        x = vals[np.abs(vals) <= a32]
        a = (x * inv).astype(np.float32)
        lo = ON.float_to_e4m3((a * down).astype(np.float32))
        hi = ON.float_to_e4m3((a * up).astype(np.float32))
        same = lo == hi
        quotient = ON.float_to_e4m3((x / s).astype(np.float32))
        assert np.array_equal(lo[same], quotient[same]), f"amax={amax}"
        differ_total += int((~same).sum())
        checked += x.size
    assert differ_total < checked / 20, (differ_total, checked)


def tau_half(tau):
    with np.errstate(over="ignore"):
        h = np.float16(tau)
        if np.float32(h) < np.float32(tau):
            h = np.nextafter(h, np.float16(np.inf))
    return h


@pytest.mark.parametrize("tau", [6.0, 6.0001, float(np.nextafter(np.float32(6.0), np.float32(0))), 1e-8, 0.0, -1.0,
                                 2.5, 65504.0, 65519.0, 70000.0, float("inf"), 5.96e-8, 3e-8])
def test_threshold_in_half_precision(tau):
    x = np.concatenate([finite_halves(), np.array([np.inf, -np.inf], np.float16)])
    binary32 = np.abs(x.astype(np.float32)) >= np.float32(tau)
    th = tau_half(tau)
    half = np.abs(x) >= th
    assert np.array_equal(binary32, half), (tau, th)
