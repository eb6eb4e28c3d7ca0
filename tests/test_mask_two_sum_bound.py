"""The error bound the Threshold-l2 vector path relies on, checked on the CPU.

The keep decision is exact (a token is kept when sum x^2 >= tau^2 in exact
arithmetic), but the kernel first forms a filter sum and only recomputes the
sum exactly inside a relative band of 2^-26 around tau^2, so the filter sum
must be within a relative 2^-29 of the exact one.  For f16 / bf16 rows the
vector path forms it as follows: 16 lanes per token, each taking every 16th
16-byte vector (8 elements); per lane, the squares of the even and of the odd
elements of each vector go into two fp32 accumulators with an error-free
two-sum that keeps the rounding errors in a second pair; the 16 lanes' pairs
are then added in fp64.  With n <= 256 terms per accumulator the stated bound
is n^2 2^-48 <= 2^-32 per pair, 2^-31 in all.

This file restates that accumulation with numpy float32 arithmetic (IEEE
round-to-nearest, no fused operations) and compares it with the exact sum of
squares, formed in Python integers, on random rows and on rows built to make
rounding errors large (magnitudes spread over the whole f16 range, long runs
of one value, cancellation-free but alignment-heavy sums).
"""
import numpy as np
import pytest

import synthetic


def two_sum_filter(x16, dtype):
    """The vector path's filter sum of one token (x16: the stored 16-bit values)."""
    xf = (x16.view(np.float16).astype(np.float32) if dtype == "f16"
          else (x16.astype(np.uint32) << 16).view(np.float32))
    C = xf.size
    assert C % 8 == 0
    nvec = C // 8
    total = 0.0
    for lane in range(16):
        s = np.zeros(2, np.float32)
        c = np.zeros(2, np.float32)
        for v in range(lane, nvec, 16):
            vec = xf[8 * v:8 * v + 8]
            for i in range(4):
                y = np.array([vec[2 * i] * vec[2 * i], vec[2 * i + 1] * vec[2 * i + 1]], np.float32)
                t = s + y
                bp = t - s
                e = (s - (t - bp)) + (y - bp)
                s = t
                c = c + e
        total += (float(s[0]) + float(c[0])) + (float(s[1]) + float(c[1]))
    return total


def exact_sum(x16, dtype):
    """sum x^2 exactly, as a Python integer in units of 2^-298."""
    xf = (x16.view(np.float16).astype(np.float64) if dtype == "f16"
          else (x16.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    acc = 0
    for v in xf:
        if v == 0.0:
            continue
        m, e = np.frexp(abs(v))             # v = m 2^e, 0.5 <= m < 1
        m, e = float(m), int(e)
        mi = int(m * 2 ** 53)               # exact: 16-bit values have few mantissa bits
        acc += (mi * mi) << (2 * (e - 53) + 298)
    return acc


def rel_error(x16, dtype):
    ex = exact_sum(x16, dtype)
    got = two_sum_filter(x16, dtype)
    if ex == 0:
        return 0.0 if got == 0.0 else float("inf")
    return abs(to_units(got) - ex) / ex


def to_units(d):
    """A double as a Python integer in units of 2^-298 (rounded down below that unit)."""
    m, e = np.frexp(d)
    m, e = float(m), int(e)
    sh = e - 53 + 298
    mi = int(m * 2 ** 53)
    return mi << sh if sh >= 0 else mi >> -sh


def rows(dtype, seed):
    rng = synthetic.rng_for(3101, seed)
    C = 8192 if seed % 2 else 384
    out = []
    out.append(rng.standard_normal(C).astype(np.float32))
    # magnitudes spread over the format's range, sorted so small terms meet a large sum
    hi = 15 if dtype == "f16" else 60
    lo = -24 if dtype == "f16" else -60
    mags = np.ldexp(1.0, rng.integers(lo, hi, size=C)).astype(np.float32)
    out.append(np.sort(mags * (1 + rng.random(C).astype(np.float32))))
    out.append(np.sort(mags)[::-1].copy())
    # one large value then a long run of values just below its rounding step
    r = np.full(C, 2.0 ** -6, np.float32)
    r[0] = 2.0 ** 6
    out.append(r)
    stored = []
    for r in out:
        if dtype == "f16":
            stored.append(np.clip(r, -65504, 65504).astype(np.float16).view(np.uint16))
        else:
            b = r.astype(np.float32).view(np.uint32)
            stored.append(((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16))   # round to nearest even
    return stored


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("seed", [0, 1])
def test_two_sum_filter_within_its_bound(dtype, seed):
    worst = 0.0
    for x in rows(dtype, seed):
        worst = max(worst, rel_error(x, dtype))
    assert worst <= 2.0 ** -31, worst
    # and the bound is not vacuous: plain fp32 accumulation misses it on these rows
    x = rows(dtype, seed)[1]
    xf = (x.view(np.float16).astype(np.float32) if dtype == "f16"
          else (x.astype(np.uint32) << 16).view(np.float32))
    plain = np.float32(0)
    for v in xf:
        plain = np.float32(plain + v * v)
    ex = exact_sum(x, dtype)
    assert abs(to_units(float(plain)) - ex) / ex > 2.0 ** -29
