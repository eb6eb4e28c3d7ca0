"""Pins for the CPU oracle's keep-mask producers (CPU only).

Readings (the pages name Threshold-l2 among the pruning methods the pipeline
serves, radpulse "Integrated pack pipeline", without spelling out a rule):
  top-k      image b keeps CLS and the k_b - 1 other tokens with the highest
             scores; ties go to the lower index, NaN ranks below every
             number; k_b is clamped to [1, L_full];
  l2         token kept when the Euclidean norm of its features is >= tau;
             CLS is always kept.
Each pin ties the oracle to something other than itself: a sort by numpy's
lexsort, exact rational arithmetic, closed cases and invariants.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synthetic


def _topk_by_lexsort(scores, k):
    B, L = scores.shape
    keep = np.zeros((B, L), dtype=np.uint8)
    for b in range(B):
        with np.errstate(invalid="ignore"):                 # signalling NaNs widen quietly
            s = scores[b, 1:].astype(np.float64)
        nan = np.isnan(s)
        key_score = np.where(nan, 0.0, -s)                 # descending score
        order = np.lexsort((np.arange(1, L), key_score, nan))  # numbers first, then score, then index
        kk = int(min(max(k[b], 1), L))
        keep[b, 0] = 1
        keep[b, 1 + order[:kk - 1]] = 1
    return keep


def _random_scores(rng, B, L, ties=False, nans=False):
    s = rng.standard_normal((B, L)).astype(np.float32)
    if ties:
        s = np.round(s * 2) / 2                            # many exact ties
    if nans:
        s[rng.random((B, L)) < 0.1] = np.nan
    return s


@pytest.mark.parametrize("ties,nans", [(False, False), (True, False), (False, True), (True, True)])
def test_topk_matches_lexsort(ties, nans):
    rng = synthetic.rng_for(2001, int(ties) * 2 + int(nans))
    B, L = 7, 97
    s = _random_scores(rng, B, L, ties, nans)
    k = rng.integers(-2, L + 5, size=B).astype(np.int32)   # includes out-of-range counts
    assert np.array_equal(oracle.mask_topk(s, k), _topk_by_lexsort(s, k))


def test_topk_special_values_match_lexsort():
    """Signed zeros tie, denormals stay apart from zero, infinities sit at the
    ends of the numbers, and NaNs of every payload and sign tie below -inf."""
    bits = np.array([0x00000000, 0x80000000, 0x00000001, 0x80000001, 0x007fffff, 0x807fffff,
                     0x7f800000, 0xff800000, 0x7f7fffff, 0xff7fffff, 0x7fc00000, 0xffc00000,
                     0x7f800001, 0xffffffff, 0x3f800000, 0xbf800000], dtype=np.uint32)
    rng = synthetic.rng_for(2005)
    B, L = 9, 131
    s = bits[rng.integers(0, bits.size, size=(B, L))].view(np.float32)
    k = rng.integers(1, L + 1, size=B).astype(np.int32)
    assert np.array_equal(oracle.mask_topk(s, k), _topk_by_lexsort(s, k))
    z = np.array([[0.0, 0.0, -0.0, 0.0]], dtype=np.float32)
    z[0, 1] = -0.0
    assert oracle.mask_topk(z, np.array([2])).tolist() == [[1, 1, 0, 0]]   # -0 ties +0: lower index
    d = np.array([[0.0, 0.0, 0.0, 0.0]], dtype=np.float32)
    d[0, 3] = np.uint32(1).view(np.float32)                                 # smallest denormal beats zero
    assert oracle.mask_topk(d, np.array([2])).tolist() == [[1, 0, 0, 1]]


def test_topk_closed_cases():
    s = np.array([[0.0, 3.0, 1.0, 2.0, 3.0, np.nan]], dtype=np.float32)
    # top-2 of indices 1..5: the two 3.0s (tie: lower index first is irrelevant, both kept)
    assert oracle.mask_topk(s, np.array([3])).tolist() == [[1, 1, 0, 0, 1, 0]]
    # top-1: the lower-index 3.0
    assert oracle.mask_topk(s, np.array([2])).tolist() == [[1, 1, 0, 0, 0, 0]]
    # k = 1: CLS only; k >= L: everything, NaN included
    assert oracle.mask_topk(s, np.array([1])).tolist() == [[1, 0, 0, 0, 0, 0]]
    assert oracle.mask_topk(s, np.array([99])).tolist() == [[1, 1, 1, 1, 1, 1]]
    # the NaN token is the last one chosen
    assert oracle.mask_topk(s, np.array([5])).tolist() == [[1, 1, 1, 1, 1, 0]]
    # CLS's own score never matters
    s2 = s.copy()
    s2[0, 0] = -np.inf
    assert np.array_equal(oracle.mask_topk(s2, np.array([3])), oracle.mask_topk(s, np.array([3])))


def test_topk_counts_and_cls():
    rng = synthetic.rng_for(2002)
    s = _random_scores(rng, 16, 197, nans=True)
    k = rng.integers(1, 197, size=16).astype(np.int32)
    keep = oracle.mask_topk(s, k)
    assert np.all(keep[:, 0] == 1)
    assert np.array_equal(keep.sum(1), k)


def _exact_norm_sq(row_values):
    return sum(Fraction(float(v)) ** 2 for v in row_values)


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
def test_l2_matches_exact_arithmetic(dtype):
    rng = synthetic.rng_for(2003, ["f16", "bf16", "f32"].index(dtype))
    B, L, C = 3, 41, 70
    x = synthetic.store(rng.standard_normal((B, L, C)).astype(np.float32), dtype)
    xf = oracle.decode(x, dtype).reshape(B, L, C)
    norms = np.sqrt(np.sum(xf * xf, axis=2))
    tau = float(np.median(norms))
    keep = oracle.mask_l2(x, dtype, tau)
    tau_sq = Fraction(tau) ** 2
    for b in range(B):
        for j in range(L):
            want = 1 if j == 0 or _exact_norm_sq(xf[b, j]) >= tau_sq else 0
            assert keep[b, j] == want, (b, j)


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
def test_l2_exact_at_and_next_to_tau(dtype):
    """Thresholds at, one ulp below and one ulp above the double nearest each
    token's norm: the decision must be the exact rational comparison
    sum(x^2) >= tau^2 (Python fractions), whatever fp64 rounding would say."""
    rng = synthetic.rng_for(2004, ["f16", "bf16", "f32"].index(dtype))
    B, L, C = 2, 9, 384
    x = synthetic.store(rng.standard_normal((B, L, C)).astype(np.float32), dtype)
    xf = oracle.decode(x, dtype).reshape(B, L, C)
    for b in range(B):
        for j in range(1, L):
            exact = _exact_norm_sq(xf[b, j])
            t0 = math.sqrt(float(exact))
            for tau in (np.nextafter(t0, 0.0), t0, np.nextafter(t0, np.inf)):
                keep = oracle.mask_l2(x, dtype, float(tau))
                want = 1 if exact >= Fraction(float(tau)) ** 2 else 0
                assert keep[b, j] == want, (b, j, tau)


def test_l2_decides_where_fp64_sums_round():
    """Sums of squares that fp64 addition rounds: 1 + 2^-51 + 2^-104 (squares
    of 1, 2^-26, 2^-26, 2^-52) is exactly (1 + 2^-52)^2; sixteen squares of
    2^-30 added to 1 vanish in any fp64 order that starts from 1."""
    x = np.zeros((1, 3, 64), dtype=np.float32)
    x[0, 1, :4] = [1.0, 2.0 ** -26, 2.0 ** -26, 2.0 ** -52]
    x[0, 2, 0] = 1.0
    x[0, 2, 1:17] = 2.0 ** -30
    tau = 1.0 + 2.0 ** -52
    assert Fraction(tau) ** 2 == _exact_norm_sq(x[0, 1])
    assert oracle.mask_l2(x, "f32", tau).tolist() == [[1, 1, 0]]
    assert oracle.mask_l2(x, "f32", float(np.nextafter(tau, 2.0))).tolist() == [[1, 0, 0]]
    # row 2: 1 + 16 * 2^-60 = 1 + 2^-56 > 1, so it reaches tau = 1 and not the next double
    assert oracle.mask_l2(x, "f32", 1.0).tolist() == [[1, 1, 1]]
    assert oracle.mask_l2(x, "f32", float(np.nextafter(1.0, 2.0))).tolist() == [[1, 1, 0]]


def test_l2_subnormals_nan_and_infinity():
    tiny = np.float32(2.0 ** -149)                 # the smallest f32 subnormal; its square is 2^-298
    x = np.zeros((1, 5, 8), dtype=np.float32)
    x[0, 1, 3] = tiny
    x[0, 2, 0], x[0, 2, 5] = tiny, tiny            # norm 2^-149 * sqrt(2)
    x[0, 3, 0], x[0, 3, 1] = np.nan, 100.0
    x[0, 4, 2] = -np.inf
    t = 2.0 ** -149
    assert oracle.mask_l2(x, "f32", t).tolist() == [[1, 1, 1, 0, 1]]
    assert oracle.mask_l2(x, "f32", float(np.nextafter(t, 1.0))).tolist() == [[1, 0, 1, 0, 1]]
    assert oracle.mask_l2(x, "f32", t * math.sqrt(2.0) * (1 + 2.0 ** -40)).tolist() == [[1, 0, 0, 0, 1]]
    # a threshold far below the smallest nonzero square, and one far above any sum
    assert oracle.mask_l2(x, "f32", 1e-300).tolist() == [[1, 1, 1, 0, 1]]
    assert oracle.mask_l2(x, "f32", 1e300).tolist() == [[1, 0, 0, 0, 1]]
    # an infinite norm reaches even an infinite tau (inf >= inf); a NaN norm reaches nothing
    assert oracle.mask_l2(x, "f32", float("inf")).tolist() == [[1, 0, 0, 0, 1]]


def test_l2_boundary_and_closed_cases():
    # norm exactly tau (3-4-5 and 5-12-13) is kept; a hair below is not
    x = np.zeros((1, 5, 64), dtype=np.float32)
    x[0, 1, 0], x[0, 1, 40] = 3.0, 4.0            # norm 5, elements in different partial sums
    x[0, 2, 7], x[0, 2, 39] = 5.0, 12.0           # norm 13
    x[0, 3, 0] = np.nextafter(np.float32(5.0), np.float32(0.0))
    x[0, 4, :] = 0.625                            # norm 0.625 * 8 = 5
    assert oracle.mask_l2(x, "f32", 5.0).tolist() == [[1, 1, 1, 0, 1]]
    assert oracle.mask_l2(x, "f32", 13.0).tolist() == [[1, 0, 1, 0, 0]]
    # CLS is kept even with zero features; tau <= 0 keeps everything
    assert oracle.mask_l2(np.zeros((2, 3, 8), np.float32), "f32", 1.0).tolist() == [[1, 0, 0], [1, 0, 0]]
    assert oracle.mask_l2(np.zeros((2, 3, 8), np.float32), "f32", 0.0).tolist() == [[1, 1, 1], [1, 1, 1]]
