"""The seeded input generators against the input recipe (CPU only).

Each workload must have the shapes, formats and survivor-count rules the
recipe states: the tiny DeiT-S batch with counts {197, 120, 60, 40} and q/k/v
projected from N(0,1) tokens; DeiT-B at 80% pruning with L_b ~ U{30..48};
the serving regime with p_b = clamp(p + U[-0.1, 0.1], 0, 0.95) and
L_b = 1 + round((1 - p_b) * 196); 384x384 with L_b = 1 + round(r * 576),
r ~ U[0.3, 0.7]; the sweep with round(N(1 + round((1 - p) * 196), 8))
redrawn into [1, 197].  Every mask keeps CLS and exactly L_b tokens, and
every generator is deterministic for its seed."""
import numpy as np
import pytest

import synthetic


def _check_mask(w):
    assert w.keep.shape == (w.B, w.L_full) and w.keep.dtype == np.uint8
    assert set(np.unique(w.keep)) <= {0, 1}
    assert np.all(w.keep[:, 0] == 1)
    assert np.array_equal(w.keep.sum(1), w.lengths)


def _check_qkv(w, dtype):
    assert w.qkv.shape == (w.B, w.L_full, 3, w.H, 64)
    assert w.dtype == dtype
    assert w.qkv.dtype == (np.float32 if dtype == "f32" else (np.float16 if dtype == "f16" else np.uint16))


def test_tiny_batch():
    w = synthetic.tiny("f16")
    assert (w.B, w.L_full, w.H) == (4, 197, 6)
    assert w.lengths.tolist() == [197, 120, 60, 40]
    _check_mask(w)
    _check_qkv(w, "f16")
    assert w.tokens.shape == (4, 197, 384) and w.weights.shape == (3, 384, 384)
    assert abs(float(w.weights.var()) * 384 - 1.0) < 0.02          # W ~ N(0, 1/384)
    # q/k/v are the tokens projected by W (head h = columns 64h..64h+63) in float64,
    # rounded to float32 and stored in the workload's format
    b, j = 1, 57
    ref = np.einsum("c,tcn->tn", w.tokens[b, j].astype(np.float64), w.weights.astype(np.float64))
    got = w.qkv[b, j].astype(np.float64).reshape(3, 384)
    assert np.array_equal(got, ref.astype(np.float32).astype(np.float16).astype(np.float64))


def test_deit_b_pruned80():
    w = synthetic.deit_b_pruned80()
    assert (w.B, w.L_full, w.H) == (32, 197, 12)
    assert w.lengths.min() >= 30 and w.lengths.max() <= 48
    _check_mask(w)
    _check_qkv(w, "bf16")


@pytest.mark.parametrize("B", [1, 2, 4])
@pytest.mark.parametrize("rate", [0.0, 0.25, 0.5, 0.8])
def test_serving_lengths_follow_the_jitter_rule(B, rate):
    w = synthetic.serving(B, rate)
    assert (w.B, w.L_full, w.H) == (B, 197, 6)
    _check_mask(w)
    _check_qkv(w, "f16")
    if rate == 0.0:
        assert np.all(w.lengths == 197)
    else:
        lo = 1 + int(np.floor((1 - min(rate + 0.1, 0.95)) * 196 + 0.5))
        hi = 1 + int(np.floor((1 - max(rate - 0.1, 0.0)) * 196 + 0.5))
        assert np.all((w.lengths >= lo) & (w.lengths <= hi)), (w.lengths, lo, hi)


def test_serving_jitter_spans_its_range():
    rng = synthetic.rng_for(77)
    L = synthetic.serving_lengths(rng, 20000, 0.5)
    # p_b uniform on [0.4, 0.6]: L_b from 1 + round(0.4 * 196) = 79 to 1 + round(0.6 * 196) = 119
    assert L.min() == 79 and L.max() == 119
    assert abs(L.mean() - (1 + 0.5 * 196)) < 0.3


def test_hires_384():
    w = synthetic.hires_384()
    assert (w.B, w.L_full, w.H) == (64, 577, 12)
    assert w.lengths.min() >= 1 + int(0.3 * 576) and w.lengths.max() <= 1 + int(np.ceil(0.7 * 576))
    _check_mask(w)
    _check_qkv(w, "bf16")


@pytest.mark.parametrize("rate", [0.0, 0.3, 0.5, 0.9])
def test_sweep_lengths(rate):
    rng = synthetic.rng_for(91, int(rate * 10))
    L = synthetic.sweep_lengths(rng, 4096, rate)
    assert L.min() >= 1 and L.max() <= 197
    if rate == 0.0:
        assert np.all(L == 197)
        return
    target = 1 + int(np.floor((1 - rate) * 196 + 0.5))
    # sigma 8 around the target; truncation to [1, 197] is far from the target here
    assert abs(L.mean() - target) < 0.5
    assert 7.0 < L.std() < 9.0


def test_sweep_workload_shape():
    w = synthetic.sweep(0.5, B=16)
    assert (w.B, w.L_full, w.H) == (16, 197, 6)
    _check_mask(w)
    _check_qkv(w, "f16")


def test_generators_are_deterministic_and_copies_differ():
    a, b = synthetic.serving(4, 0.5), synthetic.serving(4, 0.5)
    assert np.array_equal(a.qkv, b.qkv) and np.array_equal(a.keep, b.keep)
    c = synthetic.serving(4, 0.5, copy=1)
    assert not np.array_equal(a.qkv, c.qkv)
    assert np.array_equal(synthetic.deit_b_pruned80().keep, synthetic.deit_b_pruned80().keep)


def test_qkv_is_standard_normal():
    w = synthetic.sweep(0.0, B=64)
    x = w.qkv.astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
