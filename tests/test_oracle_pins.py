"""Pins for the CPU oracle: checks against facts that do not come from the oracle.

Each test ties the oracle to something outside itself: a hand-worked example,
a library routine that computes the same quantity on a special case (numpy's
flatnonzero, numpy/torch format widening, torch's fp64 scaled-dot-product
attention on padded inputs), a closed form, or an invariant of softmax
attention.  Paper facts pinned ("Dispatch-Aware Ragged Attention for Pruned
Vision Transformers"):
  - packing survivors into a contiguous ragged buffer and running varlen
    attention equals the padded, masked computation (radpulse sections on
    padding and on the FA2 dispatch ceiling);
  - the kernel is bidirectional, without causal mask or KV cache, so every
    sequence attends to all of its own rows and nothing else ("Bypassing the
    binding");
  - 80% pruning cuts attention FLOPs by 96% (radpulse lead paragraph).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _forced(keep):
    k = (np.asarray(keep) != 0).astype(np.uint8)
    if k.shape[1]:
        k[:, 0] = 1
    return k


# --------------------------------------------------------------------------
# survivor bookkeeping, pack, unpack
# --------------------------------------------------------------------------

def test_hand_example_seqlens_and_pack():
    g = json.load(open(os.path.join(GOLDEN, "pack_hand_example.json")))
    keep = np.array(g["keep"], dtype=np.uint8)
    cu, src = oracle.seqlens(keep)
    assert cu.tolist() == g["cu_seqlens"]
    assert src.tolist() == g["src_idx"]
    dense = np.arange(g["B"] * g["L_full"] * 3, dtype=np.int32).reshape(g["B"], g["L_full"], 3)
    packed, cu2 = oracle.pack(dense, keep)
    assert cu2.tolist() == g["cu_seqlens"]
    assert np.array_equal(packed, dense.reshape(-1, 3)[g["src_idx"]])
    cls = oracle.unpack_cls(packed, cu2)
    assert np.array_equal(cls, dense.reshape(-1, 3)[g["cls_dense_rows"]])
    assert np.array_equal(cls, packed[g["cls_packed_rows"]])


def _random_masks():
    rng = np.random.default_rng(7)
    cases = [
        rng.integers(0, 2, size=(6, 37), dtype=np.uint8),
        np.zeros((3, 11), dtype=np.uint8),                    # only CLS survives
        np.ones((2, 17), dtype=np.uint8),                     # nothing pruned
        rng.integers(0, 4, size=(1, 197), dtype=np.uint8) * 60,  # nonzero bytes != 1
        np.zeros((4, 1), dtype=np.uint8),                     # L_full = 1
        np.zeros((0, 9), dtype=np.uint8),                     # empty batch
        (rng.random((17, 577)) < 0.3).astype(np.uint8),
    ]
    return cases


@pytest.mark.parametrize("keep", _random_masks())
def test_seqlens_matches_flatnonzero(keep):
    cu, src = oracle.seqlens(keep)
    B, L = keep.shape
    forced = _forced(keep)
    # library routine on the flattened forced mask gives the packed source rows
    assert np.array_equal(src, np.flatnonzero(forced.reshape(-1)))
    assert cu[0] == 0 and cu[-1] == forced.sum() == src.shape[0]
    if B:
        assert np.all(np.diff(cu) >= 1)                       # CLS keeps every L_b >= 1
        assert np.array_equal(np.diff(cu), forced.sum(axis=1))


@pytest.mark.parametrize("keep", _random_masks())
def test_pack_unpack_roundtrip(keep):
    B, L = keep.shape
    rng = np.random.default_rng(11)
    dense = rng.integers(0, 2**16, size=(B, L, 24), dtype=np.uint16)
    packed, cu = oracle.pack(dense, keep)
    forced = _forced(keep).astype(bool)
    assert np.array_equal(packed, dense[forced])              # boolean-index library gather
    if B:
        assert np.array_equal(packed[cu[:-1]], dense[:, 0])   # CLS is the first row
        assert np.array_equal(oracle.unpack_cls(packed, cu), dense[:, 0])
    sentinel = np.full_like(dense, 0xDEAD)
    back = oracle.unpack(packed, keep, sentinel)
    assert np.array_equal(back[forced], dense[forced])
    assert np.all(back[~forced] == 0xDEAD)                    # dropped rows untouched


# --------------------------------------------------------------------------
# exact widening of the stored formats
# --------------------------------------------------------------------------

def test_decode_f16_all_bit_patterns():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = oracle.decode(bits.view(np.float16), "f16")
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_decode_bf16_all_bit_patterns():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = oracle.decode(bits, "bf16")
    ref = torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

def _packed_workload(B, L_full, H, lengths, dtype, seed):
    w = synthetic.make_workload("pin", B, L_full, H, lengths, dtype, seed)
    packed, cu = oracle.pack(w.qkv, w.keep)
    return w, packed, cu


def _as_torch64(x, dtype):
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x).astype(np.int16)).view(torch.bfloat16).double()
    return torch.from_numpy(np.ascontiguousarray(x)).double()


def _torch_padded(packed, cu, dtype, scale):
    """Pad every sequence to the longest, mask padded keys, run torch fp64 SDPA."""
    B = cu.shape[0] - 1
    T, _, H, d = packed.shape
    L = np.diff(cu)
    Lmax = int(L.max())
    qkv = _as_torch64(packed, dtype)                          # [T, 3, H, d]
    pad = torch.zeros(B, 3, H, Lmax, d, dtype=torch.float64)
    mask = torch.zeros(B, 1, 1, Lmax, dtype=torch.bool)
    for b in range(B):
        pad[b, :, :, :L[b]] = qkv[cu[b]:cu[b + 1]].permute(1, 2, 0, 3)
        mask[b, ..., :L[b]] = True
    o = torch.nn.functional.scaled_dot_product_attention(
        pad[:, 0], pad[:, 1], pad[:, 2], attn_mask=mask, scale=scale)
    out = np.zeros((T, H, d))
    for b in range(B):
        out[cu[b]:cu[b + 1]] = o[b, :, :L[b]].permute(1, 0, 2).numpy()
    return out


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
def test_attention_equals_padded_masked_sdpa(dtype):
    lengths = [1, 2, 17, 40, 40, 33, 64, 5]
    w, packed, cu = _packed_workload(len(lengths), 64, 3, lengths, dtype, 21)
    got = oracle.attention(packed[:, 0], packed[:, 1], packed[:, 2], cu, dtype, 0.125)
    ref = _torch_padded(packed, cu, dtype, 0.125)
    assert np.max(np.abs(got - ref)) < 1e-12


def test_attention_no_pruning_equals_dense_sdpa():
    B, L, H, d = 3, 97, 2, 64
    w, packed, cu = _packed_workload(B, L, H, [L] * B, "bf16", 5)
    got = oracle.attention(packed[:, 0], packed[:, 1], packed[:, 2], cu, "bf16", 0.125)
    dense = _as_torch64(w.qkv, "bf16")                        # [B, L, 3, H, d]
    o = torch.nn.functional.scaled_dot_product_attention(
        dense[:, :, 0].transpose(1, 2), dense[:, :, 1].transpose(1, 2),
        dense[:, :, 2].transpose(1, 2), scale=0.125)          # [B, H, L, d]
    ref = o.transpose(1, 2).reshape(B * L, H, d).numpy()
    assert np.max(np.abs(got - ref)) < 1e-12


def _f64_seq(q, k, v):
    """Single sequence, single head, float64 storage: arrays [L, 1, d]."""
    L = q.shape[0]
    cu = np.array([0, L], dtype=np.int32)
    return oracle.attention(q, k, v, cu, "f64", 0.125)


def test_weights_sum_to_one():
    rng = np.random.default_rng(3)
    for L in (1, 3, 50, 577):
        q = rng.standard_normal((L, 1, 64)) * 3
        k = rng.standard_normal((L, 1, 64)) * 3
        for c in (1.0, -2.5):
            v = np.full((L, 1, 64), c)
            assert np.max(np.abs(_f64_seq(q, k, v) - c)) < 1e-13


def test_closed_forms():
    rng = np.random.default_rng(4)
    d = 64
    # L = 1: the only weight is 1, output equals v
    q, k, v = (rng.standard_normal((1, 1, d)) for _ in range(3))
    assert np.max(np.abs(_f64_seq(q, k, v) - v)) < 1e-15
    # q = 0 or all keys equal: uniform weights, output is the mean of v
    L = 13
    v = rng.standard_normal((L, 1, d))
    k = rng.standard_normal((L, 1, d))
    out = _f64_seq(np.zeros((L, 1, d)), k, v)
    assert np.max(np.abs(out - v.mean(axis=0))) < 1e-14
    kk = np.repeat(rng.standard_normal((1, 1, d)), L, axis=0)
    out = _f64_seq(rng.standard_normal((L, 1, d)), kk, v)
    assert np.max(np.abs(out - v.mean(axis=0))) < 1e-14
    # L = 2: o_1 = sigmoid(s11 - s12) v1 + sigmoid(s12 - s11) v2
    q, k, v = (rng.standard_normal((2, 1, d)) for _ in range(3))
    s = 0.125 * (q[:, 0] @ k[:, 0].T)
    sig = lambda x: 1.0 / (1.0 + math.exp(-x))
    for i in range(2):
        expect = sig(s[i, 0] - s[i, 1]) * v[0, 0] + sig(s[i, 1] - s[i, 0]) * v[1, 0]
        assert np.max(np.abs(_f64_seq(q, k, v)[i, 0] - expect)) < 1e-14


def test_hand_example_attention():
    g = json.load(open(os.path.join(GOLDEN, "attention_hand_example.json")))
    num = lambda x: math.log(3.0) if x == "ln3" else float(x)
    q = np.array([[num(x) for x in r] for r in g["q"]])[:, None, :]
    k = np.array([[num(x) for x in r] for r in g["k"]])[:, None, :]
    v = np.array([[num(x) for x in r] for r in g["v"]])[:, None, :]
    cu = np.array([0, 2], dtype=np.int32)
    out = oracle.attention(q, k, v, cu, "f64", g["scale"])
    assert np.max(np.abs(out[:, 0] - np.array(g["out"]))) < 1e-14


def test_brute_force_tiny_lengths():
    """L <= 4 against exp/sum without max subtraction, in Python loops."""
    rng = np.random.default_rng(9)
    for L in (1, 2, 3, 4):
        q, k, v = (rng.standard_normal((L, 1, 8)) for _ in range(3))
        cu = np.array([0, L], dtype=np.int32)
        got = oracle.attention(q, k, v, cu, "f64", 0.3)
        for i in range(L):
            w = [math.exp(0.3 * sum(q[i, 0, c] * k[j, 0, c] for c in range(8))) for j in range(L)]
            z = sum(w)
            for c in range(8):
                assert abs(got[i, 0, c] - sum(w[j] * v[j, 0, c] for j in range(L)) / z) < 1e-14


def test_permutation_equivariance_and_independence():
    lengths = [30, 45, 12]
    w, packed, cu = _packed_workload(3, 64, 2, lengths, "f16", 17)
    base = oracle.attention(packed[:, 0], packed[:, 1], packed[:, 2], cu, "f16")
    # permuting the rows of sequence 1 permutes its output rows the same way
    perm = np.random.default_rng(1).permutation(lengths[1])
    p2 = packed.copy()
    p2[cu[1]:cu[2]] = packed[cu[1]:cu[2]][perm]
    out = oracle.attention(p2[:, 0], p2[:, 1], p2[:, 2], cu, "f16")
    assert np.array_equal(out[cu[1]:cu[2]], base[cu[1]:cu[2]][perm]) or \
        np.max(np.abs(out[cu[1]:cu[2]] - base[cu[1]:cu[2]][perm])) < 1e-14
    # changing sequences 0 and 2 leaves sequence 1 bit-identical
    p3 = packed.copy()
    p3[cu[0]:cu[1]] = np.float16(3.0)
    p3[cu[2]:cu[3]] = -p3[cu[2]:cu[3]]
    out = oracle.attention(p3[:, 0], p3[:, 1], p3[:, 2], cu, "f16")
    assert np.array_equal(out[cu[1]:cu[2]], base[cu[1]:cu[2]])


def test_key_shift_invariance_and_convex_hull():
    rng = np.random.default_rng(12)
    L = 40
    q, k, v = (rng.standard_normal((L, 1, 64)) for _ in range(3))
    base = _f64_seq(q, k, v)
    shifted = _f64_seq(q, k + rng.standard_normal((1, 1, 64)), v)  # s_ij += q_i . c
    assert np.max(np.abs(shifted - base)) < 1e-12
    assert np.all(base[:, 0] <= v[:, 0].max(axis=0) + 1e-15)
    assert np.all(base[:, 0] >= v[:, 0].min(axis=0) - 1e-15)


def test_strides_subset_and_threads():
    w = synthetic.tiny("f16")
    packed, cu = oracle.pack(w.qkv, w.keep)
    full = oracle.attention(packed[:, 0], packed[:, 1], packed[:, 2], cu, "f16", threads=1)
    # separate contiguous q/k/v arrays give the same numbers as fused views
    sep = oracle.attention(np.ascontiguousarray(packed[:, 0]), np.ascontiguousarray(packed[:, 1]),
                           np.ascontiguousarray(packed[:, 2]), cu, "f16", threads=4)
    assert np.array_equal(full, sep)
    sub = oracle.attention(packed[:, 0], packed[:, 1], packed[:, 2], cu, "f16", seqs=[3, 1])
    for b in (1, 3):
        assert np.array_equal(sub[cu[b]:cu[b + 1]], full[cu[b]:cu[b + 1]])
    assert np.all(sub[cu[0]:cu[1]] == 0) and np.all(sub[cu[2]:cu[3]] == 0)


def test_flop_accounting_quadratic():
    """80% pruning of 197 tokens cuts attention FLOPs by 1 - 0.2^2 = 96%."""
    L = 10_000  # a length divisible by 5 so 20% survive exactly
    full = synthetic.Workload("a", 1, L, 1, 64, "f16", np.array([L]), None, None)
    pruned = synthetic.Workload("b", 1, L, 1, 64, "f16", np.array([L // 5]), None, None)
    assert full.useful_flops() == 4 * 64 * L * L
    assert abs(1 - pruned.useful_flops() / full.useful_flops() - 0.96) < 1e-12
