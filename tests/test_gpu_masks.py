"""GPU parity of the device-side keep-mask producers against the CPU oracle.

Readings (the pages name Threshold-l2 among the pruning methods the pipeline
serves, radpulse "Integrated pack pipeline"; the rules are not spelled out):
Threshold-l2 keeps a token whose feature norm is >= tau; top-k keeps CLS and
the k_b - 1 highest-scoring other tokens (ties: lower index, NaN last).  Masks,
cu_seqlens and packed rows are integer / byte results: bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle
import ragged_variable_length_b200 as rv
import synthetic
from helpers import to_device, to_host_bits

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("B,L,C", [(4, 197, 384), (3, 577, 768), (2, 33, 70)])
def test_mask_l2_matches_oracle(dtype, B, L, C):
    rng = synthetic.rng_for(3001, B * 1000 + C)
    x = synthetic.store(rng.standard_normal((B, L, C)).astype(np.float32), dtype)
    xf = oracle.decode(x, dtype).reshape(B, L, C)
    norms = np.sqrt((xf * xf).sum(2))
    for tau in (float(np.median(norms)), float(norms.min()), float(norms.max()), 0.0):
        got = rv.ragged_mask_l2(to_device(x, dtype), tau).cpu().numpy()
        assert np.array_equal(got, oracle.mask_l2(x, dtype, tau)), tau


def test_mask_l2_at_the_threshold():
    x = np.zeros((1, 5, 64), dtype=np.float32)
    x[0, 1, 0], x[0, 1, 40] = 3.0, 4.0
    x[0, 2, 7], x[0, 2, 39] = 5.0, 12.0
    x[0, 3, 0] = np.nextafter(np.float32(5.0), np.float32(0.0))
    x[0, 4, :] = 0.625
    for tau in (5.0, 13.0):
        got = rv.ragged_mask_l2(torch.from_numpy(x).cuda(), tau).cpu().numpy()
        assert np.array_equal(got, oracle.mask_l2(x, "f32", tau))
    assert rv.ragged_mask_l2(torch.from_numpy(x).cuda(), 5.0).cpu().tolist() == [[1, 1, 1, 0, 1]]


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
def test_mask_l2_exact_at_and_next_to_each_norm(dtype):
    """Each token's own norm as tau (the double nearest it, and one ulp either
    side), so every decision falls in the band where the kernel's fp64 sum
    cannot decide and its exact integer sum must: bit-exact against the oracle."""
    rng = synthetic.rng_for(3007, ["f16", "bf16", "f32"].index(dtype))
    B, L, C = 2, 12, 384
    x = synthetic.store(rng.standard_normal((B, L, C)).astype(np.float32), dtype)
    xf = oracle.decode(x, dtype).reshape(B, L, C)
    xd = to_device(x, dtype)
    norms = np.sqrt((xf * xf).sum(2))
    for b in range(B):
        for j in (1, 5, 11):
            t0 = float(norms[b, j])
            for tau in (float(np.nextafter(t0, 0.0)), t0, float(np.nextafter(t0, np.inf))):
                got = rv.ragged_mask_l2(xd, tau).cpu().numpy()
                assert np.array_equal(got, oracle.mask_l2(x, dtype, tau)), (b, j, tau)


def test_mask_l2_where_fp64_sums_round_subnormals_nan_inf():
    x = np.zeros((1, 8, 64), dtype=np.float32)
    x[0, 1, :4] = [1.0, 2.0 ** -26, 2.0 ** -26, 2.0 ** -52]     # sum of squares (1 + 2^-52)^2 exactly
    x[0, 2, 0] = 1.0
    x[0, 2, 1:17] = 2.0 ** -30                                   # 1 + 2^-56
    x[0, 3, 3] = 2.0 ** -149                                     # square 2^-298
    x[0, 4, 0], x[0, 4, 63] = 2.0 ** -149, 2.0 ** -149
    x[0, 5, 0], x[0, 5, 1] = np.nan, 100.0
    x[0, 6, 2] = -np.inf
    x[0, 7, :] = 0.625                                           # norm 5 exactly
    xd = torch.from_numpy(x).cuda()
    for tau in (1.0 + 2.0 ** -52, float(np.nextafter(1.0 + 2.0 ** -52, 2.0)), 1.0, float(np.nextafter(1.0, 2.0)),
                2.0 ** -149, float(np.nextafter(2.0 ** -149, 1.0)), 2.0 ** -149 * 2 ** 0.5, 5.0, 1e-300, 1e300,
                float("inf"), 0.0, -1.0):
        got = rv.ragged_mask_l2(xd, tau).cpu().numpy()
        assert np.array_equal(got, oracle.mask_l2(x, "f32", tau)), tau


def test_mask_l2_on_a_strided_view():
    """Norm of the q part of a dense fused [B, L, 3, H, 64] buffer (token stride 3 * H * 64)."""
    w = synthetic.serving(4, 0.0)
    dense = to_device(w.qkv, w.dtype)                       # [B, L, 3, H, 64]
    q = dense.view(w.B, w.L_full, 3 * w.H * 64)[:, :, :w.H * 64]
    qn = w.qkv[:, :, 0].reshape(w.B, w.L_full, w.H * 64)
    norms = np.sqrt((oracle.decode(np.ascontiguousarray(qn), w.dtype).reshape(qn.shape) ** 2).sum(2))
    tau = float(np.median(norms))
    got = rv.ragged_mask_l2(q, tau).cpu().numpy()
    assert np.array_equal(got, oracle.mask_l2(np.ascontiguousarray(qn), w.dtype, tau))


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_mask_l2_vector_path_special_values(dtype):
    """16-bit rows on 16-byte boundaries take the vector path (fp32 squares,
    two-sum accumulation): tokens whose sum it cannot trust (NaN, an infinite
    element, bf16 squares above or below fp32's range, all zeros) go back to the
    fp64 sum, and a near-tie still reaches the exact comparison."""
    big, tiny = (2.0 ** 70, 2.0 ** -80) if dtype == "bf16" else (65504.0, 2.0 ** -24)
    x = np.zeros((1, 10, 64), dtype=np.float32)
    x[0, 1, :3] = big                          # bf16: squares overflow fp32
    x[0, 2, :40] = tiny                        # bf16: squares underflow fp32
    x[0, 3, 0] = 1.0
    x[0, 3, 1:33] = 2.0 ** -70 if dtype == "bf16" else 2.0 ** -24    # 1 plus tiny squares
    x[0, 4, 5], x[0, 4, 6] = np.nan, 3.0
    x[0, 5, 9] = np.inf
    x[0, 7, :] = 0.625                         # norm 5 exactly
    x[0, 8, :] = -0.625
    x[0, 9, ::2] = 1.5
    xs = synthetic.store(x, dtype)
    xd = to_device(xs, dtype)
    xf = oracle.decode(xs, dtype).reshape(1, 10, 64)
    norms = np.sqrt((xf.astype(np.float64) ** 2).sum(2))
    taus = [0.0, -1.0, 5.0, float(np.nextafter(5.0, 0.0)), float(np.nextafter(5.0, 6.0)), 1.0,
            float(np.nextafter(1.0, 2.0)), float(big), float(tiny), 1e-300, 1e300, float("inf")]
    taus += [float(v) for v in norms[0] if np.isfinite(v) and v > 0]
    for tau in taus:
        got = rv.ragged_mask_l2(xd, tau).cpu().numpy()
        assert np.array_equal(got, oracle.mask_l2(xs, dtype, tau)), tau


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_mask_l2_rows_off_16_byte_boundaries(dtype):
    """A view starting one element into its buffer (rows on 2-byte boundaries)
    takes the per-element path; both paths give the oracle's mask."""
    rng = synthetic.rng_for(3011, ["f16", "bf16"].index(dtype))
    B, L, C = 3, 50, 128
    x = synthetic.store(rng.standard_normal((B, L, C + 8)).astype(np.float32), dtype)
    full = to_device(x, dtype)                                 # [B, L, C + 8]
    for off in (0, 1):
        view = full[:, :, off:off + C]
        xs = np.ascontiguousarray(x[:, :, off:off + C])
        xf = oracle.decode(xs, dtype).reshape(B, L, C)
        tau = float(np.median(np.sqrt((xf.astype(np.float64) ** 2).sum(2))))
        got = rv.ragged_mask_l2(view, tau).cpu().numpy()
        assert np.array_equal(got, oracle.mask_l2(xs, dtype, tau)), off


def _topk_case(rng, B, L, ties, nans):
    s = rng.standard_normal((B, L)).astype(np.float32)
    if ties:
        s = np.round(s * 2) / 2
    if nans:
        s[rng.random((B, L)) < 0.1] = np.nan
    k = rng.integers(-3, L + 4, size=B).astype(np.int32)
    k[:2] = [1, L]
    return s, k


@pytest.mark.parametrize("B,L,H,dtype", [(4, 197, 6, "f16"), (32, 197, 12, "bf16"), (64, 577, 12, "bf16"),
                                         (3, 40, 2, "f16")])
@pytest.mark.parametrize("ties,nans", [(False, False), (True, True)])
def test_pack_topk_matches_oracle(B, L, H, dtype, ties, nans):
    rng = synthetic.rng_for(3002, B * 100 + int(ties) * 2 + int(nans))
    s, k = _topk_case(rng, B, L, ties, nans)
    qkv = synthetic.store(rng.standard_normal((B, L, 3, H, 64)).astype(np.float32), dtype)
    dense = to_device(qkv, dtype)
    keep_out = torch.full((B, L), 7, dtype=torch.uint8, device="cuda")
    src_idx = torch.full((B * L,), -1, dtype=torch.int32, device="cuda")
    packed, cu = rv.ragged_pack_topk(dense, torch.from_numpy(s).cuda(), torch.from_numpy(k).cuda(),
                                     src_idx=src_idx, keep_out=keep_out)
    torch.cuda.synchronize()
    keep_ref = oracle.mask_topk(s, k)
    assert np.array_equal(keep_out.cpu().numpy(), keep_ref)
    packed_ref, cu_ref = oracle.pack(qkv, keep_ref)
    cu_h = cu.cpu().numpy()
    assert np.array_equal(cu_h, cu_ref)
    T = int(cu_h[-1])
    assert np.array_equal(to_host_bits(packed[:T], dtype), packed_ref)
    src_ref = np.concatenate([b * L + np.flatnonzero(keep_ref[b]) for b in range(B)])
    assert np.array_equal(src_idx[:T].cpu().numpy(), src_ref)


def test_pack_topk_then_attention():
    """Selection, pack and attention chain: the attention of the top-k packed
    rows equals the oracle's attention of the oracle's selection."""
    rng = synthetic.rng_for(3003)
    B, L, H = 8, 197, 6
    s, _ = _topk_case(rng, B, L, False, False)
    k = rng.integers(20, 120, size=B).astype(np.int32)
    w = synthetic.make_workload("topk_chain", B, L, H, k, "f16", 3004)
    packed, cu = rv.ragged_pack_topk(to_device(w.qkv, "f16"), torch.from_numpy(s).cuda(), torch.from_numpy(k).cuda())
    out = rv.ragged_attn_fwd(packed[:, 0], packed[:, 1], packed[:, 2], cu, L, 0.125)
    torch.cuda.synchronize()
    keep_ref = oracle.mask_topk(s, k)
    packed_ref, cu_ref = oracle.pack(w.qkv, keep_ref)
    ref = oracle.attention(packed_ref[:, 0], packed_ref[:, 1], packed_ref[:, 2], cu_ref, "f16", 0.125)
    T = int(cu_ref[-1])
    got = out[:T].double().cpu().numpy()
    assert np.abs(got - ref).max() <= 4e-3


def _special_scores(rng, B, L):
    """Scores drawn from the values where a sort key could go wrong: both
    zeros, denormals of both signs, infinities, the extreme finite values and
    NaNs of several payloads and both signs, mixed with ordinary numbers."""
    bits = np.array([0x00000000, 0x80000000, 0x00000001, 0x80000001, 0x007fffff, 0x807fffff,
                     0x7f800000, 0xff800000, 0x7f7fffff, 0xff7fffff, 0x7fc00000, 0xffc00000,
                     0x7f800001, 0xffffffff, 0x3f800000, 0xbf800000], dtype=np.uint32)
    pick = bits[rng.integers(0, bits.size, size=(B, L))].view(np.float32)
    s = np.where(rng.random((B, L)) < 0.6, pick, rng.standard_normal((B, L)).astype(np.float32))
    return np.ascontiguousarray(s.astype(np.float32))


@pytest.mark.parametrize("B,L", [(6, 197), (4, 256), (4, 257), (3, 2), (5, 1), (2, 4097), (2, 8192)])
def test_pack_topk_special_values(B, L):
    """Total order on signed zeros (tie), denormals (distinct from zero),
    infinities and NaN payloads (all tie, below -inf), at lengths on and just
    past a power of two and at the largest supported length."""
    rng = synthetic.rng_for(3005, B * 10000 + L)
    s = _special_scores(rng, B, L)
    k = rng.integers(1, L + 1, size=B).astype(np.int32)
    row = 32
    dense_h = rng.integers(0, 256, size=(B, L, row), dtype=np.uint8)
    keep_out = torch.full((B, L), 7, dtype=torch.uint8, device="cuda")
    packed, cu = rv.ragged_pack_topk(torch.from_numpy(dense_h).cuda(), torch.from_numpy(s).cuda(),
                                     torch.from_numpy(k).cuda(), keep_out=keep_out)
    torch.cuda.synchronize()
    keep_ref = oracle.mask_topk(s, k)
    assert np.array_equal(keep_out.cpu().numpy(), keep_ref)
    assert np.array_equal(keep_ref.sum(1), k)
    cu_h = cu.cpu().numpy()
    assert np.array_equal(cu_h, np.concatenate([[0], np.cumsum(k)]))
    T = int(cu_h[-1])
    rows = np.concatenate([dense_h[b][keep_ref[b].astype(bool)] for b in range(B)])
    assert np.array_equal(packed[:T].cpu().numpy(), rows)


def test_mask_l2_more_images_than_one_launch_holds():
    """B above the 65,535 images one launch covers: the host splits the batch."""
    rng = synthetic.rng_for(3006)
    B, L, C = 70001, 2, 8
    x = rng.standard_normal((B, L, C)).astype(np.float32)
    tau = 2.5
    got = rv.ragged_mask_l2(torch.from_numpy(x).cuda(), tau).cpu().numpy()
    assert np.array_equal(got, oracle.mask_l2(x, "f32", tau))
