"""GPU parity of ragged attention against the fp64 CPU oracle, through the C ABI.

Bar: max-abs error <= 4e-3 for f16 / bf16 inputs (fp32 accumulation, output
rounded to the input format), and max |gpu - oracle| <= 1e-5 max |oracle| on
the fp32 check path.  Small cases are compared element by element; the full
workloads are compared on sampled sequences (always including the shortest
and the longest), in the same launch configuration the benchmark times.
"""
import numpy as np
import pytest
import torch

import oracle
import ragged_variable_length_b200 as rv
import synthetic
from helpers import TOL_16BIT, ulps_from_rounded, TORCH_DTYPE, attn_error, to_device, to_f64

pytestmark = pytest.mark.gpu


KERNELS = {"auto": rv.RAGGED_ATTN_AUTO, "streaming": rv.RAGGED_ATTN_STREAMING,
           "resident": rv.RAGGED_ATTN_RESIDENT, "tcgen05": rv.RAGGED_ATTN_TCGEN05,
           "persistent": rv.RAGGED_ATTN_PERSISTENT}
TC05 = ["tcgen05", "persistent"]


def run_pipeline(w, separate_qkv=False, out_pad=0, max_seqlen=None, kernel="auto"):
    """Device pack -> attend (with fused CLS) for a synthetic workload, with
    the given attention kernel (the fp32 check path has a single kernel)."""
    dense = to_device(w.qkv, w.dtype)
    keep = torch.from_numpy(w.keep).cuda()
    packed, cu = rv.ragged_pack(dense, keep)
    T_cap = w.B * w.L_full
    out_full = torch.full((T_cap, w.H * w.d + out_pad), float("nan"), dtype=TORCH_DTYPE[w.dtype], device="cuda")
    out = out_full[:, :w.H * w.d].view(T_cap, w.H, w.d) if out_pad == 0 else \
        out_full.as_strided((T_cap, w.H, w.d), (w.H * w.d + out_pad, w.d, 1))
    cls = torch.full((w.B, w.H, w.d), float("nan"), dtype=TORCH_DTYPE[w.dtype], device="cuda")
    if separate_qkv:
        q, k, v = (packed[:, i].contiguous() for i in range(3))
    else:
        q, k, v = packed[:, 0], packed[:, 1], packed[:, 2]
    prev = rv.ragged_set_attn_kernel(KERNELS[kernel])
    try:
        rv.ragged_attn_fwd(q, k, v, cu, max_seqlen or w.L_full, w.scale, out=out, cls_out=cls)
    finally:
        rv.ragged_set_attn_kernel(prev)
    torch.cuda.synchronize()
    assert rv.ragged_get_device_status() == 0
    return cu.cpu().numpy(), out, cls, out_full


def sample_sequences(lengths, n, seed=0):
    L = np.asarray(lengths)
    pick = {int(np.argmin(L)), int(np.argmax(L))}
    rng = np.random.default_rng(seed)
    while len(pick) < min(n, len(L)):
        pick.add(int(rng.integers(0, len(L))))
    return sorted(pick)


def check_against_oracle(w, seqs=None, **kw):
    cu, out, cls, out_full = run_pipeline(w, **kw)
    packed_o, cu_o = oracle.pack(w.qkv, w.keep)
    assert np.array_equal(cu, cu_o)
    ref = oracle.attention(packed_o[:, 0], packed_o[:, 1], packed_o[:, 2], cu_o, w.dtype, w.scale, seqs=seqs)
    T = int(cu[-1])
    got = to_f64(out[:T])
    rows = np.concatenate([np.arange(cu[b], cu[b + 1]) for b in (seqs if seqs is not None else range(w.B))])
    err, bound = attn_error(got[rows], ref[rows], w.dtype)
    assert err <= bound, f"{w.name} {w.dtype}: error {err:.3e} above {bound:.3e}"
    assert not torch.isnan(out[:T]).any()
    # rows past T are left as they were
    assert torch.isnan(out_full[T:]).all()
    # fused CLS equals the first row of every sequence, bit for bit
    assert torch.equal(cls, out[torch.from_numpy(cu[:-1]).long().cuda()])
    return err


KERNEL_CASES = [("f16", k) for k in KERNELS] + [("bf16", k) for k in KERNELS] + [("f32", "auto")]


@pytest.mark.parametrize("dtype,kernel", KERNEL_CASES)
def test_tiny_all_elements(dtype, kernel):
    check_against_oracle(synthetic.tiny(dtype), kernel=kernel)


@pytest.mark.parametrize("dtype,kernel", KERNEL_CASES)
def test_tile_edge_lengths(dtype, kernel):
    lengths = [1, 2, 15, 16, 17, 31, 32, 33, 63, 64, 65, 127, 128, 129, 191, 192, 193, 200]
    w = synthetic.make_workload("edges", len(lengths), 200, 3, lengths, dtype, 77)
    check_against_oracle(w, kernel=kernel)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_streaming_kernel_under_a_loose_bound(dtype):
    """A max_seqlen far above the longest sequence only sizes the launch."""
    lengths = [1, 2, 63, 64, 65, 128, 129, 200]
    w = synthetic.make_workload("edges_loose", len(lengths), 200, 3, lengths, dtype, 76)
    check_against_oracle(w, max_seqlen=1000)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("kernel", ["auto", "streaming"])
def test_long_sequences_above_the_resident_limit(dtype, kernel):
    """L_full above the resident limit (640 keys): the streaming kernel, and
    AUTO (which picks a tcgen05 kernel for sequences over 256 keys)."""
    w = synthetic.make_workload("long", 4, 1000, 2, [1000, 700, 641, 65], dtype, 81)
    check_against_oracle(w, kernel=kernel)


def test_kernel_limits_are_reported():
    """The kernel that holds whole sequences refuses launches longer than 640 keys."""
    w = synthetic.make_workload("too_long", 1, 700, 1, [700], "f16", 82)
    with pytest.raises(rv.RaggedError, match="640"):
        run_pipeline(w, kernel="resident")


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("kernel", TC05)
def test_long_sequences_tcgen05(dtype, kernel):
    """The tcgen05 kernels stream K/V, so they take sequences of any length."""
    w = synthetic.make_workload("long_tc", 4, 1000, 2, [1000, 700, 641, 65], dtype, 83)
    check_against_oracle(w, kernel=kernel)


@pytest.mark.parametrize("kernel", TC05)
def test_tcgen05_rescale_path(kernel):
    """Keys whose logits jump by far more than the rescale threshold after the
    first tile force the in-TMEM rescaling of O."""
    w = synthetic.make_workload("jump", 3, 300, 2, [300, 200, 129], "f16", 84)
    q = w.qkv[:, :, 0].astype(np.float32)
    k = w.qkv[:, :, 1].astype(np.float32)
    k[:, 150:, :, :] = (k[:, 150:, :, :] * 6.0)          # later keys: logits up to ~6x larger
    q *= 2.0
    w.qkv = w.qkv.copy()
    w.qkv[:, :, 0] = q.astype(np.float16)
    w.qkv[:, :, 1] = k.astype(np.float16)
    check_against_oracle(w, kernel=kernel)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("kernel", list(KERNELS))
def test_hires_lengths_448_449_576_577_640(dtype, kernel):
    """Lengths around whole key tiles (448 = 7 x 64, 576 = 9 x 64), the 577 tokens of a 384x384 ViT, and the resident limit (640)."""
    w = synthetic.make_workload("hires_edges", 6, 640, 2, [577, 576, 300, 640, 448, 449], dtype, 78)
    check_against_oracle(w, kernel=kernel)


@pytest.mark.parametrize("kernel", list(KERNELS))
def test_deit_b_pruned80_all_sequences(kernel):
    check_against_oracle(synthetic.deit_b_pruned80(), kernel=kernel)


@pytest.mark.parametrize("B", synthetic.SERVING_BATCHES)
@pytest.mark.parametrize("rate", synthetic.SERVING_RATES)
def test_serving_all_sequences(B, rate):
    check_against_oracle(synthetic.serving(B, rate))


# Full-size workloads, every sequence and head element by element.  The fp64
# oracle for a workload is computed once and shared by the kernels.
_FULL_REF = {}


def _full_reference(w):
    if w.name not in _FULL_REF:
        packed_o, cu_o = oracle.pack(w.qkv, w.keep)
        _FULL_REF[w.name] = (cu_o, oracle.attention(packed_o[:, 0], packed_o[:, 1], packed_o[:, 2], cu_o, w.dtype,
                                                    w.scale))
    return _FULL_REF[w.name]


def check_full(w, kernel):
    cu, out, cls, out_full = run_pipeline(w, kernel=kernel)
    cu_o, ref = _full_reference(w)
    assert np.array_equal(cu, cu_o)
    T = int(cu[-1])
    got = to_f64(out[:T])
    err, bound = attn_error(got, ref[:T], w.dtype)
    assert err <= bound, f"{w.name} {kernel}: error {err:.3e} above {bound:.3e}"
    # The plain reading of the bar: max-abs 4e-3 everywhere except where the
    # output format alone forces more (bf16 values of magnitude 2 or more,
    # whose half-ulp is 3.9e-3 or more).
    over = np.abs(got - ref[:T]) > TOL_16BIT
    if w.dtype == "f16":
        assert not over.any(), f"{w.name} {kernel}: plain max-abs error above 4e-3"
    else:
        assert np.all(np.abs(ref[:T][over]) >= 2.0), f"{w.name} {kernel}: plain error above 4e-3 below magnitude 2"
        ulps = ulps_from_rounded(got, ref[:T], "bf16")
        assert ulps <= 1, f"{w.name} {kernel}: {ulps} bf16 ulps from the correctly rounded result"
    assert torch.isnan(out_full[T:]).all()
    assert torch.equal(cls, out[torch.from_numpy(cu[:-1]).long().cuda()])


@pytest.mark.parametrize("kernel", ["auto", "persistent", "tcgen05", "streaming"])
def test_hires_384_every_sequence(kernel):
    check_full(synthetic.hires_384(), kernel)


@pytest.mark.parametrize("rate", [0.0, 0.5, 0.9])
@pytest.mark.parametrize("kernel", ["auto", "persistent", "tcgen05", "streaming"])
def test_sweep_b512_every_sequence(rate, kernel):
    check_full(synthetic.sweep(rate), kernel)


def test_deit_b_pruned80_bf16_within_one_ulp_of_the_rounded_oracle():
    w = synthetic.deit_b_pruned80()
    cu, out, _, _ = run_pipeline(w)
    cu_o, ref = _full_reference(w)
    T = int(cu[-1])
    assert ulps_from_rounded(to_f64(out[:T]), ref[:T], "bf16") <= 1


@pytest.mark.parametrize("dtype,kernel", KERNEL_CASES)
def test_separate_qkv_and_padded_output_rows(dtype, kernel):
    w = synthetic.make_workload("layout", 5, 130, 4, [130, 1, 64, 65, 99], dtype, 79)
    check_against_oracle(w, separate_qkv=True, out_pad=64 if dtype != "f32" else 32, kernel=kernel)


@pytest.mark.parametrize("dtype,kernel", KERNEL_CASES)
def test_deterministic(dtype, kernel):
    w = synthetic.make_workload("det", 6, 197, 6, [197, 40, 88, 3, 150, 64], dtype, 80)
    _, out1, cls1, _ = run_pipeline(w, kernel=kernel)
    _, out2, cls2, _ = run_pipeline(w, kernel=kernel)
    T = int(w.lengths.sum())
    assert torch.equal(out1[:T], out2[:T]) and torch.equal(cls1, cls2)


@pytest.mark.parametrize("kernel", list(KERNELS))
def test_bad_cu_seqlens_are_flagged_and_skipped(kernel):
    H, d = 2, 64
    q = torch.randn(100, H, d, device="cuda", dtype=torch.float16)
    out = torch.full((100, H, d), 7.0, dtype=torch.float16, device="cuda")
    rv.ragged_get_device_status()
    # sequence 0 is longer than the host bound; sequence 1 has a negative length
    cu = torch.tensor([0, 80, 60], dtype=torch.int32, device="cuda")
    prev = rv.ragged_set_attn_kernel(KERNELS[kernel])
    try:
        rv.ragged_attn_fwd(q, q, q, cu, max_seqlen=64, out=out)
    finally:
        rv.ragged_set_attn_kernel(prev)
    assert rv.ragged_get_device_status() & rv.RAGGED_DEV_BAD_SEQLENS
    assert torch.all(out == 7.0)
    assert rv.ragged_get_device_status() == 0     # reading clears the word


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_persistent_flags_sequences_past_its_tensor_maps(dtype):
    """cu_seqlens shifted by 100 rows (cu[0] != 0): the persistent kernel's TMA
    maps cover rows [0, B * max_seqlen), so the last sequence, which ends past
    them, is flagged and left untouched; the others are still correct."""
    B, H, L = 4, 2, 197
    rng = np.random.default_rng(88)
    rows = 100 + B * L
    qkv = synthetic.store(rng.standard_normal((rows, 3, H, 64)).astype(np.float32), dtype)
    dev = to_device(qkv, dtype)
    cu_h = np.array([100 + i * L for i in range(B + 1)], dtype=np.int32)
    cu = torch.from_numpy(cu_h).cuda()
    out = torch.full((rows, H, 64), float("nan"), dtype=TORCH_DTYPE[dtype], device="cuda")
    rv.ragged_get_device_status()
    prev = rv.ragged_set_attn_kernel(rv.RAGGED_ATTN_PERSISTENT)
    try:
        rv.ragged_attn_fwd(dev[:, 0], dev[:, 1], dev[:, 2], cu, L, 0.125, out=out)
    finally:
        rv.ragged_set_attn_kernel(prev)
    torch.cuda.synchronize()
    assert rv.ragged_get_device_status() & rv.RAGGED_DEV_BAD_SEQLENS
    assert torch.isnan(out[:100]).all() and torch.isnan(out[int(cu_h[3]):]).all()
    ref = oracle.attention(qkv[:, 0], qkv[:, 1], qkv[:, 2], cu_h, dtype, 0.125, seqs=[0, 1, 2])
    got = to_f64(out[100:int(cu_h[3])])
    err, bound = attn_error(got, ref[100:int(cu_h[3])], dtype)
    assert err <= bound, f"{err:.3e} > {bound:.3e}"


def test_pipeline_call_and_graph_replay_match_separate_calls():
    w = synthetic.serving(4, 0.25)
    cu_ref, out_ref, cls_ref, _ = run_pipeline(w)
    p = rv.Pipeline(w.B, w.L_full, w.H, torch.float16)
    p.dense_qkv.copy_(to_device(w.qkv, "f16"))
    p.keep.copy_(torch.from_numpy(w.keep))
    p()
    torch.cuda.synchronize()
    T = int(cu_ref[-1])
    assert np.array_equal(p.cu_seqlens.cpu().numpy(), cu_ref)
    assert torch.equal(p.out[:T], out_ref[:T]) and torch.equal(p.cls_out, cls_ref)
    p.cls_out.zero_()
    p.capture()
    p.replay()
    torch.cuda.synchronize()
    assert torch.equal(p.cls_out, cls_ref)
    # new inputs written into the same buffers are picked up by the replay
    w2 = synthetic.serving(4, 0.25, copy=1)
    p.dense_qkv.copy_(to_device(w2.qkv, "f16"))
    p.keep.copy_(torch.from_numpy(w2.keep))
    p.replay()
    torch.cuda.synchronize()
    _, out2, cls2, _ = run_pipeline(w2)
    assert torch.equal(p.cls_out, cls2)


def test_ragged_pipeline_binding():
    w = synthetic.deit_b_pruned80()
    cu_ref, out_ref, cls_ref, _ = run_pipeline(w)
    packed, cu, out, cls = rv.ragged_pipeline(to_device(w.qkv, w.dtype), torch.from_numpy(w.keep).cuda())
    torch.cuda.synchronize()
    T = int(cu_ref[-1])
    assert np.array_equal(cu.cpu().numpy(), cu_ref)
    assert torch.equal(out[:T], out_ref[:T]) and torch.equal(cls, cls_ref)


@pytest.mark.parametrize("kernel", list(KERNELS))
def test_zero_length_sequences(kernel):
    """Empty sequences (cu[b] == cu[b + 1]) anywhere in the batch produce no
    rows and leave their neighbours' results unchanged."""
    H, d = 3, 64
    lengths = [0, 70, 0, 0, 129, 1, 0, 64, 0]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    T = int(cu[-1])
    rng = synthetic.rng_for(85)
    qkv = rng.standard_normal((T, 3, H, d)).astype(np.float16)
    dev = to_device(qkv, "f16")
    out = torch.full((T + 8, H, d), float("nan"), dtype=torch.float16, device="cuda")
    cls = torch.full((len(lengths), H, d), 5.0, dtype=torch.float16, device="cuda")
    rv.ragged_get_device_status()
    prev = rv.ragged_set_attn_kernel(KERNELS[kernel])
    try:
        rv.ragged_attn_fwd(dev[:, 0], dev[:, 1], dev[:, 2], torch.from_numpy(cu).cuda(), 200, 0.125, out=out,
                           cls_out=cls)
    finally:
        rv.ragged_set_attn_kernel(prev)
    torch.cuda.synchronize()
    assert rv.ragged_get_device_status() == 0
    ref = oracle.attention(qkv[:, 0], qkv[:, 1], qkv[:, 2], cu, "f16", 0.125)
    err, bound = attn_error(to_f64(out[:T]), ref, "f16")
    assert err <= bound
    assert torch.isnan(out[T:]).all()
    for b, L in enumerate(lengths):
        if L == 0:
            assert torch.all(cls[b] == 5.0)
        else:
            assert torch.equal(cls[b], out[int(cu[b])])


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_persistent_above_its_batch_limit(dtype):
    """More sequences than the persistent kernel keeps in shared memory: the
    launch runs the per-tile tcgen05 kernel instead, with the same results."""
    rng = np.random.default_rng(86)
    lengths = rng.integers(1, 80, size=1100)
    w = synthetic.make_workload("many", 1100, 80, 2, lengths, dtype, 86)
    check_against_oracle(w, seqs=sample_sequences(w.lengths, 12, seed=3), kernel="persistent")


@pytest.mark.parametrize("H", [1023, 1024])
def test_persistent_at_its_head_limit(H):
    """A packed work item holds a head index of 10 bits: H = 1023 runs the
    persistent kernel with every head index in use, H = 1024 runs the per-tile
    tcgen05 kernel instead; both match the oracle on every sequence."""
    rng = np.random.default_rng(88)
    lengths = np.array([70, 1, 129])
    w = synthetic.make_workload("heads", 3, 130, H, lengths, "f16", 88)
    check_against_oracle(w, kernel="persistent")


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_persistent_many_items_per_cta(dtype):
    """Several items per CTA with every length class (full and partial query
    tiles, full and partial key tiles) checked element by element."""
    rng = np.random.default_rng(87)
    lengths = rng.integers(1, 400, size=160)
    lengths[:6] = [1, 64, 128, 129, 256, 399]
    w = synthetic.make_workload("items", 160, 400, 4, lengths, dtype, 87)
    check_against_oracle(w, kernel="persistent")
