"""GPU parity of the one-call pipeline (ragged_pipeline) in its fused single
launch and its two-launch form: cu_seqlens and the packed q/k/v bit-exact
against the oracle, attention within the bound of helpers.attn_error, and the
two forms identical to each other."""
import numpy as np
import pytest
import torch

import oracle
import ragged_variable_length_b200 as rv
import synthetic
from helpers import TORCH_DTYPE, attn_error, to_device, to_f64, to_host_bits

pytestmark = pytest.mark.gpu


def run(w, flags, materialize_packed=True):
    dense = to_device(w.qkv, w.dtype)
    keep = torch.from_numpy(w.keep).cuda()
    T_cap = w.B * w.L_full
    dt = TORCH_DTYPE[w.dtype]
    packed = torch.full((T_cap, 3, w.H, w.d), float("nan"), dtype=dt, device="cuda") if materialize_packed else None
    out = torch.full((T_cap, w.H, w.d), float("nan"), dtype=dt, device="cuda")
    cls = torch.full((w.B, w.H, w.d), float("nan"), dtype=dt, device="cuda")
    cu = torch.full((w.B + 1,), -1, dtype=torch.int32, device="cuda")
    rv.ragged_pipeline(dense, keep, w.scale, packed_qkv=packed, cu_seqlens=cu, out=out, cls_out=cls,
                       flags=flags, materialize_packed=materialize_packed)
    torch.cuda.synchronize()
    assert rv.ragged_get_device_status() == 0
    return packed, cu, out, cls


def check(w, flags, seqs=None, materialize_packed=True):
    packed, cu, out, cls = run(w, flags, materialize_packed)
    packed_o, cu_o = oracle.pack(w.qkv, w.keep)
    T = int(cu_o[-1])
    assert np.array_equal(cu.cpu().numpy(), cu_o)
    if materialize_packed:
        assert np.array_equal(to_host_bits(packed[:T], w.dtype), packed_o)
        assert torch.isnan(packed[T:]).all()
    ref = oracle.attention(packed_o[:, 0], packed_o[:, 1], packed_o[:, 2], cu_o, w.dtype, w.scale, seqs=seqs)
    rows = np.concatenate([np.arange(cu_o[b], cu_o[b + 1]) for b in (seqs if seqs is not None else range(w.B))])
    err, bound = attn_error(to_f64(out[:T])[rows], ref[rows], w.dtype)
    assert err <= bound, f"{w.name}: {err:.3e} > {bound:.3e}"
    assert torch.isnan(out[T:]).all()
    assert torch.equal(cls, out[torch.from_numpy(cu_o[:-1]).long().cuda()])
    return packed, cu, out, cls


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("flags", [rv.RAGGED_PIPELINE_FUSED, rv.RAGGED_PIPELINE_SPLIT])
def test_tiny(dtype, flags):
    check(synthetic.tiny(dtype), flags)


def test_tiny_f32_runs_split():
    check(synthetic.tiny("f32"), rv.RAGGED_PIPELINE_AUTO)


@pytest.mark.parametrize("B", synthetic.SERVING_BATCHES)
@pytest.mark.parametrize("rate", synthetic.SERVING_RATES)
def test_serving_fused(B, rate):
    check(synthetic.serving(B, rate), rv.RAGGED_PIPELINE_FUSED)


@pytest.mark.parametrize("flags", [rv.RAGGED_PIPELINE_FUSED, rv.RAGGED_PIPELINE_SPLIT, rv.RAGGED_PIPELINE_AUTO])
def test_deit_b_pruned80(flags):
    check(synthetic.deit_b_pruned80(), flags)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_edge_lengths_fused(dtype):
    lengths = [1, 2, 63, 64, 65, 127, 128, 129, 197]
    w = synthetic.make_workload("edges", len(lengths), 197, 3, lengths, dtype, 91)
    check(w, rv.RAGGED_PIPELINE_FUSED)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_two_key_tiles_fused(dtype):
    """L_full in 65..128 with a small batch: two warps share each row block's keys."""
    w = synthetic.make_workload("two_tiles", 3, 100, 6, [100, 65, 64], dtype, 95)
    check(w, rv.RAGGED_PIPELINE_FUSED)
    check(w, rv.RAGGED_PIPELINE_SPLIT)


def test_fused_577_and_640():
    w = synthetic.make_workload("hires_edges", 3, 640, 2, [640, 577, 1], "bf16", 92)
    check(w, rv.RAGGED_PIPELINE_FUSED)


def test_hires_sampled_fused():
    w = synthetic.hires_384()
    check(w, rv.RAGGED_PIPELINE_FUSED, seqs=[0, int(np.argmax(w.lengths)), int(np.argmin(w.lengths)), 63])


def test_fused_without_packed_output():
    check(synthetic.serving(4, 0.5), rv.RAGGED_PIPELINE_FUSED, materialize_packed=False)


def test_cls_byte_zero_and_odd_mask_bytes_fused():
    w = synthetic.make_workload("odd", 5, 197, 6, [50, 1, 197, 120, 7], "f16", 93)
    w.keep = w.keep.copy()
    w.keep[:, 0] = 0                     # CLS is kept whatever its mask byte says
    w.keep[w.keep == 1] = 200            # any nonzero byte keeps its token
    check(w, rv.RAGGED_PIPELINE_FUSED)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_fused_equals_split_bitwise(dtype):
    w = synthetic.make_workload("cmp", 8, 197, 6, [197, 150, 100, 60, 40, 39, 2, 1], dtype, 94)
    a = run(w, rv.RAGGED_PIPELINE_FUSED)
    b = run(w, rv.RAGGED_PIPELINE_SPLIT)
    T = int(w.lengths.sum())
    assert torch.equal(a[1], b[1])
    assert torch.equal(a[0][:T], b[0][:T])
    assert torch.equal(a[2][:T], b[2][:T]) and torch.equal(a[3], b[3])


def test_empty_batch_fused():
    cu = torch.full((1,), 9, dtype=torch.int32, device="cuda")
    st = rv.load().ragged_pipeline(None, None, 0, 197, 6, 64, 0.125, 0, None, cu.data_ptr(), None, None,
                                   rv.RAGGED_PIPELINE_FUSED, torch.cuda.current_stream().cuda_stream)
    assert st == rv.RAGGED_OK and cu.item() == 0


@pytest.mark.parametrize("flags", [rv.RAGGED_PIPELINE_FUSED, rv.RAGGED_PIPELINE_SPLIT])
def test_run_sync_matches_enqueue_then_sync(flags):
    w = synthetic.serving(2, 0.5)
    p = rv.Pipeline(w.B, w.L_full, w.H, torch.float16, flags=flags)
    p.dense_qkv.copy_(to_device(w.qkv, "f16"))
    p.keep.copy_(torch.from_numpy(w.keep))
    p()
    torch.cuda.synchronize()
    cls_ref = p.cls_out.clone()
    p.cls_out.zero_()
    p.run_sync()                      # returns with the results in place
    assert torch.equal(p.cls_out, cls_ref)
    packed_o, cu_o = oracle.pack(w.qkv, w.keep)
    assert np.array_equal(p.cu_seqlens.cpu().numpy(), cu_o)


def test_recorded_graph_matches_the_direct_call():
    """ragged_pipeline_graph_create / _launch: the recorded pipeline gives what
    ragged_pipeline gives, and picks up new inputs written into its buffers."""
    w = synthetic.serving(4, 0.5)
    p = rv.Pipeline(w.B, w.L_full, w.H, torch.float16, flags=rv.RAGGED_PIPELINE_FUSED)
    s = torch.cuda.Stream()
    p.dense_qkv.copy_(to_device(w.qkv, "f16"))
    p.keep.copy_(torch.from_numpy(w.keep))
    torch.cuda.synchronize()
    p.bind_inputs(p.dense_qkv, p.keep, stream=s)
    p.record(stream=s)
    for wk in (w, synthetic.serving(4, 0.5, copy=1)):
        p.dense_qkv.copy_(to_device(wk.qkv, "f16"))
        p.keep.copy_(torch.from_numpy(wk.keep))
        torch.cuda.synchronize()
        p.cls_out.zero_()
        p.launch(sync=True)
        _, cu_ref, out_ref, cls_ref = run(wk, rv.RAGGED_PIPELINE_FUSED, materialize_packed=False)
        T = int(cu_ref[-1].item())
        assert torch.equal(p.cu_seqlens, cu_ref)
        assert torch.equal(p.out[:T], out_ref[:T]) and torch.equal(p.cls_out, cls_ref)
    p.release()
    assert rv.ragged_get_device_status() == 0
