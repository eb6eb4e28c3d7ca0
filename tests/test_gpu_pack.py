"""GPU parity of survivor bookkeeping, pack, scatter-back and CLS extraction:
bit-exact against the CPU oracle on the same seeded inputs, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import ragged_variable_length_b200 as rv
import synthetic
from helpers import to_device, to_host_bits

pytestmark = pytest.mark.gpu

CANARY = 0xA5


def _gpu_pack(dense_np, keep_np, dtype_tag=None, keep_offset=0):
    """Runs ragged_pack with canary-filled outputs; returns host copies."""
    B, L = keep_np.shape
    dense = torch.from_numpy(np.ascontiguousarray(dense_np).view(np.uint8)).cuda()
    row_bytes = dense_np.itemsize * int(np.prod(dense_np.shape[2:]))
    # keep buffer at an arbitrary byte offset inside a larger allocation
    keep_buf = torch.zeros(B * L + keep_offset + 64, dtype=torch.uint8, device="cuda")
    keep = keep_buf[keep_offset:keep_offset + B * L]
    keep.copy_(torch.from_numpy(np.ascontiguousarray(keep_np).reshape(-1)))
    margin = 4096
    packed_buf = torch.full((2 * margin + B * L * row_bytes,), CANARY, dtype=torch.uint8, device="cuda")
    packed = packed_buf[margin:margin + B * L * row_bytes]
    cu_buf = torch.full((B + 1 + 8,), -7, dtype=torch.int32, device="cuda")
    cu = cu_buf[4:4 + B + 1]
    src = torch.full((max(B * L, 1),), -9, dtype=torch.int32, device="cuda")
    lib = rv.load()
    st = lib.ragged_pack(dense.data_ptr(), B, L, row_bytes, keep.data_ptr(), packed.data_ptr(),
                         cu.data_ptr(), src.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == rv.RAGGED_OK, rv.ragged_last_error()
    torch.cuda.synchronize()
    assert rv.ragged_get_device_status() == 0
    pb = packed_buf.cpu().numpy()
    assert np.all(pb[:margin] == CANARY) and np.all(pb[margin + B * L * row_bytes:] == CANARY)
    cub = cu_buf.cpu().numpy()
    assert np.all(cub[:4] == -7) and np.all(cub[4 + B + 1:] == -7)
    return pb[margin:margin + B * L * row_bytes].reshape(B * L, row_bytes), cu.cpu().numpy(), src.cpu().numpy(), row_bytes


def _check_pack(dense_np, keep_np, keep_offset=0):
    B, L = keep_np.shape
    packed_g, cu_g, src_g, row_bytes = _gpu_pack(dense_np, keep_np, keep_offset=keep_offset)
    cu_o, src_o = oracle.seqlens(keep_np)
    packed_o, cu_o2 = oracle.pack(dense_np, keep_np)
    T = int(cu_o[-1])
    assert np.array_equal(cu_g, cu_o)
    assert np.array_equal(src_g[:T], src_o)
    assert np.all(src_g[T:] == -9)
    assert np.array_equal(packed_g[:T], np.ascontiguousarray(packed_o).view(np.uint8).reshape(T, row_bytes))
    assert np.all(packed_g[T:] == CANARY)            # rows past T are not written


WORKLOADS = {
    "tiny_tokens_f32": lambda: (synthetic.tiny("f32").tokens, synthetic.tiny("f32").keep),
    "tiny_qkv_f16": lambda: (synthetic.tiny("f16").qkv, synthetic.tiny("f16").keep),
    "deit_b_p80_bf16": lambda: (synthetic.deit_b_pruned80().qkv, synthetic.deit_b_pruned80().keep),
    "serving_b4_p50": lambda: (synthetic.serving(4, 0.5).qkv, synthetic.serving(4, 0.5).keep),
    "serving_b1_p0": lambda: (synthetic.serving(1, 0.0).qkv, synthetic.serving(1, 0.0).keep),
    "hires384_b64": lambda: (synthetic.hires_384().qkv, synthetic.hires_384().keep),
    "sweep_b512_p50": lambda: (synthetic.sweep(0.5).qkv, synthetic.sweep(0.5).keep),
}


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_pack_bit_exact_on_workloads(name):
    dense, keep = WORKLOADS[name]()
    _check_pack(dense, keep)


def _edge_masks():
    rng = np.random.default_rng(5)
    return {
        "L1": np.zeros((3, 1), dtype=np.uint8),
        "only_cls": np.zeros((5, 197), dtype=np.uint8),
        "all_kept": np.ones((4, 197), dtype=np.uint8),
        "cls_byte_zero": np.concatenate([np.zeros((6, 1), np.uint8), np.ones((6, 40), np.uint8)], 1),
        "odd_bytes": (rng.integers(0, 3, size=(7, 301)) * 127).astype(np.uint8),
        "long_rows": (rng.random((2, 1500)) < 0.5).astype(np.uint8),
        "max_tokens": (rng.random((1, rv.RAGGED_MAX_TOKENS)) < 0.2).astype(np.uint8),
        "many_images": (rng.random((3000, 9)) < 0.5).astype(np.uint8),
    }


@pytest.mark.parametrize("name", sorted(_edge_masks()))
@pytest.mark.parametrize("row_bytes", [16, 48, 4608])
def test_pack_edge_cases(name, row_bytes):
    keep = _edge_masks()[name]
    B, L = keep.shape
    if B * L * row_bytes > 64 << 20:
        row_bytes = 16
    rng = np.random.default_rng(B * 1000 + L)
    dense = rng.integers(0, 256, size=(B, L, row_bytes), dtype=np.uint8)
    _check_pack(dense, keep)


@pytest.mark.parametrize("offset", [1, 3, 8, 13])
def test_pack_unaligned_keep(offset):
    keep = (np.random.default_rng(offset).random((9, 197)) < 0.4).astype(np.uint8)
    dense = np.random.default_rng(0).integers(0, 256, size=(9, 197, 32), dtype=np.uint8)
    _check_pack(dense, keep, keep_offset=offset)


def test_pack_empty_batch():
    cu = torch.full((1,), 5, dtype=torch.int32, device="cuda")
    st = rv.load().ragged_pack(None, 0, 197, 768, None, None, cu.data_ptr(), None,
                               torch.cuda.current_stream().cuda_stream)
    assert st == rv.RAGGED_OK
    assert cu.item() == 0


@pytest.mark.parametrize("name", ["tiny_qkv_f16", "deit_b_p80_bf16", "hires384_b64", "serving_b4_p50"])
def test_unpack_and_cls_bit_exact(name):
    dense_np, keep_np = WORKLOADS[name]()
    B, L = keep_np.shape
    dense = torch.from_numpy(np.ascontiguousarray(dense_np).view(np.uint8).reshape(B, L, -1)).cuda()
    keep = torch.from_numpy(keep_np).cuda()
    packed, cu = rv.ragged_pack(dense, keep)
    cls = rv.ragged_unpack_cls(packed, cu)
    back = torch.full_like(dense, 0x3C)
    rv.ragged_unpack(packed, cu, keep, back)
    torch.cuda.synchronize()
    assert rv.ragged_get_device_status() == 0
    packed_o, cu_o = oracle.pack(dense_np, keep_np)
    pb = np.ascontiguousarray(packed_o).view(np.uint8).reshape(packed_o.shape[0], -1)
    cls_o = oracle.unpack_cls(pb, cu_o)
    assert np.array_equal(cls.cpu().numpy(), cls_o)
    sentinel = np.full((B, L, pb.shape[1]), 0x3C, dtype=np.uint8)
    back_o = oracle.unpack(pb, keep_np, sentinel)
    assert np.array_equal(back.cpu().numpy(), back_o)


def test_unpack_flags_inconsistent_cu_seqlens():
    keep = torch.ones((2, 8), dtype=torch.uint8, device="cuda")
    packed = torch.zeros((16, 16), dtype=torch.uint8, device="cuda")
    cu = torch.tensor([0, 5, 16], dtype=torch.int32, device="cuda")   # image 0 has 8 survivors
    dense_out = torch.full((2, 8, 16), 7, dtype=torch.uint8, device="cuda")
    rv.ragged_get_device_status()
    rv.ragged_unpack(packed, cu, keep, dense_out)
    assert rv.ragged_get_device_status() & rv.RAGGED_DEV_BAD_SEQLENS
    assert torch.all(dense_out[0] == 7)                                # skipped, not written
