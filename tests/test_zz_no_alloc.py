"""ragged_pipeline_noalloc: the two-launch pipeline for callers that cannot
allocate device memory (a plugin whose host framework owns the allocator, code
running beside a global-mode graph capture, a service with a footprint fixed
at start-up).  Its packed q/k/v lives in a fixed array inside the library, so
the caller passes only inputs and outputs.

The GPU test calls the entry point through the C ABI twice in a row, on two
different batches, and compares each result with ragged_pipeline's own
two-launch form on the same inputs: cu_seqlens bit-exact, attention and CLS
rows within the bound the other attention tests use.  The file is named to be
collected last, so that a run stopping at its first failure has already run
every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import ragged_variable_length_b200 as rv
import synthetic
from helpers import TORCH_DTYPE, attn_error, to_device, to_f64
from ragged_variable_length_b200 import build as rbuild


@pytest.fixture(scope="module")
def lib():
    rbuild.build()
    return rv.load()


def _outputs(w):
    dt = TORCH_DTYPE[w.dtype]
    cap = w.B * w.L_full
    cu = torch.full((w.B + 1,), -1, dtype=torch.int32, device="cuda")
    out = torch.full((cap, w.H, w.d), float("nan"), dtype=dt, device="cuda")
    cls = torch.full((w.B, w.H, w.d), float("nan"), dtype=dt, device="cuda")
    return cu, out, cls


def _noalloc(lib, w, dense, keep):
    cu, out, cls = _outputs(w)
    stream = torch.cuda.current_stream().cuda_stream
    st = lib.ragged_pipeline_noalloc(dense.data_ptr(), keep.data_ptr(), w.B, w.L_full, w.H, w.d,
                                     ctypes.c_float(w.scale), rv.DTYPE_CODES[TORCH_DTYPE[w.dtype]],
                                     cu.data_ptr(), out.data_ptr(), cls.data_ptr(), stream)
    assert st == rv.RAGGED_OK, rv.ragged_last_error()
    return cu, out, cls


def _split(w, dense, keep):
    cu, out, cls = _outputs(w)
    rv.ragged_pipeline(dense, keep, w.scale, cu_seqlens=cu, out=out, cls_out=cls,
                       flags=rv.RAGGED_PIPELINE_SPLIT)
    return cu, out, cls


@pytest.mark.gpu
def test_noalloc_matches_the_split_pipeline_on_two_calls_in_a_row(lib):
    # Two different batches back to back: the second call finds the first
    # call's rows in the shared array and must not depend on them.
    batches = [synthetic.serving(4, 0.5), synthetic.tiny("bf16")]
    for w in batches:
        assert w.B * w.L_full * w.row_bytes <= rv.RAGGED_NOALLOC_SCRATCH_BYTES
        dense = to_device(w.qkv, w.dtype)
        keep = torch.from_numpy(w.keep).cuda()
        cu_n, out_n, cls_n = _noalloc(lib, w, dense, keep)
        cu_s, out_s, cls_s = _split(w, dense, keep)
        torch.cuda.synchronize()
        assert rv.ragged_get_device_status() == 0
        cu_ref = cu_s.cpu().numpy()
        assert np.array_equal(cu_n.cpu().numpy(), cu_ref), w.name
        T = int(cu_ref[-1])
        err, bound = attn_error(to_f64(out_n[:T]), to_f64(out_s[:T]), w.dtype)
        assert err <= bound, f"{w.name}: out differs by {err:.3e} > {bound:.3e}"
        err, bound = attn_error(to_f64(cls_n), to_f64(cls_s), w.dtype)
        assert err <= bound, f"{w.name}: CLS differs by {err:.3e} > {bound:.3e}"
        assert torch.isnan(out_n[T:]).all(), "rows past T must stay untouched"


def test_noalloc_rejects_batches_beyond_the_fixed_scratch(lib):
    # DeiT-B rows (3 * 12 * 64 * 2 = 4,608 bytes): 32 images of 197 tokens need
    # 29 MB, more than the 16 MiB array.  Rejected on the host before any CUDA
    # call, so this runs without a GPU (the pointers are never dereferenced).
    fake = 1 << 20
    st = lib.ragged_pipeline_noalloc(fake, fake, 32, 197, 12, 64, ctypes.c_float(0.125), rv.RAGGED_BF16,
                                     fake, fake, None, None)
    assert st == rv.RAGGED_ERR_UNSUPPORTED
    assert "fixed scratch" in rv.ragged_last_error()
    rows = rv.RAGGED_NOALLOC_SCRATCH_BYTES // 4608
    assert rows < 32 * 197
