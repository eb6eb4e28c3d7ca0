"""The tcgen05 kernels' bounded waits, made to expire on the GPU without a fault.

libragged_testhooks.so is the library built with RAGGED_TEST_HOOKS: a test can
shorten every bounded mbarrier wait and tell one producer to issue nothing (the
persistent kernel's load warp, or the per-tile kernel's MMA thread).  The
waits on that producer then run out.  Each test checks that the launch
returns, that RAGGED_DEV_TIMEOUT is set in the status word, that no output row
was written, and that the next normal launch of the same kernel, which
allocates the same TMEM, finishes and matches the product library bit for bit.

No GPU fault, trap or unbounded wait is involved: nothing is read out of
bounds, and every wait gives up after its poll limit.
"""
import ctypes

import numpy as np
import pytest
import torch

import ragged_variable_length_b200 as rv
import synthetic
from helpers import TORCH_DTYPE, to_device
from ragged_variable_length_b200 import build as rbuild

pytestmark = pytest.mark.gpu

SHORT_SPIN = 1 << 10
PRODUCT_SPIN = 1 << 22


@pytest.fixture(scope="module")
def hooks():
    rbuild.build()
    lib = rv.load(rbuild.build_test_hooks())
    lib.ragged_test_set_hooks.argtypes = [ctypes.c_int32, ctypes.c_uint32]
    lib.ragged_test_set_hooks.restype = ctypes.c_int
    yield lib
    lib.ragged_test_set_hooks(0, PRODUCT_SPIN)


def _status(lib):
    v = ctypes.c_uint32(0)
    assert lib.ragged_get_device_status(ctypes.byref(v), torch.cuda.current_stream().cuda_stream) == 0
    return int(v.value)


def _attend(lib, kernel, packed, cu, w, out):
    D = w.H * w.d
    base = packed.data_ptr()
    e = packed.element_size()
    prev = lib.ragged_set_attn_kernel(kernel)
    try:
        st = lib.ragged_attn_fwd(base, base + D * e, base + 2 * D * e, 3 * D, w.d, cu.data_ptr(), w.B, w.L_full,
                                 w.H, w.d, ctypes.c_float(w.scale), rv.DTYPE_CODES[packed.dtype], out.data_ptr(), D,
                                 None, torch.cuda.current_stream().cuda_stream)
    finally:
        lib.ragged_set_attn_kernel(prev)
    assert st == 0
    torch.cuda.synchronize()


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("kernel,hook", [(rv.RAGGED_ATTN_PERSISTENT, 1), (rv.RAGGED_ATTN_TCGEN05, 2)])
def test_expired_wait_is_reported_and_the_next_launch_is_exact(hooks, dtype, kernel, hook):
    rng = np.random.default_rng(91)
    lengths = rng.integers(1, 300, size=24)
    w = synthetic.make_workload("waits", 24, 300, 3, lengths, dtype, 91)
    dense = to_device(w.qkv, dtype)
    keep = torch.from_numpy(w.keep).cuda()
    packed, cu = rv.ragged_pack(dense, keep)
    T = int(w.lengths.sum())
    dt = TORCH_DTYPE[dtype]

    # reference: the product library, same kernel
    ref = torch.full((w.B * w.L_full, w.H, w.d), float("nan"), dtype=dt, device="cuda")
    _attend(rv.load(), kernel, packed, cu, w, ref)
    assert rv.ragged_get_device_status() == 0

    _status(hooks)   # clear
    assert hooks.ragged_test_set_hooks(hook, SHORT_SPIN) == 0
    out = torch.full_like(ref, 3.0)
    try:
        _attend(hooks, kernel, packed, cu, w, out)
    finally:
        assert hooks.ragged_test_set_hooks(0, PRODUCT_SPIN) == 0
    assert _status(hooks) & rv.RAGGED_DEV_TIMEOUT
    assert torch.all(out == 3.0), "a launch whose waits expired must not write output rows"

    # the same kernel again, normal: it allocates the TMEM the failed launch
    # freed, finishes, and equals the product library bit for bit
    out2 = torch.full_like(ref, float("nan"))
    _attend(hooks, kernel, packed, cu, w, out2)
    assert _status(hooks) == 0
    assert torch.equal(out2[:T], ref[:T])
    assert torch.isnan(out2[T:]).all()


def test_hook_settings_are_checked(hooks):
    assert hooks.ragged_test_set_hooks(3, SHORT_SPIN) == rv.RAGGED_ERR_INVALID_ARG
    assert hooks.ragged_test_set_hooks(1, 0) == rv.RAGGED_ERR_INVALID_ARG
