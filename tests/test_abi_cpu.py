"""C ABI checks that need no GPU: the library builds, loads, exports every
symbol declared in include/ragged.h, and rejects bad arguments on the host
before anything is enqueued."""
import ctypes
import os
import re

import pytest

import ragged_variable_length_b200 as rv
from ragged_variable_length_b200 import build as rbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ragged.h")


@pytest.fixture(scope="module")
def lib():
    rbuild.build()
    return rv.load()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"RAGGED_API\s+[\w\s\*]+?\b(ragged_\w+)\s*\(", text)


def test_header_declares_the_binding_exports():
    names = declared_functions()
    assert sorted(names) == sorted(rv.EXPORTS)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_only_declared_symbols_are_exported():
    out = os.popen(f"nm -D --defined-only {rv.LIB_PATH}").read()
    exported = {m.group(1) for m in re.finditer(r" T (\w+)", out)}
    assert exported == set(declared_functions())


def test_version_and_status_strings(lib):
    assert rv.ragged_abi_version() == 1
    assert rv.ragged_status_string(rv.RAGGED_OK) == "ok"
    assert "invalid" in rv.ragged_status_string(rv.RAGGED_ERR_INVALID_ARG)
    assert rv.ragged_status_string(99) == "unknown status"


# Fake, never-dereferenced device addresses: validation fails before any CUDA call.
A16 = 1 << 20
A8 = A16 + 8


def _pack(lib, **kw):
    a = dict(dense=A16, B=2, L_full=197, row_bytes=768, keep=A16, packed=A16, cu=A16, src=None)
    a.update(kw)
    return lib.ragged_pack(a["dense"], a["B"], a["L_full"], a["row_bytes"], a["keep"], a["packed"],
                           a["cu"], a["src"], None)


@pytest.mark.parametrize("kw,status,needle", [
    (dict(B=-1), rv.RAGGED_ERR_INVALID_ARG, "negative"),
    (dict(B=70000), rv.RAGGED_ERR_UNSUPPORTED, "65535"),
    (dict(L_full=0), rv.RAGGED_ERR_INVALID_ARG, "L_full"),
    (dict(L_full=rv.RAGGED_MAX_TOKENS + 1), rv.RAGGED_ERR_INVALID_ARG, "L_full"),
    (dict(row_bytes=24), rv.RAGGED_ERR_INVALID_ARG, "multiple of 16"),
    (dict(row_bytes=0), rv.RAGGED_ERR_INVALID_ARG, "multiple of 16"),
    (dict(cu=None), rv.RAGGED_ERR_INVALID_ARG, "cu_seqlens"),
    (dict(cu=A16 + 2), rv.RAGGED_ERR_INVALID_ARG, "aligned"),
    (dict(dense=None), rv.RAGGED_ERR_INVALID_ARG, "NULL"),
    (dict(packed=None), rv.RAGGED_ERR_INVALID_ARG, "NULL"),
    (dict(dense=A8), rv.RAGGED_ERR_INVALID_ARG, "16-byte"),
    (dict(packed=A8), rv.RAGGED_ERR_INVALID_ARG, "16-byte"),
    (dict(B=40000, L_full=60000), rv.RAGGED_ERR_INVALID_ARG, "L_full"),
])
def test_pack_rejects(lib, kw, status, needle):
    assert _pack(lib, **kw) == status
    assert needle in rv.ragged_last_error()


def _attn(lib, **kw):
    a = dict(q=A16, k=A16, v=A16, ts=3 * 6 * 64, hs=64, cu=A16, B=4, maxL=197, H=6, d=64,
             scale=0.125, dt=0, out=A16, ots=6 * 64, cls=None)
    a.update(kw)
    return lib.ragged_attn_fwd(a["q"], a["k"], a["v"], a["ts"], a["hs"], a["cu"], a["B"], a["maxL"],
                               a["H"], a["d"], a["scale"], a["dt"], a["out"], a["ots"], a["cls"], None)


@pytest.mark.parametrize("kw,status,needle", [
    (dict(B=-3), rv.RAGGED_ERR_INVALID_ARG, "negative"),
    (dict(d=128), rv.RAGGED_ERR_UNSUPPORTED, "head_dim"),
    (dict(d=32), rv.RAGGED_ERR_UNSUPPORTED, "head_dim"),
    (dict(dt=7), rv.RAGGED_ERR_INVALID_ARG, "dtype"),
    (dict(H=0), rv.RAGGED_ERR_INVALID_ARG, "H ="),
    (dict(maxL=0), rv.RAGGED_ERR_INVALID_ARG, "max_seqlen"),
    (dict(maxL=rv.RAGGED_MAX_TOKENS + 1), rv.RAGGED_ERR_INVALID_ARG, "max_seqlen"),
    (dict(scale=0.0), rv.RAGGED_ERR_INVALID_ARG, "scale"),
    (dict(scale=-0.125), rv.RAGGED_ERR_INVALID_ARG, "scale"),
    (dict(scale=float("nan")), rv.RAGGED_ERR_INVALID_ARG, "scale"),
    (dict(scale=float("inf")), rv.RAGGED_ERR_INVALID_ARG, "scale"),
    (dict(q=None), rv.RAGGED_ERR_INVALID_ARG, "NULL"),
    (dict(out=None), rv.RAGGED_ERR_INVALID_ARG, "NULL"),
    (dict(cu=None), rv.RAGGED_ERR_INVALID_ARG, "NULL"),
    (dict(k=A8), rv.RAGGED_ERR_INVALID_ARG, "16-byte"),
    (dict(cls=A8), rv.RAGGED_ERR_INVALID_ARG, "16-byte"),
    (dict(ts=3 * 6 * 64 + 4), rv.RAGGED_ERR_INVALID_ARG, "stride"),
    (dict(hs=60), rv.RAGGED_ERR_INVALID_ARG, "stride"),
    (dict(ots=6 * 64 - 8), rv.RAGGED_ERR_INVALID_ARG, "out_tok_stride"),
    (dict(dt=2, ots=6 * 64 + 2), rv.RAGGED_ERR_INVALID_ARG, "out_tok_stride"),
])
def test_attn_rejects(lib, kw, status, needle):
    assert _attn(lib, **kw) == status
    assert needle in rv.ragged_last_error()


def test_empty_batch_attention_is_a_noop(lib):
    assert _attn(lib, B=0, q=None, k=None, v=None, out=None, cu=None) == rv.RAGGED_OK


@pytest.mark.parametrize("kw,status,needle", [
    (dict(B=-1), rv.RAGGED_ERR_INVALID_ARG, "negative"),
    (dict(L_full=0), rv.RAGGED_ERR_INVALID_ARG, "L_full"),
    (dict(C=0), rv.RAGGED_ERR_INVALID_ARG, "C ="),
    (dict(tok_stride=10), rv.RAGGED_ERR_INVALID_ARG, "tok_stride"),
    (dict(dtype=7), rv.RAGGED_ERR_INVALID_ARG, "dtype"),
    (dict(tau=float("nan")), rv.RAGGED_ERR_INVALID_ARG, "NaN"),
    (dict(x=None), rv.RAGGED_ERR_INVALID_ARG, "NULL"),
    (dict(keep=None), rv.RAGGED_ERR_INVALID_ARG, "NULL"),
    (dict(x=A16 + 1), rv.RAGGED_ERR_INVALID_ARG, "aligned"),
    (dict(B=40000, L_full=60000), rv.RAGGED_ERR_INVALID_ARG, "L_full"),
])
def test_mask_l2_rejects(lib, kw, status, needle):
    a = dict(x=A16, B=2, L_full=197, C=384, tok_stride=384, dtype=rv.RAGGED_F16, tau=1.0, keep=A16)
    a.update(kw)
    assert lib.ragged_mask_l2(a["x"], a["B"], a["L_full"], a["C"], a["tok_stride"], a["dtype"], a["tau"],
                              a["keep"], None) == status
    assert needle in rv.ragged_last_error()


def test_empty_batch_mask_is_a_noop(lib):
    assert lib.ragged_mask_l2(None, 0, 197, 384, 384, rv.RAGGED_F16, 1.0, None, None) == rv.RAGGED_OK


@pytest.mark.parametrize("kw,status,needle", [
    (dict(B=-1), rv.RAGGED_ERR_INVALID_ARG, "negative"),
    (dict(L_full=9000), rv.RAGGED_ERR_UNSUPPORTED, "8192"),
    (dict(row_bytes=24), rv.RAGGED_ERR_INVALID_ARG, "multiple of 16"),
    (dict(cu=None), rv.RAGGED_ERR_INVALID_ARG, "cu_seqlens"),
    (dict(scores=None), rv.RAGGED_ERR_INVALID_ARG, "NULL"),
    (dict(count=None), rv.RAGGED_ERR_INVALID_ARG, "NULL"),
    (dict(scores=A16 + 2), rv.RAGGED_ERR_INVALID_ARG, "4-byte"),
    (dict(dense=A8), rv.RAGGED_ERR_INVALID_ARG, "16-byte"),
])
def test_pack_topk_rejects(lib, kw, status, needle):
    a = dict(dense=A16, B=2, L_full=197, row_bytes=768, scores=A16, count=A16, packed=A16, cu=A16)
    a.update(kw)
    assert lib.ragged_pack_topk(a["dense"], a["B"], a["L_full"], a["row_bytes"], a["scores"], a["count"],
                                a["packed"], a["cu"], None, None, None) == status
    assert needle in rv.ragged_last_error()


def test_unpack_rejects(lib):
    assert lib.ragged_unpack(A16, A16, A16, 2, 197, 40, A16, None) == rv.RAGGED_ERR_INVALID_ARG
    assert lib.ragged_unpack(None, A16, A16, 2, 197, 48, A16, None) == rv.RAGGED_ERR_INVALID_ARG
    assert lib.ragged_unpack(A16, A16, A16, 2, 197, 48, A8, None) == rv.RAGGED_ERR_INVALID_ARG
    assert lib.ragged_unpack_cls(A16, A16, -1, 48, A16, None) == rv.RAGGED_ERR_INVALID_ARG
    assert lib.ragged_unpack_cls(A16, A16, 2, 40, A16, None) == rv.RAGGED_ERR_INVALID_ARG
    assert lib.ragged_unpack_cls(A16, None, 2, 48, A16, None) == rv.RAGGED_ERR_INVALID_ARG
    assert lib.ragged_unpack_cls(A16, A16, 0, 48, None, None) == rv.RAGGED_OK


def _pipe(lib, **kw):
    a = dict(dense=A16, keep=A16, B=2, L=197, H=6, d=64, scale=0.125, dt=0, packed=A16, cu=A16, out=A16,
             cls=None, flags=0)
    a.update(kw)
    return lib.ragged_pipeline(a["dense"], a["keep"], a["B"], a["L"], a["H"], a["d"], a["scale"], a["dt"],
                               a["packed"], a["cu"], a["out"], a["cls"], a["flags"], None)


@pytest.mark.parametrize("kw,status,needle", [
    (dict(d=32), rv.RAGGED_ERR_UNSUPPORTED, "head_dim"),
    (dict(H=0), rv.RAGGED_ERR_INVALID_ARG, "H ="),
    (dict(dense=A8), rv.RAGGED_ERR_INVALID_ARG, "16-byte"),
    (dict(out=A8), rv.RAGGED_ERR_INVALID_ARG, "16-byte"),
    (dict(flags=3), rv.RAGGED_ERR_INVALID_ARG, "flags"),
    (dict(flags=7), rv.RAGGED_ERR_INVALID_ARG, "flags"),
    (dict(flags=5, dense=A8), rv.RAGGED_ERR_INVALID_ARG, "16-byte"),
    (dict(flags=8), rv.RAGGED_ERR_INVALID_ARG, "flags"),
    (dict(scale=0.0), rv.RAGGED_ERR_INVALID_ARG, "scale"),
    (dict(L=0), rv.RAGGED_ERR_INVALID_ARG, "L_full"),
    (dict(B=-1), rv.RAGGED_ERR_INVALID_ARG, "negative"),
    (dict(flags=1, L=641), rv.RAGGED_ERR_UNSUPPORTED, "fused"),
    (dict(flags=1, dt=2), rv.RAGGED_ERR_UNSUPPORTED, "fused"),
    (dict(flags=2, packed=None), rv.RAGGED_ERR_INVALID_ARG, "packed_qkv"),
    (dict(flags=1, cu=None), rv.RAGGED_ERR_INVALID_ARG, "cu_seqlens"),
    (dict(flags=1, keep=None), rv.RAGGED_ERR_INVALID_ARG, "NULL"),
])
def test_pipeline_rejects(lib, kw, status, needle):
    assert _pipe(lib, **kw) == status
    assert needle in rv.ragged_last_error()


def test_device_status_needs_an_output_pointer(lib):
    assert lib.ragged_get_device_status(None, None) == rv.RAGGED_ERR_INVALID_ARG


def test_binding_fails_loudly_without_the_library():
    missing = os.path.join(os.path.dirname(os.path.abspath(__file__)), "no_such_dir", "nope.so")
    assert not os.path.exists(missing)
    with pytest.raises(RuntimeError, match="missing"):
        rv.load(missing)


def test_test_hooks_live_only_in_the_test_build():
    """The failure-path switches are compiled into libragged_testhooks.so only."""
    hooks = rbuild.build_test_hooks()
    prod = os.popen(f"nm -D --defined-only {rv.LIB_PATH}").read()
    test = os.popen(f"nm -D --defined-only {hooks}").read()
    assert "ragged_test_set_hooks" not in prod
    assert re.search(r" T ragged_test_set_hooks\b", test)
    header = open(os.path.join(ROOT, "include", "ragged_test_hooks.h")).read()
    assert "RAGGED_API ragged_status ragged_test_set_hooks(" in header


def test_pipeline_graph_rejects_bad_arguments(lib):
    """ragged_pipeline_graph_*: argument errors come back before any CUDA call."""
    out = ctypes.c_void_p(123)
    args = (A16, A16, 4, 197, 6, 64, ctypes.c_float(0.125), rv.RAGGED_F16, None, A16, A16, None)
    assert lib.ragged_pipeline_graph_create(*args, rv.RAGGED_PIPELINE_FUSED, A16, None) == rv.RAGGED_ERR_INVALID_ARG
    assert "graph_out" in rv.ragged_last_error()
    assert lib.ragged_pipeline_graph_create(*args, rv.RAGGED_PIPELINE_SYNC, A16,
                                            ctypes.byref(out)) == rv.RAGGED_ERR_INVALID_ARG
    assert out.value is None and "SYNC" in rv.ragged_last_error()
    assert lib.ragged_pipeline_graph_create(*args, 0, None, ctypes.byref(out)) == rv.RAGGED_ERR_INVALID_ARG
    assert "default" in rv.ragged_last_error()
    assert lib.ragged_pipeline_graph_launch(None, None, 0) == rv.RAGGED_ERR_INVALID_ARG
    assert lib.ragged_pipeline_graph_launch(A16, None, 8) == rv.RAGGED_ERR_INVALID_ARG
    assert lib.ragged_pipeline_graph_destroy(None) == rv.RAGGED_OK
