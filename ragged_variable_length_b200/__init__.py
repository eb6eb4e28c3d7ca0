"""Python binding of libragged (the C ABI declared in include/ragged.h).

Argument marshalling only: every function below hands device pointers and
sizes to the CUDA library, whose kernels do all of the work.  There is no CPU
fallback; if the compiled library is missing the import of the binding's
functions fails loudly.

Entry points (same names as the C ABI):
  ragged_pack        keep mask -> cu_seqlens; survivors gathered into a flat buffer
  ragged_attn_fwd    bidirectional softmax attention over every packed sequence
  ragged_unpack_cls  CLS row of every sequence
  ragged_unpack      scatter packed rows back to their dense positions
  ragged_pipeline    pack -> attend -> CLS in one host call
  ragged_mask_l2     Threshold-l2 keep mask from token feature norms
  ragged_pack_topk   top-k keep selection by score fused into pack
  ragged_pipeline_noalloc  the two-launch pipeline with its packed q/k/v in a
                     fixed library array, for callers that cannot allocate
``Pipeline`` keeps the buffers and the marshalled arguments of one shape so
that a call costs one foreign-function crossing, and can replay the whole
pipeline as one CUDA graph.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libragged.so")

RAGGED_OK = 0
RAGGED_ERR_INVALID_ARG = 1
RAGGED_ERR_UNSUPPORTED = 2
RAGGED_ERR_CUDA = 3
RAGGED_ERR_DEVICE = 4
RAGGED_DEV_BAD_SEQLENS = 0x1
RAGGED_DEV_TIMEOUT = 0x2
RAGGED_MAX_TOKENS = 16384
RAGGED_NOALLOC_SCRATCH_BYTES = 16 << 20
RAGGED_PIPELINE_AUTO = 0
RAGGED_PIPELINE_FUSED = 1
RAGGED_PIPELINE_SPLIT = 2
RAGGED_PIPELINE_SYNC = 4
RAGGED_ATTN_AUTO = 0
RAGGED_ATTN_STREAMING = 1
RAGGED_ATTN_RESIDENT = 2
RAGGED_ATTN_TCGEN05 = 3
RAGGED_ATTN_PERSISTENT = 4
RAGGED_F16, RAGGED_BF16, RAGGED_F32 = 0, 1, 2

DTYPE_CODES = {torch.float16: 0, torch.bfloat16: 1, torch.float32: 2}
DTYPE_NAMES = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}

EXPORTS = ("ragged_pack", "ragged_attn_fwd", "ragged_unpack_cls", "ragged_unpack",
           "ragged_pipeline", "ragged_get_device_status", "ragged_status_string",
           "ragged_last_error", "ragged_abi_version", "ragged_set_attn_kernel",
           "ragged_mask_l2", "ragged_pack_topk", "ragged_pipeline_noalloc", "ragged_pipeline_graph_create",
           "ragged_pipeline_graph_launch", "ragged_pipeline_graph_destroy")


class RaggedError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{message} (status {status})")
        self.status = status


_lib = None


def load(path: Optional[str] = None):
    """Load libragged.so and declare the C signatures.  Raises if it is missing."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"{p} is missing: build it with `python -m ragged_variable_length_b200.build`")
    lib = ctypes.CDLL(p)
    i64, vp, f32, i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_float, ctypes.c_int
    lib.ragged_pack.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, vp]
    lib.ragged_attn_fwd.argtypes = [vp, vp, vp, i64, i64, vp, i64, i64, i64, i64, f32, i32, vp, i64, vp, vp]
    lib.ragged_unpack_cls.argtypes = [vp, vp, i64, i64, vp, vp]
    lib.ragged_mask_l2.argtypes = [vp, i64, i64, i64, i64, i32, ctypes.c_double, vp, vp]
    lib.ragged_pack_topk.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, vp, vp, vp]
    lib.ragged_unpack.argtypes = [vp, vp, vp, i64, i64, i64, vp, vp]
    lib.ragged_pipeline.argtypes = [vp, vp, i64, i64, i64, i64, f32, i32, vp, vp, vp, vp, ctypes.c_uint32, vp]
    lib.ragged_pipeline_noalloc.argtypes = [vp, vp, i64, i64, i64, i64, f32, i32, vp, vp, vp, vp]
    lib.ragged_pipeline_graph_create.argtypes = [vp, vp, i64, i64, i64, i64, f32, i32, vp, vp, vp, vp,
                                                 ctypes.c_uint32, vp, ctypes.POINTER(vp)]
    lib.ragged_pipeline_graph_launch.argtypes = [vp, vp, ctypes.c_uint32]
    lib.ragged_pipeline_graph_destroy.argtypes = [vp]
    lib.ragged_get_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint32), vp]
    for name in ("ragged_pack", "ragged_attn_fwd", "ragged_unpack_cls", "ragged_unpack",
                 "ragged_pipeline", "ragged_get_device_status", "ragged_pipeline_noalloc",
                 "ragged_pipeline_graph_create", "ragged_pipeline_graph_launch", "ragged_pipeline_graph_destroy"):
        getattr(lib, name).restype = ctypes.c_int
    lib.ragged_status_string.argtypes = [ctypes.c_int]
    lib.ragged_status_string.restype = ctypes.c_char_p
    lib.ragged_last_error.argtypes = []
    lib.ragged_last_error.restype = ctypes.c_char_p
    lib.ragged_abi_version.argtypes = []
    lib.ragged_abi_version.restype = ctypes.c_int32
    lib.ragged_set_attn_kernel.argtypes = [ctypes.c_int32]
    lib.ragged_set_attn_kernel.restype = ctypes.c_int32
    if path is None:
        _lib = lib
    return lib


def _check(status: int) -> None:
    if status != RAGGED_OK:
        lib = load()
        raise RaggedError(status, f"{lib.ragged_status_string(status).decode()}: "
                                  f"{lib.ragged_last_error().decode()}")


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _dtype_code(t: torch.Tensor) -> int:
    try:
        return DTYPE_CODES[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}") from None


def ragged_abi_version() -> int:
    return int(load().ragged_abi_version())


def ragged_set_attn_kernel(kernel: int) -> int:
    """Process-wide attention kernel choice (RAGGED_ATTN_*); returns the previous one."""
    prev = int(load().ragged_set_attn_kernel(int(kernel)))
    if prev < 0:
        raise ValueError(f"unknown attention kernel {kernel}")
    return prev


def ragged_status_string(status: int) -> str:
    return load().ragged_status_string(status).decode()


def ragged_last_error() -> str:
    return load().ragged_last_error().decode()


def ragged_pack(dense: torch.Tensor, keep: torch.Tensor, packed: Optional[torch.Tensor] = None,
                cu_seqlens: Optional[torch.Tensor] = None, src_idx: Optional[torch.Tensor] = None,
                stream=None):
    """dense [B, L_full, ...] contiguous, keep uint8 [B, L_full] -> (packed, cu_seqlens).

    packed has capacity B * L_full rows (rows >= T are not written).
    """
    B, L_full = int(keep.shape[0]), int(keep.shape[1])
    if not dense.is_contiguous() or tuple(dense.shape[:2]) != (B, L_full):
        raise ValueError("dense must be contiguous [B, L_full, ...]")
    row_bytes = dense.element_size() * (dense[0, 0].numel() if B else int(torch.tensor(dense.shape[2:]).prod()))
    if packed is None:
        packed = torch.empty((B * L_full,) + tuple(dense.shape[2:]), dtype=dense.dtype, device=dense.device)
    if cu_seqlens is None:
        cu_seqlens = torch.empty(B + 1, dtype=torch.int32, device=dense.device)
    _check(load().ragged_pack(_ptr(dense), B, L_full, row_bytes, _ptr(keep), _ptr(packed),
                              _ptr(cu_seqlens), _ptr(src_idx), _stream(stream)))
    return packed, cu_seqlens


def ragged_mask_l2(x: torch.Tensor, tau: float, keep: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Threshold-l2 keep mask of x [B, L_full, C] (f16 / bf16 / f32, unit stride
    along C): keep[b, j] = 1 when ||x[b, j]||_2 >= tau, and always for j = 0."""
    B, L_full, C = x.shape
    if x.stride(2) != 1 or x.stride(0) != L_full * x.stride(1):
        raise ValueError("x must be [B, L_full, C] with unit stride along C and tokens evenly spaced")
    if keep is None:
        keep = torch.empty((B, L_full), dtype=torch.uint8, device=x.device)
    _check(load().ragged_mask_l2(_ptr(x), B, L_full, C, x.stride(1), _dtype_code(x), float(tau), _ptr(keep),
                                 _stream(stream)))
    return keep


def ragged_pack_topk(dense: torch.Tensor, scores: torch.Tensor, keep_count: torch.Tensor,
                     packed: Optional[torch.Tensor] = None, cu_seqlens: Optional[torch.Tensor] = None,
                     src_idx: Optional[torch.Tensor] = None, keep_out: Optional[torch.Tensor] = None, stream=None):
    """Top-k selection fused into pack.  dense [B, L_full, ...] contiguous, scores
    float32 [B, L_full], keep_count int32 [B] (survivors per image, CLS included)
    -> (packed, cu_seqlens); keep_out (uint8 [B, L_full]) receives the selection."""
    B, L_full = int(scores.shape[0]), int(scores.shape[1])
    if not dense.is_contiguous() or tuple(dense.shape[:2]) != (B, L_full):
        raise ValueError("dense must be contiguous [B, L_full, ...]")
    if scores.dtype != torch.float32 or not scores.is_contiguous():
        raise ValueError("scores must be contiguous float32 [B, L_full]")
    if keep_count.dtype != torch.int32 or keep_count.numel() != B:
        raise ValueError("keep_count must be int32 [B]")
    row_bytes = dense.element_size() * (dense[0, 0].numel() if B else int(torch.tensor(dense.shape[2:]).prod()))
    if packed is None:
        packed = torch.empty((B * L_full,) + tuple(dense.shape[2:]), dtype=dense.dtype, device=dense.device)
    if cu_seqlens is None:
        cu_seqlens = torch.empty(B + 1, dtype=torch.int32, device=dense.device)
    _check(load().ragged_pack_topk(_ptr(dense), B, L_full, row_bytes, _ptr(scores), _ptr(keep_count), _ptr(packed),
                                   _ptr(cu_seqlens), _ptr(src_idx), _ptr(keep_out), _stream(stream)))
    return packed, cu_seqlens


def ragged_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor,
                    max_seqlen: int, scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                    cls_out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """q, k, v: [T, H, 64] views sharing strides (e.g. slices of a packed [T, 3, H, 64]).

    Returns out [T, H, 64] (allocated if not given).  cls_out [B, H, 64] is filled
    with each sequence's first row when given.
    """
    T, H, d = q.shape
    if not (q.stride() == k.stride() == v.stride()) or q.stride(2) != 1:
        raise ValueError("q, k, v must share strides with unit innermost stride")
    B = int(cu_seqlens.shape[0]) - 1
    if out is None:
        out = torch.empty((T, H, d), dtype=q.dtype, device=q.device)
    if out.stride(2) != 1 or out.stride(1) != d:
        raise ValueError("out must be [T, H, head_dim] with contiguous heads")
    if scale is None:
        scale = d ** -0.5
    _check(load().ragged_attn_fwd(_ptr(q), _ptr(k), _ptr(v), q.stride(0), q.stride(1), _ptr(cu_seqlens),
                                  B, int(max_seqlen), H, d, float(scale), _dtype_code(q), _ptr(out),
                                  out.stride(0), _ptr(cls_out), _stream(stream)))
    return out


def ragged_unpack_cls(packed: torch.Tensor, cu_seqlens: torch.Tensor, cls_out: Optional[torch.Tensor] = None,
                      stream=None) -> torch.Tensor:
    B = int(cu_seqlens.shape[0]) - 1
    if not packed.is_contiguous():
        raise ValueError("packed must be contiguous")
    row_bytes = packed.element_size() * packed[0].numel()
    if cls_out is None:
        cls_out = torch.empty((B,) + tuple(packed.shape[1:]), dtype=packed.dtype, device=packed.device)
    _check(load().ragged_unpack_cls(_ptr(packed), _ptr(cu_seqlens), B, row_bytes, _ptr(cls_out),
                                    _stream(stream)))
    return cls_out


def ragged_unpack(packed: torch.Tensor, cu_seqlens: torch.Tensor, keep: torch.Tensor,
                  dense_out: torch.Tensor, stream=None) -> torch.Tensor:
    B, L_full = int(keep.shape[0]), int(keep.shape[1])
    if not dense_out.is_contiguous() or tuple(dense_out.shape[:2]) != (B, L_full):
        raise ValueError("dense_out must be contiguous [B, L_full, ...]")
    row_bytes = dense_out.element_size() * (dense_out[0, 0].numel() if B else 16)
    _check(load().ragged_unpack(_ptr(packed), _ptr(cu_seqlens), _ptr(keep), B, L_full, row_bytes,
                                _ptr(dense_out), _stream(stream)))
    return dense_out


def ragged_pipeline(dense_qkv: torch.Tensor, keep: torch.Tensor, scale: Optional[float] = None,
                    packed_qkv=None, cu_seqlens=None, out=None, cls_out=None,
                    flags: int = RAGGED_PIPELINE_AUTO, materialize_packed: bool = True, stream=None):
    """dense_qkv [B, L_full, 3, H, 64] -> (packed_qkv or None, cu_seqlens, out [cap, H, 64], cls_out [B, H, 64]).

    With materialize_packed=False the fused mode does not write the packed q/k/v.
    """
    B, L_full, three, H, d = dense_qkv.shape
    dev, dt = dense_qkv.device, dense_qkv.dtype
    if packed_qkv is None and materialize_packed:
        packed_qkv = torch.empty((B * L_full, 3, H, d), dtype=dt, device=dev)
    if cu_seqlens is None:
        cu_seqlens = torch.empty(B + 1, dtype=torch.int32, device=dev)
    if out is None:
        out = torch.empty((B * L_full, H, d), dtype=dt, device=dev)
    if cls_out is None:
        cls_out = torch.empty((B, H, d), dtype=dt, device=dev)
    if scale is None:
        scale = d ** -0.5
    _check(load().ragged_pipeline(_ptr(dense_qkv), _ptr(keep), B, L_full, H, d, float(scale),
                                  _dtype_code(dense_qkv), _ptr(packed_qkv), _ptr(cu_seqlens), _ptr(out),
                                  _ptr(cls_out), int(flags), _stream(stream)))
    return packed_qkv, cu_seqlens, out, cls_out


def ragged_pipeline_noalloc(dense_qkv: torch.Tensor, keep: torch.Tensor, cu_seqlens: torch.Tensor,
                            out: torch.Tensor, cls_out: Optional[torch.Tensor] = None,
                            scale: Optional[float] = None, stream=None):
    """ragged_pipeline's two-launch form with the packed q/k/v in the library's
    fixed device array: allocates nothing, so every output is passed in.

    dense_qkv [B, L_full, 3, H, 64]; cu_seqlens int32 [B + 1]; out [B * L_full, H, 64];
    cls_out [B, H, 64] or None.  B * L_full * 3 * H * 64 * element size must not
    exceed RAGGED_NOALLOC_SCRATCH_BYTES.  Calls that overlap on the GPU race on
    the shared array.
    """
    B, L_full, three, H, d = dense_qkv.shape
    if scale is None:
        scale = d ** -0.5
    _check(load().ragged_pipeline_noalloc(_ptr(dense_qkv), _ptr(keep), B, L_full, H, d, float(scale),
                                          _dtype_code(dense_qkv), _ptr(cu_seqlens), _ptr(out), _ptr(cls_out),
                                          _stream(stream)))
    return cu_seqlens, out, cls_out


def ragged_get_device_status(stream=None) -> int:
    """Reads and clears the device status word (synchronises with the stream)."""
    val = ctypes.c_uint32(0)
    _check(load().ragged_get_device_status(ctypes.byref(val), _stream(stream)))
    return int(val.value)


class _PipelineArgs(ctypes.Structure):
    """The parameters of ragged_pipeline, in order (argument block of _fastcall)."""
    _fields_ = [("dense_qkv", ctypes.c_void_p), ("keep", ctypes.c_void_p), ("B", ctypes.c_int64),
                ("L_full", ctypes.c_int64), ("H", ctypes.c_int64), ("head_dim", ctypes.c_int64),
                ("scale", ctypes.c_float), ("dtype", ctypes.c_int32), ("packed_qkv", ctypes.c_void_p),
                ("cu_seqlens", ctypes.c_void_p), ("out", ctypes.c_void_p), ("cls_out", ctypes.c_void_p),
                ("flags", ctypes.c_uint32), ("stream", ctypes.c_void_p)]


class _GraphArgs(ctypes.Structure):
    """The parameters of ragged_pipeline_graph_launch (argument block of _fastcall.graph_run)."""
    _fields_ = [("graph", ctypes.c_void_p), ("stream", ctypes.c_void_p), ("flags", ctypes.c_uint32)]


_fast = None


def _fast_forwarder():
    """The single-crossing forwarder, bound to the loaded library (None if not built)."""
    global _fast
    if _fast is None:
        try:
            import importlib
            fc = importlib.import_module(__name__ + "._fastcall")
        except ImportError:
            _fast = False
            return None
        if fc.args_size() != ctypes.sizeof(_PipelineArgs):
            raise RuntimeError("_fastcall argument block does not match the binding")
        fc.bind(ctypes.cast(load().ragged_pipeline, ctypes.c_void_p).value)
        if fc.graph_args_size() != ctypes.sizeof(_GraphArgs):
            raise RuntimeError("_fastcall graph argument block does not match the binding")
        fc.bind_graph(ctypes.cast(load().ragged_pipeline_graph_launch, ctypes.c_void_p).value)
        _fast = fc
    return _fast or None


class Pipeline:
    """Pre-marshalled pack -> attend -> CLS for one (B, L_full, H, dtype) shape.

    Buffers are allocated once; ``__call__`` is a single call into the C ABI with
    cached ctypes arguments (the host dispatch path), and ``capture`` records the
    same launches into a CUDA graph that ``replay`` launches with one call.
    """

    def __init__(self, B: int, L_full: int, H: int, dtype: torch.dtype, device="cuda",
                 scale: Optional[float] = None, head_dim: int = 64, flags: int = RAGGED_PIPELINE_AUTO,
                 materialize_packed: bool = True):
        self.B, self.L_full, self.H, self.d = B, L_full, H, head_dim
        self.dtype = dtype
        self.flags = flags
        dev = torch.device(device)
        self.dense_qkv = torch.empty((B, L_full, 3, H, head_dim), dtype=dtype, device=dev)
        self.keep = torch.empty((B, L_full), dtype=torch.uint8, device=dev)
        self.packed_qkv = (torch.empty((B * L_full, 3, H, head_dim), dtype=dtype, device=dev)
                           if materialize_packed else None)
        self.cu_seqlens = torch.empty(B + 1, dtype=torch.int32, device=dev)
        self.out = torch.empty((B * L_full, H, head_dim), dtype=dtype, device=dev)
        self.cls_out = torch.empty((B, H, head_dim), dtype=dtype, device=dev)
        self.scale = head_dim ** -0.5 if scale is None else scale
        self.graph = None
        self.bind_inputs(self.dense_qkv, self.keep)

    def bind_inputs(self, dense_qkv: torch.Tensor, keep: torch.Tensor, stream=None) -> None:
        """Point the cached call at other input buffers of the same shape."""
        assert dense_qkv.shape == self.dense_qkv.shape and keep.shape == self.keep.shape
        self._inputs = (dense_qkv, keep)
        c = ctypes
        self._args = (c.c_void_p(dense_qkv.data_ptr()), c.c_void_p(keep.data_ptr()), c.c_int64(self.B),
                      c.c_int64(self.L_full), c.c_int64(self.H), c.c_int64(self.d), c.c_float(self.scale),
                      c.c_int(DTYPE_CODES[self.dtype]), c.c_void_p(_ptr(self.packed_qkv)),
                      c.c_void_p(self.cu_seqlens.data_ptr()), c.c_void_p(self.out.data_ptr()),
                      c.c_void_p(self.cls_out.data_ptr()), c.c_uint32(self.flags), c.c_void_p(_stream(stream)))
        self._fn = load().ragged_pipeline
        self._block = _PipelineArgs(*[a.value for a in self._args])
        self._block_sync = _PipelineArgs(*[a.value for a in self._args])
        self._block_sync.flags = self.flags | RAGGED_PIPELINE_SYNC
        self._block_addr = ctypes.addressof(self._block)
        self._block_sync_addr = ctypes.addressof(self._block_sync)
        self._fc = _fast_forwarder()

    def __call__(self) -> None:
        """Enqueue pack -> attend -> CLS on the bound stream."""
        st = self._fc.run(self._block_addr) if self._fc else self._fn(*self._args)
        if st:
            _check(st)

    def run_sync(self) -> None:
        """Enqueue the pipeline and return once it has finished (one call)."""
        st = self._fc.run(self._block_sync_addr) if self._fc else \
            self._fn(*self._args[:12], ctypes.c_uint32(self.flags | RAGGED_PIPELINE_SYNC), self._args[13])
        if st:
            _check(st)

    def capture(self) -> None:
        """Record the pipeline's launches into a CUDA graph (on a side stream)."""
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.bind_inputs(*self._inputs, stream=s)
            self()  # warm-up: sets per-device kernel attributes outside capture
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                self()
        torch.cuda.current_stream().wait_stream(s)
        self.bind_inputs(*self._inputs)
        self.graph = g

    def record(self, stream=None) -> None:
        """Record the pipeline as a CUDA graph that libragged owns
        (ragged_pipeline_graph_create); launch() then costs one crossing into
        the library: one graph launch, and with sync=True the wait for it."""
        lib = load()
        strm = _stream(stream)
        a = self._args
        handle = ctypes.c_void_p()
        _check(lib.ragged_pipeline_graph_create(a[0], a[1], a[2], a[3], a[4], a[5], a[6], a[7], a[8], a[9],
                                                a[10], a[11], ctypes.c_uint32(self.flags), ctypes.c_void_p(strm),
                                                ctypes.byref(handle)))
        self.release()
        self._graph_handle = handle
        self._graph_block = _GraphArgs(handle.value, strm, RAGGED_PIPELINE_SYNC)
        self._graph_block_async = _GraphArgs(handle.value, strm, 0)
        self._graph_block_addr = ctypes.addressof(self._graph_block)
        self._graph_block_async_addr = ctypes.addressof(self._graph_block_async)

    def launch(self, sync: bool = True) -> None:
        """Launch the graph recorded by record(); with sync=True, return once it has finished."""
        addr = self._graph_block_addr if sync else self._graph_block_async_addr
        st = self._fc.graph_run(addr) if self._fc else \
            load().ragged_pipeline_graph_launch(self._graph_handle, ctypes.c_void_p(self._graph_block.stream),
                                                ctypes.c_uint32(self._graph_block.flags if sync else 0))
        if st:
            _check(st)

    def release(self) -> None:
        """Free the graph recorded by record(), if any."""
        h = getattr(self, "_graph_handle", None)
        if h is not None and h.value:
            load().ragged_pipeline_graph_destroy(h)
        self._graph_handle = None

    def __del__(self):
        try:
            self.release()
        except Exception:  # noqa: BLE001 - interpreter shutdown
            pass

    def replay(self) -> None:
        self.graph.replay()
