"""CPU oracle for the pack -> attend -> unpack pipeline (TEST INFRASTRUCTURE ONLY).

The arithmetic lives in ``ragged_oracle.c`` (plain C, fp64, built with gcc);
this module compiles it on first use and marshals numpy arrays to it.  Only
the tests, the smoke check and the benchmark's CPU-baseline leg import it.
The CUDA product path never does, and this module imports nothing from the
product package.

What each function follows ("Dispatch-Aware Ragged Attention for Pruned
Vision Transformers"):
  seqlens / pack      radpulse article, "Integrated pack pipeline": compute
                      cu_seqlens, copy survivors into one contiguous flat buffer
  attention           abstract and radpulse "Bypassing the binding":
                      bidirectional softmax attention per sequence, no causal
                      mask, no KV cache, no padding
  unpack_cls          radpulse "Integrated pack pipeline": extract the CLS token
  unpack              scatter the packed rows back to their dense positions
  mask_topk / mask_l2 keep-mask producers (radpulse "Integrated pack
                      pipeline": the pipeline serves any pruning method, e.g.
                      Threshold-l2); the rules are readings, see the C file
  deit_block_cls      one encoder block on each image's survivors, CLS rows
                      out (radpulse "Integrated pack pipeline": attention and
                      the MLP run on the packed tokens, then CLS is
                      extracted; "Implications": the MLP acts token by token);
                      plain numpy float64
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ragged_oracle.c")
_LIB = os.path.join(_HERE, "_build", "libragged_oracle.so")
_lock = threading.Lock()
_lib = None

DTYPE_CODES = {"f16": 0, "bf16": 1, "f32": 2, "f64": 3}
_STORAGE = {"f16": np.float16, "bf16": np.uint16, "f32": np.float32, "f64": np.float64}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, IEEE semantics) if stale.

    -ffp-contract=off (already the ISO C default) is spelled out: no a + b * c
    may become a fused multiply-add, since the Threshold-l2 sum must round
    every product and every addition on its own."""
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.run(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-Wall", "-Wextra", "-shared", "-fPIC",
                        "-pthread", _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def bind(path: str):
    """Load an oracle shared library at ``path`` and declare its signatures."""
    lib = ctypes.CDLL(path)
    i64, vp = ctypes.c_int64, ctypes.c_void_p
    lib.oracle_seqlens.argtypes = [vp, i64, i64, vp, vp]
    lib.oracle_seqlens.restype = i64
    lib.oracle_pack.argtypes = [vp, i64, i64, i64, vp, vp, vp]
    lib.oracle_pack.restype = i64
    lib.oracle_unpack_cls.argtypes = [vp, vp, i64, i64, vp]
    lib.oracle_unpack_cls.restype = None
    lib.oracle_unpack.argtypes = [vp, vp, i64, i64, i64, vp]
    lib.oracle_unpack.restype = None
    lib.oracle_decode.argtypes = [vp, ctypes.c_int, i64, vp]
    lib.oracle_decode.restype = None
    lib.oracle_attention.argtypes = [vp, vp, vp, ctypes.c_int, i64, i64, vp, i64, i64, i64,
                                     ctypes.c_double, vp, i64, vp, ctypes.c_int]
    lib.oracle_attention.restype = ctypes.c_int
    lib.oracle_num_cores.argtypes = []
    lib.oracle_num_cores.restype = ctypes.c_int
    lib.oracle_mask_topk.argtypes = [vp, i64, i64, vp, vp]
    lib.oracle_mask_topk.restype = None
    lib.oracle_mask_l2.argtypes = [vp, ctypes.c_int, i64, i64, i64, i64, ctypes.c_double, vp]
    lib.oracle_mask_l2.restype = None
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = bind(build())
    return _lib


def use_library(lib) -> None:
    """Swap the loaded oracle library (tests use this to plant mistakes)."""
    global _lib
    with _lock:
        _lib = lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def num_cores() -> int:
    return int(_load().oracle_num_cores())


def seqlens(keep: np.ndarray):
    """keep uint8 [B, L_full] -> (cu_seqlens int32 [B+1], src_idx int32 [T])."""
    keep = np.ascontiguousarray(keep, dtype=np.uint8)
    B, L_full = keep.shape
    cu = np.zeros(B + 1, dtype=np.int32)
    src = np.zeros(max(B * L_full, 1), dtype=np.int32)
    T = _load().oracle_seqlens(_ptr(keep), B, L_full, _ptr(cu), _ptr(src))
    return cu, src[:T].copy()


def pack(dense: np.ndarray, keep: np.ndarray):
    """dense [B, L_full, ...] (any dtype) -> (packed [T, ...], cu int32 [B+1])."""
    dense = np.ascontiguousarray(dense)
    keep = np.ascontiguousarray(keep, dtype=np.uint8)
    B, L_full = keep.shape
    assert dense.shape[:2] == (B, L_full)
    row_bytes = dense.itemsize * int(np.prod(dense.shape[2:], dtype=np.int64))
    packed = np.zeros((max(B * L_full, 1),) + dense.shape[2:], dtype=dense.dtype)
    cu = np.zeros(B + 1, dtype=np.int32)
    T = _load().oracle_pack(_ptr(dense), B, L_full, row_bytes, _ptr(keep), _ptr(packed), _ptr(cu))
    return packed[:T].copy(), cu


def unpack_cls(packed: np.ndarray, cu: np.ndarray) -> np.ndarray:
    """packed [T, ...], cu [B+1] -> cls [B, ...] (row cu[b] of each sequence)."""
    packed = np.ascontiguousarray(packed)
    cu = np.ascontiguousarray(cu, dtype=np.int32)
    B = cu.shape[0] - 1
    row_bytes = packed.itemsize * int(np.prod(packed.shape[1:], dtype=np.int64))
    cls = np.zeros((B,) + packed.shape[1:], dtype=packed.dtype)
    _load().oracle_unpack_cls(_ptr(packed), _ptr(cu), B, row_bytes, _ptr(cls))
    return cls


def unpack(packed: np.ndarray, keep: np.ndarray, dense_out: np.ndarray) -> np.ndarray:
    """Scatter packed rows to their dense positions in a copy of ``dense_out``."""
    packed = np.ascontiguousarray(packed)
    keep = np.ascontiguousarray(keep, dtype=np.uint8)
    out = np.array(dense_out, copy=True, order="C")
    B, L_full = keep.shape
    assert out.shape[:2] == (B, L_full) and out.dtype == packed.dtype
    row_bytes = out.itemsize * int(np.prod(out.shape[2:], dtype=np.int64))
    _load().oracle_unpack(_ptr(packed), _ptr(keep), B, L_full, row_bytes, _ptr(out))
    return out


def decode(x: np.ndarray, dtype: str) -> np.ndarray:
    """Exact widening of stored f16 / bf16-bits / f32 values to float64."""
    x = np.ascontiguousarray(x, dtype=_STORAGE[dtype])
    out = np.empty(x.shape, dtype=np.float64)
    _load().oracle_decode(_ptr(x), DTYPE_CODES[dtype], x.size, _ptr(out))
    return out


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, cu: np.ndarray, dtype: str,
              scale: float = 0.125, seqs: Optional[Sequence[int]] = None,
              threads: int = 0, out: Optional[np.ndarray] = None) -> np.ndarray:
    """Per-sequence softmax attention in float64.

    q, k, v: [T, H, d] arrays in the storage format of ``dtype`` (views with a
    common token stride and head stride are fine, e.g. the three slices of a
    packed fused [T, 3, H, d] array; the innermost stride must be 1).
    Returns float64 [T, H, d]; with ``seqs`` only those sequences' rows are
    computed (the rest are left as in ``out``, zeros by default).
    """
    if not (q.strides == k.strides == v.strides and q.shape == k.shape == v.shape):
        raise ValueError("q, k, v must share shape and strides")
    T, H, d = q.shape
    item = q.itemsize
    if q.strides[2] != item or q.strides[0] % item or q.strides[1] % item:
        raise ValueError("innermost stride must be one element")
    if q.dtype != _STORAGE[dtype]:
        raise ValueError(f"q/k/v dtype {q.dtype} does not store {dtype}")
    cu = np.ascontiguousarray(cu, dtype=np.int32)
    B = cu.shape[0] - 1
    if out is None:
        out = np.zeros((T, H, d), dtype=np.float64)
    assert out.shape == (T, H, d) and out.dtype == np.float64 and out.flags.c_contiguous
    if seqs is None:
        seq_arr, seq_ptr, n = None, None, B
    else:
        seq_arr = np.ascontiguousarray(np.asarray(seqs), dtype=np.int32)
        seq_ptr, n = _ptr(seq_arr), seq_arr.shape[0]
    rc = _load().oracle_attention(_ptr(q), _ptr(k), _ptr(v), DTYPE_CODES[dtype],
                                  q.strides[0] // item, q.strides[1] // item, _ptr(cu), B, H, d,
                                  float(scale), seq_ptr, n, _ptr(out), int(threads))
    if rc != 0:
        raise MemoryError("oracle attention could not allocate its per-sequence buffers")
    return out


def pipeline(w, seqs: Optional[Sequence[int]] = None, threads: int = 0) -> dict:
    """Full pack -> attend -> unpack for a ``synthetic.Workload``.

    Returns cu_seqlens, src_idx, the packed fused q/k/v [T, 3, H, d], the
    float64 attention output [T, H, d] and its CLS rows [B, H, d].
    """
    cu, src = seqlens(w.keep)
    packed, cu2 = pack(w.qkv, w.keep)
    assert np.array_equal(cu, cu2)
    out = attention(packed[:, 0], packed[:, 1], packed[:, 2], cu, w.dtype, w.scale,
                    seqs=seqs, threads=threads)
    cls = out[cu[:-1]] if w.B else np.zeros((0, w.H, w.d))
    return {"cu": cu, "src_idx": src, "packed": packed, "out": out, "cls": cls}


def mask_topk(scores: np.ndarray, keep_count: np.ndarray) -> np.ndarray:
    """Top-k keep mask: CLS plus the k_b - 1 highest-scoring other tokens of
    image b (ties: lower index; NaN ranks last); k_b clamped to [1, L_full]."""
    scores = np.ascontiguousarray(scores, dtype=np.float32)
    B, L_full = scores.shape
    kc = np.ascontiguousarray(keep_count, dtype=np.int32).reshape(B)
    keep = np.zeros((B, L_full), dtype=np.uint8)
    _load().oracle_mask_topk(_ptr(scores), B, L_full, _ptr(kc), _ptr(keep))
    return keep


def mask_l2(x: np.ndarray, dtype: str, tau: float) -> np.ndarray:
    """Threshold-l2 keep mask of x [B, L_full, C] (storage format of dtype):
    token kept when its Euclidean norm is >= tau; CLS always kept."""
    x = np.ascontiguousarray(x)
    if x.dtype != _STORAGE[dtype]:
        raise ValueError(f"x dtype {x.dtype} does not store {dtype}")
    B, L_full, C = x.shape
    keep = np.zeros((B, L_full), dtype=np.uint8)
    _load().oracle_mask_l2(_ptr(x), DTYPE_CODES[dtype], B, L_full, C, C, float(tau), _ptr(keep))
    return keep


def deit_block_cls(x: np.ndarray, keep: np.ndarray, Wqkv: np.ndarray, Wo: np.ndarray, W1: np.ndarray,
                   W2: np.ndarray, H: int, scale: float = 0.125, eps: float = 1e-5) -> np.ndarray:
    """CLS row of one pre-norm transformer encoder block applied to each
    image's surviving tokens, in float64.

    x [B, L_full, D] and the weights are float arrays (widened exactly); keep
    uint8 [B, L_full], token 0 always kept.  Linears carry no bias and the
    layer norms no affine parameters (unit weights, zero biases), so for the
    tokens t of one image:
        h = t + Attn(LN(t)) Wo^T,          Attn per head over the image's own tokens:
                                           softmax(scale q k^T) v, with [q k v] = LN(t) Wqkv^T
        y = h + GELU(LN(h) W1^T) W2^T,     GELU(z) = z (1 + erf(z / sqrt 2)) / 2
    LN(z) = (z - mean) / sqrt(var + eps), var the biased variance over D.
    Returns y[CLS] for every image, [B, D] float64.
    """
    from math import erf, sqrt
    x = np.asarray(x, dtype=np.float64)
    Wqkv, Wo, W1, W2 = (np.asarray(w, dtype=np.float64) for w in (Wqkv, Wo, W1, W2))
    B, L_full, D = x.shape
    d = D // H
    erf_v = np.vectorize(erf)

    def layer_norm(z):
        mu = z.mean(axis=1, keepdims=True)
        var = ((z - mu) ** 2).mean(axis=1, keepdims=True)
        return (z - mu) / np.sqrt(var + eps)

    out = np.zeros((B, D), dtype=np.float64)
    for b in range(B):
        kept = np.asarray(keep[b]) != 0
        kept[0] = True
        t = x[b][kept]                                   # [L_b, D], ascending token order
        qkv = layer_norm(t) @ Wqkv.T                     # [L_b, 3D]
        q, k, v = qkv[:, :D], qkv[:, D:2 * D], qkv[:, 2 * D:]
        att = np.zeros_like(t)
        for h in range(H):
            c = slice(h * d, (h + 1) * d)
            s = scale * (q[:, c] @ k[:, c].T)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            att[:, c] = (p / p.sum(axis=1, keepdims=True)) @ v[:, c]
        hres = t + att @ Wo.T
        z = layer_norm(hres) @ W1.T
        y = hres + (0.5 * z * (1.0 + erf_v(z / sqrt(2.0)))) @ W2.T
        out[b] = y[0]
    return out
