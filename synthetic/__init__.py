"""Seeded synthetic workloads for the pack -> attend -> unpack pipeline.

This module only draws random inputs: keep masks with the per-image survivor
counts of each workload, and N(0,1) query/key/value values stored in the
16-bit or 32-bit format a workload runs in.  It holds none of the pipeline's
arithmetic (no prefix sums, no packing, no attention); both the CUDA path and
the CPU oracle consume the arrays it returns.

Workload shapes follow "Dispatch-Aware Ragged Attention for Pruned Vision
Transformers" (DeiT-S: 6 heads, DeiT-B: 12 heads, head_dim 64, 197 tokens at
224x224 and 577 at 384x384; abstract and the radpulse article's sections on
the FA2 dispatch ceiling and the pack pipeline).  ImageNet and trained pruning
predictors are not used: survivor sets are the top-k of seeded N(0,1) scores,
with the CLS token (index 0) always kept.

Storage conventions (numpy):
  f16  -> np.float16
  bf16 -> np.uint16 holding the bfloat16 bit pattern
  f32  -> np.float32
Dense q/k/v are one fused array [B, L_full, 3, H, d] (q, k, v along axis 2).
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import numpy as np

DTYPES = ("f16", "bf16", "f32")
ELEM_BYTES = {"f16": 2, "bf16": 2, "f32": 4}

# Pruning rates of the serving and throughput workloads.
SERVING_BATCHES = (1, 2, 4)
SERVING_RATES = (0.0, 0.25, 0.50, 0.80)
SWEEP_RATES = tuple(round(0.1 * i, 1) for i in range(10))


def rng_for(seed: int, sub: int = 0) -> np.random.Generator:
    """PCG64 stream for workload ``seed`` and sub-case ``sub``."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), int(sub)])))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest even); returns uint16 bits.

    NaNs are kept quiet NaNs.  Used only to store synthetic inputs.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    nan = np.isnan(x)
    out = rounded.astype(np.uint16)
    out[nan] = ((u[nan] >> 16) | 0x40).astype(np.uint16)
    return out


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def store(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32/float64 samples to the storage format of ``dtype``."""
    if dtype == "f16":
        return np.asarray(x, dtype=np.float32).astype(np.float16)
    if dtype == "bf16":
        return f32_to_bf16_bits(np.asarray(x, dtype=np.float32))
    if dtype == "f32":
        return np.asarray(x, dtype=np.float32)
    raise ValueError(f"unknown dtype {dtype!r}")


def to_float64(x: np.ndarray, dtype: str) -> np.ndarray:
    """Exact widening of stored values, for reporting only (not used by the oracle)."""
    if dtype == "bf16":
        return bf16_bits_to_f32(x).astype(np.float64)
    return np.asarray(x).astype(np.float64)


def topk_keep_mask(rng: np.random.Generator, L_full: int, lengths: Sequence[int]) -> np.ndarray:
    """uint8 [B, L_full] keep mask: CLS plus the top-(L_b - 1) of N(0,1) scores.

    Ties (probability zero for continuous scores) go to the lower index.
    """
    lengths = np.asarray(lengths, dtype=np.int64)
    B = lengths.shape[0]
    if np.any(lengths < 1) or np.any(lengths > L_full):
        raise ValueError("every survivor count must lie in [1, L_full]")
    scores = rng.standard_normal((B, max(L_full - 1, 0)))
    keep = np.zeros((B, L_full), dtype=np.uint8)
    keep[:, 0] = 1
    for b in range(B):
        k = int(lengths[b]) - 1
        if k > 0:
            order = np.argsort(-scores[b], kind="stable")[:k]
            keep[b, order + 1] = 1
    return keep


def _round_half_up(x: np.ndarray) -> np.ndarray:
    return np.floor(np.asarray(x, dtype=np.float64) + 0.5).astype(np.int64)


@dataclasses.dataclass
class Workload:
    """One batch of synthetic input for the pipeline."""

    name: str
    B: int
    L_full: int
    H: int
    d: int
    dtype: str
    lengths: np.ndarray          # int64 [B], survivors per image incl. CLS
    keep: np.ndarray             # uint8 [B, L_full]
    qkv: np.ndarray              # [B, L_full, 3, H, d] in storage format
    scale: float = 0.125
    tokens: Optional[np.ndarray] = None   # float32 [B, L_full, C] (tiny workload only)
    weights: Optional[np.ndarray] = None  # float32 [3, C, H*d] (tiny workload only)
    rate: Optional[float] = None

    @property
    def D(self) -> int:
        return self.H * self.d

    @property
    def T(self) -> int:
        return int(self.lengths.sum())

    @property
    def elem_bytes(self) -> int:
        return ELEM_BYTES[self.dtype]

    @property
    def row_bytes(self) -> int:
        """Bytes of one dense token row of the fused q/k/v array."""
        return 3 * self.H * self.d * self.elem_bytes

    @property
    def Lmax(self) -> int:
        return int(self.lengths.max()) if self.B else 0

    def useful_flops(self) -> int:
        """Unpadded attention FLOPs: QK^T and PV, a multiply-add counted as 2."""
        L = self.lengths.astype(np.int64)
        return int(4 * self.d * self.H * int((L * L).sum()))


def make_workload(name: str, B: int, L_full: int, H: int, lengths, dtype: str,
                  seed: int, sub: int = 0, d: int = 64, rate=None) -> Workload:
    """Generic workload: given survivor counts, draw a top-k mask and N(0,1) q/k/v."""
    if dtype not in DTYPES:
        raise ValueError(dtype)
    rng = rng_for(seed, sub)
    lengths = np.asarray(lengths, dtype=np.int64).reshape(B)
    keep = topk_keep_mask(rng, L_full, lengths)
    qkv = store(rng.standard_normal((B, L_full, 3, H, d), dtype=np.float32), dtype)
    return Workload(name, B, L_full, H, d, dtype, lengths, keep, qkv, rate=rate)


# --------------------------------------------------------------------------
# The five workloads.
# --------------------------------------------------------------------------

def tiny(dtype: str = "f16", seed: int = 1001) -> Workload:
    """B=4 DeiT-S images, keep counts {197,120,60,40}; q/k/v = tokens . W.

    tokens [4,197,384] float32 N(0,1); W_q, W_k, W_v float32 N(0, 1/384),
    head h = output columns 64h..64h+63.  The projection is a model layer
    outside the pipeline; it is applied here, on the host, in float64, rounded
    to float32 (the tokens' format) and then stored in ``dtype``.  It acts row
    by row, so it commutes with packing.
    """
    rng = rng_for(seed, 0)
    B, L_full, C, H, d = 4, 197, 384, 6, 64
    lengths = np.array([197, 120, 60, 40], dtype=np.int64)
    tokens = rng.standard_normal((B, L_full, C), dtype=np.float32)
    weights = (rng.standard_normal((3, C, H * d), dtype=np.float64) / np.sqrt(C)).astype(np.float32)
    keep = topk_keep_mask(rng, L_full, lengths)
    proj = np.einsum("blc,tcn->bltn", tokens.astype(np.float64), weights.astype(np.float64))
    qkv = store(proj.reshape(B, L_full, 3, H, d).astype(np.float32), dtype)
    return Workload("tiny_deit_s_b4", B, L_full, H, d, dtype, lengths, keep, qkv,
                    tokens=tokens, weights=weights)


def deit_b_pruned80(seed: int = 1002) -> Workload:
    """DeiT-B at 80% pruning: B=32, 197 tokens, 12 heads, bf16, L_b ~ U{30..48}."""
    rng = rng_for(seed, 0)
    lengths = rng.integers(30, 49, size=32)
    return make_workload("deit_b_p80_b32", 32, 197, 12, lengths, "bf16", seed, 1)


def serving_lengths(rng: np.random.Generator, B: int, rate: float, L_full: int = 197) -> np.ndarray:
    """Per-image survivors at pruning ``rate`` with +-10 percentage points jitter.

    p_b = clamp(rate + U[-0.1, 0.1], 0, 0.95) (no jitter at rate 0);
    L_b = 1 + round((1 - p_b) * (L_full - 1)).
    """
    if rate == 0.0:
        p = np.zeros(B)
    else:
        p = np.clip(rate + rng.uniform(-0.10, 0.10, size=B), 0.0, 0.95)
    return 1 + _round_half_up((1.0 - p) * (L_full - 1))


def serving(B: int, rate: float, seed: int = 1003, copy: int = 0) -> Workload:
    """DeiT-S serving regime: B in {1,2,4}, 6 heads, f16, 197 tokens.

    ``copy`` selects an independent draw of the same workload (used to rotate
    several input sets through memory so that timing does not hit L2).
    """
    sub = 2 * (100_000 * copy + 1000 * B + int(round(rate * 100)))
    lengths = serving_lengths(rng_for(seed, sub), B, rate)
    return make_workload(f"serving_b{B}_p{int(round(rate * 100))}", B, 197, 6, lengths,
                         "f16", seed, sub + 1, rate=rate)


def hires_384(seed: int = 1004, B: int = 64) -> Workload:
    """384x384 DeiT-B: 577 tokens, 12 heads, bf16, keep ratio r ~ U[0.3, 0.7]."""
    rng = rng_for(seed, 0)
    r = rng.uniform(0.3, 0.7, size=B)
    lengths = 1 + _round_half_up(r * 576)
    return make_workload(f"hires384_b{B}", B, 577, 12, lengths, "bf16", seed, 1)


def sweep_lengths(rng: np.random.Generator, B: int, rate: float, L_full: int = 197,
                  sigma: float = 8.0) -> np.ndarray:
    """Truncated-normal survivor counts around 1 + round((1 - rate)(L_full - 1)).

    Each draw round(N(target, sigma)) outside [1, L_full] is redrawn.  At rate 0
    nothing is pruned and every image keeps all L_full tokens.
    """
    if rate == 0.0:
        return np.full(B, L_full, dtype=np.int64)
    target = 1 + int(_round_half_up((1.0 - rate) * (L_full - 1)))
    out = np.empty(B, dtype=np.int64)
    for b in range(B):
        while True:
            x = int(_round_half_up(rng.normal(target, sigma)))
            if 1 <= x <= L_full:
                out[b] = x
                break
    return out


def sweep(rate: float, seed: int = 1005, B: int = 512) -> Workload:
    """Throughput sweep: B=512 DeiT-S images, f16, pruning ``rate`` in 0..0.9."""
    idx = int(round(rate * 10))
    rng = rng_for(seed + idx, 0)
    lengths = sweep_lengths(rng, B, rate)
    return make_workload(f"sweep_b{B}_p{int(round(rate * 100))}", B, 197, 6, lengths, "f16",
                         seed + idx, 1, rate=rate)
