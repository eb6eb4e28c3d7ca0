"""Test-side marshalling between numpy (synthetic inputs, oracle) and torch device tensors."""
import numpy as np
import torch

TORCH_DTYPE = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}

# Attention tolerances against the fp64 oracle.
#  f16 / bf16: max-abs 4e-3.  The output is rounded to the input format; a bf16
#    value of magnitude >= 2 is already up to half a unit in the last place
#    (7.8e-3 on [2, 4)) away from the exact result after rounding alone, more
#    than 4e-3.  For every element the bound is therefore the larger of 4e-3
#    and that half-unit plus 1/64 of it (the room left to the fp32 arithmetic
#    before the final rounding).  This only changes the bound for bf16 outputs
#    of magnitude >= 2 and f16 outputs of magnitude >= 8.
#  f32 check path: normwise, max |gpu - oracle| <= 1e-5 max |oracle|.
TOL_16BIT = 4e-3
TOL_F32_REL = 1e-5


def half_ulp(x: np.ndarray, mantissa_bits: int) -> np.ndarray:
    """Half a unit in the last place of a format with `mantissa_bits` stored
    fraction bits, at the magnitude of x (normal range)."""
    ax = np.maximum(np.abs(x), np.finfo(np.float64).tiny)
    return np.ldexp(1.0, np.floor(np.log2(ax)).astype(np.int64) - mantissa_bits - 1)


def bound_16bit(ref: np.ndarray, dtype: str) -> np.ndarray:
    bits = 7 if dtype == "bf16" else 10
    return np.maximum(TOL_16BIT, half_ulp(ref, bits) * (1.0 + 1.0 / 64))


def to_device(x: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    """Same bytes on the device: f16 / f32 as is, bf16 from its uint16 bit patterns."""
    x = np.ascontiguousarray(x)
    if dtype == "bf16":
        return torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(x).to(device)


def to_host_bits(t: torch.Tensor, dtype: str) -> np.ndarray:
    """Device tensor back to the synthetic storage format (bit-exact)."""
    t = t.detach().contiguous().cpu()
    if dtype == "bf16":
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a device result to float64."""
    return t.detach().cpu().to(torch.float64).numpy()


def attn_error(gpu: np.ndarray, ref: np.ndarray, dtype: str):
    """(error, bound) for the worst element.

    16-bit formats: the element with the largest error / bound ratio, bounds as
    described above.  fp32: normwise max error against 1e-5 max |oracle|."""
    if not gpu.size:
        return 0.0, 1.0
    diff = np.abs(gpu - ref)
    if dtype == "f32":
        return float(diff.max()), TOL_F32_REL * float(np.max(np.abs(ref)))
    bound = bound_16bit(ref, dtype)
    i = int(np.argmax(diff / bound))
    return float(diff.flat[i]), float(bound.flat[i])


def round_to_format(x: np.ndarray, dtype: str) -> np.ndarray:
    """x (float64) rounded to nearest even in f16 or bf16, returned as float64.
    Normal range only (the attention outputs here), straight from float64 so
    that no intermediate rounding enters."""
    bits = 7 if dtype == "bf16" else 10
    m, e = np.frexp(x)                                # x = m * 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.round(np.ldexp(m, bits + 1)), e - bits - 1)   # np.round: half to even


def ulps_from_rounded(gpu: np.ndarray, ref: np.ndarray, dtype: str, floor: float = 2.0 ** -10) -> int:
    """Largest distance, in units in the last place of the 16-bit format,
    between each GPU output and the oracle value correctly rounded to that
    format.  Elements with |oracle| below `floor` are left out: near zero a
    unit in the last place shrinks without limit, while the absolute bound of
    attn_error already covers them."""
    sel = np.abs(ref) >= floor
    if not sel.any():
        return 0
    r = round_to_format(ref[sel], dtype)
    bits = 7 if dtype == "bf16" else 10
    ulp = np.ldexp(1.0, np.frexp(np.abs(r))[1] - bits - 1)
    return int(np.max(np.round(np.abs(gpu[sel] - r) / ulp)))
