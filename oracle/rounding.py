"""Rounding of fp64 results to the storage formats of the latent cache.

Latents are stored as bf16 or fp32.  Reading: the writer's exact (fp64)
result is rounded once, to nearest with ties to even, straight to the
storage format (no intermediate fp32 step).  bf16 is the top 16 bits of an
IEEE binary32 with 8 exponent bits and 7 stored mantissa bits.
"""

import numpy as np


def to_f32(x):
    """Round fp64 to IEEE binary32 (nearest-even), returned as fp64 values."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def _bf16_bits_from_f64(x):
    """uint16 bit patterns of round-to-nearest-even(x) in bf16.

    Works from the exact fp64 value: the bf16 neighbours below and above x
    are found from x's binary32 truncation, then the nearer one is chosen,
    ties going to the even mantissa.  Finite inputs only.
    """
    x = np.asarray(x, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("bf16 rounding of non-finite values is not defined here")
    sign = np.signbit(x)
    ax = np.abs(x)
    # Largest bf16 <= ax: take binary32 rounded toward zero, drop low 16 bits.
    f32 = ax.astype(np.float32)
    # astype rounds to nearest; step down where that overshot.
    over = f32.astype(np.float64) > ax
    f32 = np.where(over, np.nextafter(f32, np.float32(0)), f32)
    bits = f32.view(np.uint32) & np.uint32(0xFFFF0000)
    lo = bits.view(np.float32).astype(np.float64)
    hi_bits = bits + np.uint32(0x10000)
    hi = hi_bits.view(np.float32).astype(np.float64)
    d_lo = ax - lo
    d_hi = hi - ax
    lo_even = ((bits >> np.uint32(16)) & np.uint32(1)) == 0
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ~lo_even)
    out = np.where(take_hi, hi_bits, bits).astype(np.uint32)
    out = (out >> np.uint32(16)).astype(np.uint16)
    out = np.where(sign, out | np.uint16(0x8000), out).astype(np.uint16)
    return out


def to_bf16(x):
    """Round fp64 to bf16 (nearest-even); values returned as fp64."""
    bits = _bf16_bits_from_f64(x).astype(np.uint32) << np.uint32(16)
    return bits.view(np.float32).astype(np.float64)


def bf16_bits(x):
    """uint16 bit patterns of to_bf16(x)."""
    return _bf16_bits_from_f64(x)


def from_bf16_bits(bits):
    """fp64 values of uint16 bf16 bit patterns."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def to_storage(x, dtype):
    """Round to the storage format named by ``dtype`` ('bf16' or 'f32')."""
    if dtype == "bf16":
        return to_bf16(x)
    if dtype == "f32":
        return to_f32(x)
    raise ValueError(dtype)
