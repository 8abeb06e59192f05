"""fp8 (e4m3) latent rows with per-token scales, fp64 reference.

TEST INFRASTRUCTURE ONLY (see the package docstring): only tests/,
__graft_entry__.smoke() and bench.py's CPU legs use it.

Source: HLA summary, "Conclusion / Future directions" ("combining with
quantization") and "Practical Implications" (latent caching is
complementary to quantization).  The pages give no format; the reading taken
here is the plainest per-token scheme:

* Format: OCP FP8 E4M3 ("e4m3fn": 4 exponent bits, bias 7, 3 mantissa bits,
  no infinities, largest finite 448, subnormal spacing 2^-9), rounding to
  nearest with ties to even, values beyond +-448 saturated to +-448.
* Scales: one per token and part -- the key part c^K (rotated for HLA) and the
  value part c^V each get s = max_k |c_k| / 448, so the largest element maps
  to +-448.  The writer's latent is first rounded to binary32 (its fp32
  result); the maximum, the scale (s = amax / 448) and each quotient c_k / s
  are binary32 operations (correctly rounded), then each quotient is rounded
  to e4m3.  A part that is all zero gets s = 0 and zero codes.
* Value of a stored element: code * s (exact in fp64).
* Row bytes: [codes of c^K (r_k) | codes of c^V (r_v) | s^K fp32 | s^V fp32 |
  8 zero bytes]: r_k + r_v + 16 bytes per token.
"""

import numpy as np

E4M3_MAX = 448.0


def to_e4m3(x):
    """Round fp64 values to e4m3fn (nearest-even, saturating); fp64 out."""
    x = np.asarray(x, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("e4m3 rounding of non-finite values is not defined here")
    ax = np.abs(x)
    _, ex = np.frexp(ax)                 # ax = m * 2^ex, m in [0.5, 1)
    e = np.maximum(ex - 1, -6)           # binade exponent; below 2^-6 the subnormal spacing
    step = np.ldexp(1.0, e - 3)          # 3 mantissa bits
    q = np.round(ax / step) * step       # numpy rounds halves to even
    q = np.minimum(q, E4M3_MAX)
    return np.where(np.signbit(x), -q, q)


def _part(c32):
    amax = np.float32(np.max(np.abs(c32))) if c32.size else np.float32(0.0)
    if amax == 0.0:
        return np.zeros_like(c32, dtype=np.float64), np.float32(0.0)
    s = np.float32(amax / np.float32(E4M3_MAX))          # binary32 division
    quot = (c32 / s).astype(np.float32)                   # binary32 division per element
    return to_e4m3(quot.astype(np.float64)), s


def quantize_rows(c, r_k, r_v):
    """Quantize latent rows c [n, r_k + r_v] (exact values).

    Returns (codes [n, r_k + r_v] fp64, sK [n] and sV [n] as fp32 arrays)."""
    c = np.asarray(c, dtype=np.float64)
    c32 = c.astype(np.float32)
    n = c.shape[0]
    codes = np.zeros((n, r_k + r_v))
    sK = np.zeros(n, dtype=np.float32)
    sV = np.zeros(n, dtype=np.float32)
    for j in range(n):
        codes[j, :r_k], sK[j] = _part(c32[j, :r_k])
        codes[j, r_k:], sV[j] = _part(c32[j, r_k:r_k + r_v])
    return codes, sK, sV


def dequantize_rows(codes, sK, sV, r_k):
    """Values of stored rows: code * scale of its part (fp64)."""
    out = np.array(codes, dtype=np.float64)
    out[:, :r_k] *= np.asarray(sK, dtype=np.float64)[:, None]
    out[:, r_k:] *= np.asarray(sV, dtype=np.float64)[:, None]
    return out


def e4m3_bits(v):
    """uint8 encodings of e4m3fn values (exactly representable fp64 inputs)."""
    v = np.asarray(v, dtype=np.float64)
    sign = np.signbit(v).astype(np.uint8) << 7
    a = np.abs(v)
    _, ex = np.frexp(a)
    e = ex - 1
    normal = a >= 2.0 ** -6
    exp_field = np.where(normal, e + 7, 0)
    mant = np.where(normal, a / np.ldexp(1.0, e) - 1.0, a / 2.0 ** -6) * 8.0
    mant = np.where(a == 0, 0, mant)
    exp_field = np.where(a == 0, 0, exp_field)
    if not np.all(mant == np.round(mant)):
        raise ValueError("value is not an e4m3 number")
    return (sign | (exp_field.astype(np.uint8) << 3) | mant.astype(np.uint8)).astype(np.uint8)


def row_bytes(codes, sK, sV):
    """The stored bytes of rows [n, r_k + r_v + 16] (uint8)."""
    codes = np.asarray(codes)
    n, w = codes.shape
    out = np.zeros((n, w + 16), dtype=np.uint8)
    out[:, :w] = e4m3_bits(codes)
    out[:, w:w + 4] = np.asarray(sK, dtype=np.float32).reshape(n, 1).view(np.uint8)
    out[:, w + 4:w + 8] = np.asarray(sV, dtype=np.float32).reshape(n, 1).view(np.uint8)
    return out


def from_row_bytes(rows, r_k, r_v):
    """Values of stored fp8 rows given as bytes [n, r_k + r_v + 16] (uint8):
    each code decoded from its e4m3 bit pattern, times its part's scale."""
    rows = np.asarray(rows, dtype=np.uint8)
    w = r_k + r_v
    b = rows[:, :w].astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 7).astype(np.float64)
    if np.any((e == 15) & (m == 7)):
        raise ValueError("NaN code in a latent row")
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.ldexp(1.0, e - 7))
    codes = sign * mag
    sK = rows[:, w:w + 4].copy().view(np.float32)[:, 0]
    sV = rows[:, w + 4:w + 8].copy().view(np.float32)[:, 0]
    return dequantize_rows(codes, sK, sV, r_k)


def to_storage_fp8(c, r_k, r_v):
    """Convenience: the values the read sees for exact rows c."""
    codes, sK, sV = quantize_rows(c, r_k, r_v)
    return dequantize_rows(codes, sK, sV, r_k)


__all__ = ["E4M3_MAX", "to_e4m3", "quantize_rows", "dequantize_rows", "e4m3_bits", "row_bytes",
           "from_row_bytes", "to_storage_fp8"]
