"""Pins for the oracle's fp8 (e4m3) latent rows with per-token scales (CPU)."""

import numpy as np
import torch

from oracle import quant


def test_e4m3_rounding_matches_library():
    """In-range binary32 inputs: the oracle's e4m3 rounding equals torch's
    float32 -> float8_e4m3fn conversion, value and bit pattern."""
    rng = np.random.default_rng(0)
    x = np.concatenate([
        (rng.standard_normal(200000) * 60).astype(np.float32),
        (rng.standard_normal(20000) * 1e-3).astype(np.float32),
        np.array([0.0, -0.0, 448.0, -448.0, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -11], dtype=np.float32),
    ])
    x = x[np.abs(x) <= 448.0]
    ours = quant.to_e4m3(x.astype(np.float64))
    lib = torch.from_numpy(x).to(torch.float8_e4m3fn)
    assert np.array_equal(ours, lib.to(torch.float64).numpy())
    assert np.array_equal(quant.e4m3_bits(ours), lib.view(torch.uint8).numpy())


def test_e4m3_ties_subnormals_and_saturation():
    # spacing 1/8 in [1, 2): halfway cases go to the even mantissa
    assert quant.to_e4m3(1.0 + 1 / 16) == 1.0
    assert quant.to_e4m3(1.125 + 1 / 16) == 1.25
    # subnormal spacing 2^-9: half of it rounds to zero (even), 1.5 steps up to 2 steps
    assert quant.to_e4m3(2.0 ** -10) == 0.0
    assert quant.to_e4m3(3 * 2.0 ** -10) == 2 * 2.0 ** -9
    # the largest finite value is 448; beyond it the format saturates
    assert quant.to_e4m3(455.0) == 448.0
    assert quant.to_e4m3(-1e6) == -448.0


def test_quantized_rows_error_bound_and_scale():
    """Each part's largest element is coded +-448, every element is within half
    an e4m3 step of c / s (relative 2^-4, or 2^-10 s in the subnormal range)."""
    rng = np.random.default_rng(3)
    r_k, r_v = 96, 64
    c = rng.standard_normal((50, r_k + r_v)) * rng.uniform(0.01, 10, size=(50, 1))
    codes, sK, sV = quant.quantize_rows(c, r_k, r_v)
    deq = quant.dequantize_rows(codes, sK, sV, r_k)
    for j in range(c.shape[0]):
        for lo, hi, s in ((0, r_k, sK[j]), (r_k, r_k + r_v, sV[j])):
            part = c[j, lo:hi]
            assert np.isclose(float(s), np.max(np.abs(part)) / 448.0, rtol=1e-6)
            assert np.max(np.abs(codes[j, lo:hi])) == 448.0
            err = np.abs(deq[j, lo:hi] - part)
            assert np.all(err <= 2.0 ** -4 * np.abs(part) + float(s) * 2.0 ** -10 + 1e-6 * np.abs(part))
    # the codes are e4m3 numbers
    quant.e4m3_bits(codes)


def test_zero_part_and_row_bytes():
    c = np.zeros((2, 48))
    c[1, 32:] = np.arange(16) - 8.0           # value part only
    codes, sK, sV = quant.quantize_rows(c, 32, 16)
    assert sK[0] == 0 and sV[0] == 0 and sK[1] == 0 and not np.any(codes[0])
    rb = quant.row_bytes(codes, sK, sV)
    assert rb.shape == (2, 64)
    assert rb[1, 48:52].view(np.float32)[0] == sK[1] and rb[1, 52:56].view(np.float32)[0] == sV[1]
    assert not np.any(rb[:, 56:])
    # -8 / (8 / 448) = -448 exactly: code byte of -448 is 0xFE
    assert rb[1, 32] == 0xFE


def test_row_bytes_decode_round_trip_and_library_codes():
    """from_row_bytes inverts row_bytes, and decodes code bytes exactly as
    torch's float8_e4m3fn does."""
    rng = np.random.default_rng(8)
    c = rng.standard_normal((20, 192)) * 3
    codes, sK, sV = quant.quantize_rows(c, 128, 64)
    rows = quant.row_bytes(codes, sK, sV)
    assert np.array_equal(quant.from_row_bytes(rows, 128, 64), quant.dequantize_rows(codes, sK, sV, 128))
    allb = np.arange(256, dtype=np.uint8)
    allb = allb[(allb & 0x7F) != 0x7F]                          # drop the two NaN codes
    lib = torch.from_numpy(allb.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    row = np.zeros((1, 256 + 16), dtype=np.uint8)
    row[0, :allb.size] = allb
    row[0, 256:260] = np.array([1.0], dtype=np.float32).view(np.uint8)
    row[0, 260:264] = np.array([1.0], dtype=np.float32).view(np.uint8)
    vals = quant.from_row_bytes(row, 128, 128)[0, :allb.size]
    assert np.array_equal(vals, lib)
