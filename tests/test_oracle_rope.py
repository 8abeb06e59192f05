"""Pins for the oracle's rotary operator (CPU only)."""

import numpy as np
import pytest

from oracle import rope, codec

BASE = 10000.0


def _complex_rope(x, pos, base):
    """Textbook RoPE (RoFormer): pair p of a head vector is the complex number
    x[2p] + i x[2p+1], multiplied by exp(i * pos * base**(-2p/d))."""
    d = x.shape[-1]
    z = x[..., 0::2] + 1j * x[..., 1::2]
    theta = base ** (-2.0 * np.arange(d // 2) / d)
    z = z * np.exp(1j * pos * theta)
    out = np.empty_like(x)
    out[..., 0::2] = z.real
    out[..., 1::2] = z.imag
    return out


@pytest.mark.parametrize("d_h", [8, 64, 96, 128])
@pytest.mark.parametrize("pos", [0, 1, 7, 255, 4095, 16383])
def test_head_rotation_is_textbook_rope(d_h, pos):
    rng = np.random.default_rng(d_h * 100003 + pos)
    x = rng.standard_normal(d_h)
    np.testing.assert_allclose(rope.rotate(x, pos, d_h, BASE), _complex_rope(x, pos, BASE),
                               rtol=0, atol=1e-12)


def test_rotation_is_orthogonal_and_additive():
    d_h, r = 16, 64
    Ra = rope.matrix(5, r, d_h, BASE)
    Rb = rope.matrix(11, r, d_h, BASE)
    np.testing.assert_allclose(Ra.T @ Ra, np.eye(r), atol=1e-13)
    np.testing.assert_allclose(Ra @ Rb, rope.matrix(16, r, d_h, BASE), atol=1e-12)
    np.testing.assert_allclose(Ra.T, rope.matrix(-5, r, d_h, BASE), atol=1e-13)


@pytest.mark.parametrize("i,j", [(0, 0), (3, 9), (4095, 17), (16383, 16000)])
def test_scores_depend_on_relative_position_only(i, j):
    d_h = 64
    rng = np.random.default_rng(i + 7 * j)
    q, k = rng.standard_normal(d_h), rng.standard_normal(d_h)
    lhs = rope.rotate(q, i, d_h, BASE) @ rope.rotate(k, j, d_h, BASE)
    rhs = q @ rope.rotate(k, j - i, d_h, BASE)
    assert abs(lhs - rhs) < 1e-10 * (1 + abs(lhs))


@pytest.mark.parametrize("r,d_h", [(512, 128), (256, 128), (128, 64), (1152, 128)])
def test_pairs_per_frequency_is_r_over_dh(r, d_h):
    """HLA summary, "Rotary Embedding Alignment": m = r_k / d_h pairs share each
    frequency.  (Only integer m; 1152/128 is not used with rotation.)"""
    f = rope.pair_frequency(r, d_h)
    counts = np.bincount(f, minlength=d_h // 2)
    if r % d_h == 0:
        assert np.all(counts == r // d_h)
        # frequency-major: pairs of one frequency are consecutive
        assert np.all(np.diff(f) >= 0)


def test_latent_frequencies_when_fewer_pairs_than_frequencies():
    # r = 32, d_h = 64: m = 1/2, every other frequency is used
    assert list(rope.pair_frequency(32, 64)) == list(range(0, 32, 2))


def test_head_dimension_map_is_identity():
    assert list(rope.pair_frequency(128, 128)) == list(range(64))


def test_frequency_aligned_codec_commutes_with_rotation():
    """Invariant: A R~_phi = R_phi A for a frequency-aligned A (HLA summary,
    "Rotary Embedding Alignment")."""
    rng = np.random.default_rng(3)
    H, d_h, D, T = 2, 8, 12, 3
    W_K = rng.standard_normal((H, d_h, D))
    W_V = rng.standard_normal((H, d_h, D))
    h = rng.standard_normal((40, T, D))
    r_k = 2 * d_h
    _, A, _ = codec.hla_group(h, W_K, W_V, loops=[2, 3], r_k=r_k, r_v=8)
    for pos in [1, 13, 4095.5, -77]:
        Rt = rope.matrix(pos, r_k, d_h, BASE)
        R = rope.matrix(pos, d_h, d_h, BASE)
        for g in range(2):
            for hh in range(H):
                np.testing.assert_allclose(A[g, hh] @ Rt, R @ A[g, hh], atol=1e-13)


def test_unaligned_codec_does_not_commute():
    """Control for the test above: a dense random A does not commute."""
    rng = np.random.default_rng(4)
    A = rng.standard_normal((8, 16))
    Rt = rope.matrix(3, 16, 8, BASE)
    R = rope.matrix(3, 8, 8, BASE)
    assert np.abs(A @ Rt - R @ A).max() > 1e-3
