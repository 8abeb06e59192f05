"""Rotary position operator R_pos at head dimension and at latent dimension.

HLA summary, "Methodology / Latent Reader", eq. 3 applies a rotation R~_i to
the projected query and R~_j to the key latent; "Methodology / Rotary
Embedding Alignment" says the key latent is organised in pairs with
m = r_k / d_h pairs per rotary frequency, so that the rotation commutes with
linear combinations of same-frequency pairs.

Readings (the pages give no formula for R):

* A vector of even length d is a sequence of d/2 pairs (x[2p], x[2p+1]).
* Pair p uses rotary frequency index f(p) = floor(p * d_h / d).  For d = d_h
  this is f(p) = p (textbook interleaved RoPE).  For a latent of rank r with
  integer m = r / d_h it gives m consecutive pairs per frequency
  (frequency-major order).  For m < 1 (for example r = 32, d_h = 64) it picks
  every (1/m)-th frequency.
* theta_f = base ** (-2 f / d_h), angle phi = pos * theta_f, and the pair is
  rotated by +phi: (x, y) -> (x cos phi - y sin phi, x sin phi + y cos phi).
"""

import numpy as np


def pair_frequency(d, d_h):
    """Frequency index f(p) = floor(p * d_h / d) of each of the d/2 pairs."""
    if d % 2:
        raise ValueError("rotary dimension must be even")
    p = np.arange(d // 2, dtype=np.int64)
    return (p * d_h) // d


def angles(pos, d, d_h, base):
    """Angles phi_p = pos * base**(-2 f(p) / d_h) for the d/2 pairs (fp64)."""
    f = pair_frequency(d, d_h).astype(np.float64)
    theta = np.power(float(base), -2.0 * f / float(d_h))
    return float(pos) * theta


def rotate(x, pos, d_h, base):
    """Apply R_pos to the last axis of ``x`` (length d, any even d).

    ``pos`` may be a scalar or an array broadcastable against x[..., 0].
    Returns a new fp64 array.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    f = pair_frequency(d, d_h).astype(np.float64)
    theta = np.power(float(base), -2.0 * f / float(d_h))
    pos = np.asarray(pos, dtype=np.float64)
    phi = pos[..., None] * theta  # [..., d/2]
    c, s = np.cos(phi), np.sin(phi)
    xe, xo = x[..., 0::2], x[..., 1::2]
    out = np.empty(np.broadcast_shapes(x.shape, phi.shape[:-1] + (d,)), dtype=np.float64)
    out[..., 0::2] = xe * c - xo * s
    out[..., 1::2] = xe * s + xo * c
    return out


def matrix(pos, d, d_h, base):
    """Dense d x d matrix of R_pos (used by invariant checks only)."""
    return rotate(np.eye(d), pos, d_h, base).T
