"""Exact per-loop rotary attention: what the teacher's per-loop cache computes.

HLA summary, "Introduction / Key Problem": in a looped model each loop attends
to its own keys and values, so the cache holds T per-loop K/V sets.  This is
the reference the latent codecs approximate, and the one the invariants
compare against.

Shapes, one batch element: q [nt, H, d_h] (un-rotated), k, v [N, T, H, d_h]
(un-rotated keys), query at i = N-1 attending to every j <= i.
"""

import numpy as np

from . import rope


def attention(q, k, v, t0, d_h, base, rotary=True, scale=None):
    """o_{t,h} = sum_{j<=i} softmax_j((R_i q).(R_j k_{j,t,h}) * scale) v_{j,t,h}."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    nt, H, _ = q.shape
    N = k.shape[0]
    i = N - 1
    if scale is None:
        scale = 1.0 / np.sqrt(d_h)
    out = np.zeros((nt, H, d_h))
    pos = np.arange(N)
    for tt in range(nt):
        t = t0 + tt
        for h in range(H):
            keys = k[:, t, h, :]
            qq = q[tt, h]
            if rotary:
                keys = rope.rotate(keys, pos, d_h, base)
                qq = rope.rotate(qq, i, d_h, base)
            s = (keys @ qq) * scale
            e = np.exp(s - s.max())
            out[tt, h] = (e / e.sum()) @ v[:, t, h, :]
    return out
