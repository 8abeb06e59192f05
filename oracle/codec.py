"""SVD codecs for the oracle's exactness invariants.

The pages initialise every codec from an SVD/PCA of teacher keys and values
(LLA abstract: "initialized from the SVD of teacher activations"; HLA summary,
"Training Procedure": E_t, A_t, B_t from PCA of keys/values).  Codec fitting is
offline and not on the decode path; it lives here only so that tests can state
"with full rank and SVD codec matrices, latent attention equals exact
per-loop attention".

HLA keys need a frequency-aligned codec (HLA summary, "Rotary Embedding
Alignment"): for rotary frequency f, the pair (k[2f], k[2f+1]) of every loop
and head forms two samples of a (loops x heads)-vector; its SVD basis u_s
(s = 1..m) gives latent pair p = f*m + s, and A_{t,h} maps latent pair p back
into head pair f with the real weight u_s[t,h] on both components.  Every
block of A is then a multiple of the 2x2 identity, which commutes with the
rotation by the shared angle.

Conventions: W_K, W_V [H, d_h, D] project a hidden state to the head keys and
values of every loop (weights are tied across loops).
"""

import numpy as np


def _basis(samples, rank):
    """First ``rank`` right singular vectors of ``samples`` (rows = samples)."""
    _, _, vt = np.linalg.svd(np.asarray(samples, dtype=np.float64), full_matrices=True)
    if rank > vt.shape[0]:
        raise ValueError("rank exceeds the sample dimension")
    return vt[:rank]


def hla_group(h, W_K, W_V, loops, r_k, r_v):
    """Codec for one loop group (e.g. loops 2..T, or loop 1 alone).

    h [n, T, D] calibration hidden states; ``loops`` are 1-based loop indices.
    Returns (E [len(loops), r_k + r_v, D], A [len(loops), H, d_h, r_k],
    Bm [len(loops), H, r_v, d_h]).  Requires r_k to be a multiple of d_h
    (integer m = r_k / d_h pairs per frequency).
    """
    h = np.asarray(h, dtype=np.float64)
    W_K = np.asarray(W_K, dtype=np.float64)
    W_V = np.asarray(W_V, dtype=np.float64)
    H, d_h, D = W_K.shape
    G = len(loops)
    if r_k % d_h:
        raise ValueError("r_k must be a multiple of d_h for this codec")
    m = r_k // d_h
    hl = h[:, [t - 1 for t in loops], :]                  # [n, G, D]
    k = np.einsum("hdD,ngD->nghd", W_K, hl)                # [n, G, H, d_h]
    v = np.einsum("hdD,ngD->nghd", W_V, hl)
    n = h.shape[0]
    E = np.zeros((G, r_k + r_v, D))
    A = np.zeros((G, H, d_h, r_k))
    Bm = np.zeros((G, H, r_v, d_h))
    for f in range(d_h // 2):
        x = k[:, :, :, 2 * f].reshape(n, G * H)
        y = k[:, :, :, 2 * f + 1].reshape(n, G * H)
        u = _basis(np.concatenate([x, y], axis=0), m).reshape(m, G, H)
        for s in range(m):
            p = f * m + s
            for g in range(G):
                for hh in range(H):
                    w = u[s, g, hh]
                    E[g, 2 * p] += w * W_K[hh, 2 * f]
                    E[g, 2 * p + 1] += w * W_K[hh, 2 * f + 1]
                    A[g, hh, 2 * f, 2 * p] = w
                    A[g, hh, 2 * f + 1, 2 * p + 1] = w
    uv = _basis(v.reshape(n, G * H * d_h), r_v).reshape(r_v, G, H, d_h)
    for g in range(G):
        E[g, r_k:] = np.einsum("shd,hdD->sD", uv[:, g], W_V)
        Bm[g] = np.transpose(uv[:, g], (1, 0, 2))          # [H, r_v, d_h]
    return E, A, Bm


def lla_perhead(k, v, r):
    """Per-head codec from per-loop keys/values k, v [n, T, H, d_h].

    Returns (EK, EV [T, H, r, d_h], UK, UV [T, H, d_h, r]).
    """
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n, T, H, d_h = k.shape
    EK = np.zeros((T, H, r, d_h))
    EV = np.zeros((T, H, r, d_h))
    for h in range(H):
        bk = _basis(k[:, :, h, :].reshape(n, T * d_h), r).reshape(r, T, d_h)
        bv = _basis(v[:, :, h, :].reshape(n, T * d_h), r).reshape(r, T, d_h)
        for t in range(T):
            EK[t, h] = bk[:, t, :]
            EV[t, h] = bv[:, t, :]
    UK = np.transpose(EK, (0, 1, 3, 2)).copy()
    UV = np.transpose(EV, (0, 1, 3, 2)).copy()
    return EK, EV, UK, UV


def lla_folded(k, v, r_K, r_V):
    """LLA-2D codec: one latent for all loops and heads.

    Returns (EK [T, H, r_K, d_h], EV [T, H, r_V, d_h], UK [T, H, d_h, r_K],
    UV [T, H, d_h, r_V]).
    """
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n, T, H, d_h = k.shape
    bk = _basis(k.reshape(n, T * H * d_h), r_K).reshape(r_K, T, H, d_h)
    bv = _basis(v.reshape(n, T * H * d_h), r_V).reshape(r_V, T, H, d_h)
    EK = np.transpose(bk, (1, 2, 0, 3)).copy()              # [T, H, r_K, d_h]
    EV = np.transpose(bv, (1, 2, 0, 3)).copy()
    UK = np.transpose(bk, (1, 2, 3, 0)).copy()              # [T, H, d_h, r_K]
    UV = np.transpose(bv, (1, 2, 3, 0)).copy()
    return EK, EV, UK, UV
