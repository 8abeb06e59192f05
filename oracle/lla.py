"""LLA per-head and LLA-2D codecs: writers, reconstruct-on-read, absorbed read.

Source: LLA abstract ("Looped Latent Attention: Cross-Loop Key-Value
Compression For Looped Transformers", Abstract): a post-training cache codec
that stores compact K and V latents and reconstructs loop-specific vectors only
when attention reads them; the -2D variant folds heads into one latent; the
absorbed variant LLA-D reads latents without reconstruction.

The abstract gives no formulas.  Readings (the plainest linear codec that fits
"initialized from the SVD of teacher activations"):

* Per-head encoder: c^K_{j,h} = sum_t E^K_{t,h} k_{j,t,h}, E^K_{t,h} in
  R^{r x d_h}; same for V.  Decoder: k^_{j,t,h} = U^K_{t,h} c^K_{j,h},
  U^K_{t,h} in R^{d_h x r}; same for V.
* LLA-2D encoder: c^K_j = sum_{t,h} E^K_{t,h} k_{j,t,h} in R^{r_K}, and the
  decoder U^K_{t,h} in R^{d_h x r_K} maps the shared latent to each head.
* The codecs act on post-rotary keys ("full-RoPE codecs"), so no rotation is
  applied on read and the query is the rotated query.
* Decoding at i = N-1: tokens j < i-W are read from latents, tokens
  max(0,i-W) .. i from the exact ring.  W = 0 means only the current token
  (whose latent cannot exist until all its loops are done) is exact.
* One joint softmax, scale 1/sqrt(d_h).

Shapes, one batch element: k, v [n, T, H, d_h]; cK, cV [H, n_tok, r];
folded latent rows [n_tok, r_K + r_V] = [c^K | c^V]; q [nt, H, d_h];
U^K, U^V [nt, H, d_h, r]; ring [T, Wcap, H, d_h].
"""

import numpy as np


def write_perhead(k, v, EK, EV):
    """Per-head latents of n tokens: returns (cK [H, n, r], cV [H, n, r])."""
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    EK = np.asarray(EK, dtype=np.float64)
    EV = np.asarray(EV, dtype=np.float64)
    n, T, H, d_h = k.shape
    r = EK.shape[2]
    cK = np.zeros((H, n, r))
    cV = np.zeros((H, n, r))
    for h in range(H):
        for t in range(T):                 # c_{j,h} = sum_t E_{t,h} k_{j,t,h}
            cK[h] += k[:, t, h, :] @ EK[t, h].T
            cV[h] += v[:, t, h, :] @ EV[t, h].T
    return cK, cV


def write_folded(k, v, EK, EV):
    """LLA-2D rows [n, r_K + r_V] = [c^K | c^V], heads folded into one latent."""
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    EK = np.asarray(EK, dtype=np.float64)
    EV = np.asarray(EV, dtype=np.float64)
    n, T, H, d_h = k.shape
    rK, rV = EK.shape[2], EV.shape[2]
    cK = np.zeros((n, rK))
    cV = np.zeros((n, rV))
    for t in range(T):                     # c_j = sum_{t,h} E_{t,h} k_{j,t,h}
        for h in range(H):
            cK += k[:, t, h, :] @ EK[t, h].T
            cV += v[:, t, h, :] @ EV[t, h].T
    return np.concatenate([cK, cV], axis=1)


def _exact_tokens(N, W, Wcap):
    i = N - 1
    n_lat = max(0, i - W)
    j = np.arange(n_lat, i + 1)
    return n_lat, j, j % Wcap


def decode_reconstruct(cK, cV, UK, UV, q, win_k, win_v, t0, N, W, scale=None):
    """LLA per-head reconstruct-on-read for one batch element.

    For each loop t and head h, every latent token's key and value are rebuilt,
    k^_j = U^K_{t,h} c^K_{j,h}, v^_j = U^V_{t,h} c^V_{j,h}, then attention runs
    over rebuilt and exact tokens with one softmax.  Returns o [nt, H, d_h].
    """
    cK = np.asarray(cK, dtype=np.float64)
    cV = np.asarray(cV, dtype=np.float64)
    UK = np.asarray(UK, dtype=np.float64)
    UV = np.asarray(UV, dtype=np.float64)
    q = np.asarray(q, dtype=np.float64)
    nt, H, d_h = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d_h)
    n_lat, _, slots = _exact_tokens(N, W, win_k.shape[1])
    out = np.zeros((nt, H, d_h))
    for tt in range(nt):
        t = t0 + tt
        for h in range(H):
            k_hat = cK[h, :n_lat] @ UK[tt, h].T         # rows U^K c^K_j
            v_hat = cV[h, :n_lat] @ UV[tt, h].T         # rows U^V c^V_j
            keys = np.concatenate([k_hat, np.asarray(win_k[t, slots, h], dtype=np.float64)])
            vals = np.concatenate([v_hat, np.asarray(win_v[t, slots, h], dtype=np.float64)])
            s = (keys @ q[tt, h]) * scale
            e = np.exp(s - s.max())
            out[tt, h] = (e / e.sum()) @ vals
    return out


def decode_absorbed(lat, UK, UV, q, win_k, win_v, t0, N, W, r_K, r_V, scale=None):
    """LLA-D: read a (folded) latent without reconstruction.

    q~ = U^K_{t,h}^T q; s_j = q~ . c^K_j * scale; y~ = sum_j a_j c^V_j;
    o = U^V_{t,h} y~ + sum_exact a_j v_j.  Returns o [nt, H, d_h].
    """
    lat = np.asarray(lat, dtype=np.float64)
    UK = np.asarray(UK, dtype=np.float64)
    UV = np.asarray(UV, dtype=np.float64)
    q = np.asarray(q, dtype=np.float64)
    nt, H, d_h = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d_h)
    n_lat, _, slots = _exact_tokens(N, W, win_k.shape[1])
    cK = lat[:n_lat, :r_K]
    cV = lat[:n_lat, r_K:r_K + r_V]
    out = np.zeros((nt, H, d_h))
    for tt in range(nt):
        t = t0 + tt
        for h in range(H):
            q_lat = UK[tt, h].T @ q[tt, h]
            s_lat = (cK @ q_lat) * scale
            k_ex = np.asarray(win_k[t, slots, h], dtype=np.float64)
            v_ex = np.asarray(win_v[t, slots, h], dtype=np.float64)
            s = np.concatenate([s_lat, (k_ex @ q[tt, h]) * scale])
            e = np.exp(s - s.max())
            a = e / e.sum()
            out[tt, h] = UV[tt, h] @ (a[:n_lat] @ cV) + a[n_lat:] @ v_ex
    return out
