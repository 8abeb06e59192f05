"""HLA latent writer (eq. 2) and absorbed latent read (eqs. 3 and 4), fp64.

Source: HLA summary, "Methodology / Latent Writer" (eq. 2),
"Methodology / Latent Reader" (eqs. 3, 4), "Methodology / Rotary Embedding
Alignment".

Shapes for one batch element and one layer (numpy arrays, fp64 math):

* h      [n, T, D]          hidden states entering attention at loops 1..T
* E_main [T-1, r_k+r_v, D]  E_2..E_T of eq. 2
* E_1    [2 r_1, D]         E_1 of eq. 2
* lat    [n_tok, r_k+r_v]   stored rows [R~_j c^K_j | c^V_j]
* A      [nt, H, d_h, r_k]  per loop and head, A_t of eq. 3
* Bm     [nt, H, r_v, d_h]  per loop and head, B_t of eq. 4
* q      [nt, H, d_h]       query of the decoded token at loops t0..t0+nt-1
* win_k, win_v [T, Wcap, H, d_h]  exact K (post-rotary) and V ring;
                            token j sits in slot j mod Wcap

Readings of open points:

* eq. 2 sums loops t = 2..T into c_j; loop 1 is written only into c^(1)_j.
  h_{j,t} is the D-dimensional hidden state at loop t.
* The key part is stored already rotated, R~_j c^K_j: eq. 3 only ever uses
  that product, so scores are unchanged.  The value part is not rotated.
  ``rotate_keys=False`` gives the un-rotated rows (used for LLA-2D).
* The query is the last context token, i = N - 1.  Latent tokens are
  j = 0 .. i-W-1 (eq. 4's j < i - W); exact tokens are j = max(0, i-W) .. i,
  i.e. min(W, i) + 1 tokens, the current token included.
* One softmax over latent and exact scores jointly, both scaled by
  1/sqrt(d_h) (eq. 4 uses a single a_{ij,t}).
* Loop 1 is read with the same formulas, using c^(1), A_1, B_1 and rank r_1.
"""

import numpy as np

from . import rope


def write(h, E_main, E_1, pos0, r_k, r_v, r_1, d_h, base, rotate_keys=True):
    """Latent rows for tokens pos0 .. pos0+n-1 of one sequence (eq. 2), fp64.

    Returns (main [n, r_k+r_v], loop1 [n, 2 r_1]).  Rounding to the storage
    format is a separate step (``oracle.rounding.to_storage``).
    """
    h = np.asarray(h, dtype=np.float64)
    E_main = np.asarray(E_main, dtype=np.float64)
    E_1 = np.asarray(E_1, dtype=np.float64)
    n, T, D = h.shape
    if E_main.shape != (T - 1, r_k + r_v, D) or E_1.shape != (2 * r_1, D):
        raise ValueError("codec shape mismatch")
    c = np.zeros((n, r_k + r_v))
    for t in range(2, T + 1):            # c_j = sum_{t=2}^{T} E_t h_{j,t}
        c += h[:, t - 1, :] @ E_main[t - 2].T
    c1 = h[:, 0, :] @ E_1.T              # c^(1)_j = E_1 h_{j,1}
    if rotate_keys:
        pos = pos0 + np.arange(n)
        c[:, :r_k] = rope.rotate(c[:, :r_k], pos, d_h, base)
        c1[:, :r_1] = rope.rotate(c1[:, :r_1], pos, d_h, base)
    return c, c1


def decode(lat, A, Bm, q, win_k, win_v, t0, N, W, r_k, r_v, d_h, base,
           rotate_query=True, scale=None):
    """Absorbed latent read for one batch element, loops t0 .. t0+nt-1.

    eq. 3:  s^_{ij,t} = (R~_i A_t^T q_{i,t}) . (R~_j c^K_j) / sqrt(d_h)
    eq. 4:  o_{i,t} = B_t^T sum_{j<i-W} a_{ij,t} c^V_j
                      + sum_{i-W<=j<=i} a_{ij,t} v_{j,t}

    ``lat`` holds rows [R~_j c^K_j | c^V_j]; ``win_k`` holds R_j k_{j,t}.
    With ``rotate_query`` the query is the un-rotated q and both R~_i (latent
    space) and R_i (head space, for the exact tokens) are applied here; without
    it q is taken as already rotated (LLA-D with post-rotary codecs).
    Returns o [nt, H, d_h].
    """
    lat = np.asarray(lat, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    Bm = np.asarray(Bm, dtype=np.float64)
    q = np.asarray(q, dtype=np.float64)
    win_k = np.asarray(win_k, dtype=np.float64)
    win_v = np.asarray(win_v, dtype=np.float64)
    nt, H, _ = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d_h)
    i = N - 1
    n_lat = max(0, i - W)
    Wcap = win_k.shape[1]
    exact_j = np.arange(n_lat, i + 1)
    slots = exact_j % Wcap
    cK = lat[:n_lat, :r_k]
    cV = lat[:n_lat, r_k:r_k + r_v]
    out = np.zeros((nt, H, d_h))
    for tt in range(nt):
        t = t0 + tt
        for hh in range(H):
            q_lat = A[tt, hh].T @ q[tt, hh]              # A_t^T q  (R^{r_k})
            if rotate_query:
                q_lat = rope.rotate(q_lat, i, d_h, base)   # R~_i A_t^T q
                q_win = rope.rotate(q[tt, hh], i, d_h, base)  # R_i q
            else:
                q_win = q[tt, hh]
            s_lat = (cK @ q_lat) * scale                   # eq. 3
            k_ex = win_k[t, slots, hh, :]
            v_ex = win_v[t, slots, hh, :]
            s_ex = (k_ex @ q_win) * scale
            s = np.concatenate([s_lat, s_ex])
            m = s.max()
            e = np.exp(s - m)
            a = e / e.sum()                                 # one joint softmax
            a_lat, a_ex = a[:n_lat], a[n_lat:]
            y_lat = a_lat @ cV                             # sum a c^V  (R^{r_v})
            out[tt, hh] = Bm[tt, hh].T @ y_lat + a_ex @ v_ex   # eq. 4
    return out


def decode_positions(lat, A, Bm, q, win_k, win_v, t0, N, W, r_k, r_v, d_h, base,
                     rotate_query=True, scale=None):
    """The read of the last nq positions of a context of N tokens at once.

    Used for a prefill chunk, or for a block of the two-pass procedure's
    parallel second pass (HLA summary, "Methodology / Fine-tuning"), where
    every position's query exists together.  Position i_p = N - nq + p is read
    exactly as a decode at i = i_p: latent tokens j < i_p - W, exact tokens
    i_p - W .. i_p from the ring (eqs. 3-4 with N = i_p + 1).
    q [nq, nt, H, d_h] -> o [nq, nt, H, d_h].
    """
    q = np.asarray(q, dtype=np.float64)
    nq = q.shape[0]
    return np.stack([decode(lat, A, Bm, q[p], win_k, win_v, t0, N - nq + p + 1, W, r_k, r_v, d_h, base,
                            rotate_query=rotate_query, scale=scale) for p in range(nq)])


def decode_reconstruct(lat, A, Bm, q, win_k, win_v, t0, N, W, r_k, r_v, d_h,
                       base, rotate_query=True, scale=None):
    """The same read with keys and values rebuilt in head space first.

    For a query at position i, the stored key latent of token j is turned back
    into the key it stands for relative to i, k^_j = A_t R~_{j-i} c^K_j with
    R~_{j-i} = R~_i^T R~_j, and the value into v^_j = B_t^T c^V_j; then plain
    softmax attention with the un-rotated query.  Used only by the invariant
    "absorbed read equals reconstruct-then-attend".
    """
    lat = np.asarray(lat, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    Bm = np.asarray(Bm, dtype=np.float64)
    q = np.asarray(q, dtype=np.float64)
    nt, H, _ = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d_h)
    i = N - 1
    n_lat = max(0, i - W)
    Wcap = win_k.shape[1]
    exact_j = np.arange(n_lat, i + 1)
    slots = exact_j % Wcap
    out = np.zeros((nt, H, d_h))
    for tt in range(nt):
        t = t0 + tt
        for hh in range(H):
            keys, vals = [], []
            for j in range(n_lat):
                cK_unrot = lat[j, :r_k]
                if rotate_query:
                    # R~_i^T applied to R~_j c^K_j gives R~_{j-i} c^K_j
                    cK_rel = rope.rotate(cK_unrot, -i, d_h, base)
                else:
                    cK_rel = cK_unrot
                keys.append(A[tt, hh] @ cK_rel)
                vals.append(Bm[tt, hh].T @ lat[j, r_k:r_k + r_v])
            for j, sl in zip(exact_j, slots):
                k = np.asarray(win_k[t, sl, hh], dtype=np.float64)
                if rotate_query:
                    k = rope.rotate(k, -i, d_h, base)    # R_i^T R_j k
                keys.append(k)
                vals.append(np.asarray(win_v[t, sl, hh], dtype=np.float64))
            keys = np.array(keys)
            vals = np.array(vals)
            s = (keys @ q[tt, hh]) * scale
            e = np.exp(s - s.max())
            out[tt, hh] = (e / e.sum()) @ vals
    return out
