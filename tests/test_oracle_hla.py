"""Pins for the HLA oracle (writer eq. 2, absorbed read eqs. 3-4); CPU only."""

import cmath
import json
import math
import os

import numpy as np
import pytest
from scipy.special import softmax

from oracle import codec, exact, hla, lla, rope

BASE = 10000.0
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _ring(k_rot, v, N, W, Wcap):
    """Exact-token ring [T, Wcap, H, d_h]: token j in slot j mod Wcap."""
    _, T, H, d_h = k_rot.shape
    wk = np.full((T, Wcap, H, d_h), np.nan)
    wv = np.full((T, Wcap, H, d_h), np.nan)
    i = N - 1
    for j in range(max(0, i - W), i + 1):
        wk[:, j % Wcap] = k_rot[j]
        wv[:, j % Wcap] = v[j]
    return wk, wv


def _teacher(seed, N, T, H, d_h, D):
    rng = np.random.default_rng(seed)
    W_K = rng.standard_normal((H, d_h, D)) / math.sqrt(D)
    W_V = rng.standard_normal((H, d_h, D)) / math.sqrt(D)
    h = rng.standard_normal((N, T, D))
    k = np.einsum("hdD,ntD->nthd", W_K, h)
    v = np.einsum("hdD,ntD->nthd", W_V, h)
    q = rng.standard_normal((T, H, d_h))
    return W_K, W_V, h, k, v, q


@pytest.mark.parametrize("N,W", [(20, 4), (33, 0), (9, 3)])
def test_full_rank_latent_attention_is_exact(N, W):
    """Invariant: with full rank and SVD codecs, HLA equals exact per-loop
    rotary attention for every loop (HLA summary, eqs. 2-4 and "Rotary
    Embedding Alignment")."""
    T, H, d_h, D = 3, 2, 8, 12
    W_K, W_V, h, k, v, q = _teacher(11 + N, N, T, H, d_h, D)
    r_k = r_v = (T - 1) * H * d_h
    r_1 = H * d_h
    E, A, Bm = codec.hla_group(h, W_K, W_V, loops=list(range(2, T + 1)), r_k=r_k, r_v=r_v)
    E1, A1, B1 = codec.hla_group(h, W_K, W_V, loops=[1], r_k=r_1, r_v=r_1)
    lat, lat1 = hla.write(h, E, E1[0], 0, r_k, r_v, r_1, d_h, BASE)
    k_rot = rope.rotate(k, np.arange(N)[:, None, None], d_h, BASE)
    wk, wv = _ring(k_rot, v, N, W, W + 1)
    o_main = hla.decode(lat, A, Bm, q[1:], wk, wv, 1, N, W, r_k, r_v, d_h, BASE)
    o_one = hla.decode(lat1, A1, B1, q[:1], wk, wv, 0, N, W, r_1, r_1, d_h, BASE)
    ref = exact.attention(q, k, v, 0, d_h, BASE)
    np.testing.assert_allclose(o_main, ref[1:], rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(o_one, ref[:1], rtol=1e-9, atol=1e-11)


def test_reduced_rank_is_not_exact():
    """Control: the same check fails when the rank is cut."""
    N, W, T, H, d_h, D = 20, 4, 3, 2, 8, 12
    W_K, W_V, h, k, v, q = _teacher(5, N, T, H, d_h, D)
    r_k = r_v = d_h                        # m = 1 pair per frequency, not 4
    E, A, Bm = codec.hla_group(h, W_K, W_V, loops=[2, 3], r_k=r_k, r_v=r_v)
    E1, _, _ = codec.hla_group(h, W_K, W_V, loops=[1], r_k=d_h, r_v=d_h)
    lat, _ = hla.write(h, E, E1[0], 0, r_k, r_v, d_h, d_h, BASE)
    k_rot = rope.rotate(k, np.arange(N)[:, None, None], d_h, BASE)
    wk, wv = _ring(k_rot, v, N, W, W + 1)
    o = hla.decode(lat, A, Bm, q[1:], wk, wv, 1, N, W, r_k, r_v, d_h, BASE)
    ref = exact.attention(q, k, v, 0, d_h, BASE)[1:]
    assert np.abs(o - ref).max() > 1e-4


@pytest.mark.parametrize("rotate_query", [True, False])
def test_absorbed_equals_reconstruct_then_attend(rotate_query):
    """Invariant: q^T (U c) = (U^T q)^T c, for arbitrary (unaligned) A and B."""
    rng = np.random.default_rng(21)
    N, W, T, H, d_h, r_k, r_v = 17, 5, 4, 3, 8, 24, 12
    lat = rng.standard_normal((N, r_k + r_v))
    A = rng.standard_normal((T - 1, H, d_h, r_k)) / 3
    Bm = rng.standard_normal((T - 1, H, r_v, d_h)) / 3
    q = rng.standard_normal((T - 1, H, d_h))
    wk = rng.standard_normal((T, W + 2, H, d_h))
    wv = rng.standard_normal((T, W + 2, H, d_h))
    args = (lat, A, Bm, q, wk, wv, 1, N, W, r_k, r_v, d_h, BASE)
    a = hla.decode(*args, rotate_query=rotate_query)
    b = hla.decode_reconstruct(*args, rotate_query=rotate_query)
    np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("N,W", [(8, 7), (8, 30), (1, 0), (1, 5)])
def test_window_covering_context_is_exact(N, W):
    """Invariant: W >= i leaves no latent token; HLA is exact attention on the
    window (eq. 4 with an empty first sum)."""
    T, H, d_h = 3, 2, 8
    rng = np.random.default_rng(N * 31 + W)
    k = rng.standard_normal((N, T, H, d_h))
    v = rng.standard_normal((N, T, H, d_h))
    q = rng.standard_normal((T, H, d_h))
    k_rot = rope.rotate(k, np.arange(N)[:, None, None], d_h, BASE)
    wk, wv = _ring(k_rot, v, N, W, W + 1)
    lat = np.full((max(N, 1), 64), np.nan)        # must never be read
    A = rng.standard_normal((T, H, d_h, 32))
    Bm = rng.standard_normal((T, H, 32, d_h))
    o = hla.decode(lat, A, Bm, q, wk, wv, 0, N, W, 32, 32, d_h, BASE)
    np.testing.assert_allclose(o, exact.attention(q, k, v, 0, d_h, BASE), rtol=1e-11, atol=1e-12)


def test_single_token_returns_its_value():
    """Closed form: N = 1 gives o = v_0 whatever q is."""
    rng = np.random.default_rng(2)
    T, H, d_h = 4, 2, 8
    wk = rng.standard_normal((T, 3, H, d_h))
    wv = rng.standard_normal((T, 3, H, d_h))
    q = rng.standard_normal((T, H, d_h)) * 50
    lat = np.zeros((1, 32))
    A = rng.standard_normal((T, H, d_h, 16))
    Bm = rng.standard_normal((T, H, 16, d_h))
    o = hla.decode(lat, A, Bm, q, wk, wv, 0, 1, 2, 16, 16, d_h, BASE)
    np.testing.assert_allclose(o, wv[:, 0], rtol=0, atol=1e-14)


def test_zero_query_gives_mean_of_values():
    """Closed form: all scores equal -> a_j = 1/(i+1);
    o = (B^T sum_lat c^V + sum_exact v) / (i + 1)."""
    rng = np.random.default_rng(8)
    N, W, T, H, d_h, r_k, r_v = 12, 3, 2, 2, 8, 16, 10
    lat = rng.standard_normal((N, r_k + r_v))
    A = rng.standard_normal((T, H, d_h, r_k))
    Bm = rng.standard_normal((T, H, r_v, d_h))
    wk = rng.standard_normal((T, W + 1, H, d_h))
    wv = rng.standard_normal((T, W + 1, H, d_h))
    q = np.zeros((T, H, d_h))
    o = hla.decode(lat, A, Bm, q, wk, wv, 0, N, W, r_k, r_v, d_h, BASE)
    n_lat = N - 1 - W
    slots = [j % (W + 1) for j in range(n_lat, N)]
    for t in range(T):
        for h in range(H):
            expect = (Bm[t, h].T @ lat[:n_lat, r_k:].sum(0) + wv[t, slots, h].sum(0)) / N
            np.testing.assert_allclose(o[t, h], expect, rtol=1e-12, atol=1e-13)


def _textbook(q, keys, vals, i, d_h, base):
    """Single-head RoPE attention with complex rotation and scipy's softmax."""
    def rot(x, pos):
        z = x[0::2] + 1j * x[1::2]
        z = z * np.exp(1j * pos * base ** (-2.0 * np.arange(d_h // 2) / d_h))
        return np.stack([z.real, z.imag], -1).reshape(-1)
    s = np.array([rot(q, i) @ rot(keys[j], j) for j in range(len(keys))]) / math.sqrt(d_h)
    return softmax(s) @ vals


@pytest.mark.parametrize("N,W", [(16, 4), (16, 0), (40, 10)])
def test_identity_codec_single_head_is_textbook_rope_attention(N, W):
    """Special case: one head, r_1 = d_h, E_1 = [W_K; W_V], A_1 = B_1 = I.
    The loop-1 latent is then the exact key/value and eqs. 3-4 reduce to
    single-head rotary attention."""
    rng = np.random.default_rng(N + W)
    d_h, D, T = 16, 16, 2
    W_K = rng.standard_normal((d_h, D)) / 4
    W_V = rng.standard_normal((d_h, D)) / 4
    h = rng.standard_normal((N, T, D))
    E1 = np.concatenate([W_K, W_V])
    E_main = rng.standard_normal((T - 1, 2 * d_h, D))
    _, lat1 = hla.write(h, E_main, E1, 0, d_h, d_h, d_h, d_h, BASE)
    keys = h[:, 0] @ W_K.T
    vals = h[:, 0] @ W_V.T
    wk, wv = _ring(rope.rotate(keys, np.arange(N), d_h, BASE)[:, None, None, :],
                   vals[:, None, None, :], N, W, W + 1)
    A1 = np.eye(d_h)[None, None]
    q = rng.standard_normal((1, 1, d_h))
    o = hla.decode(lat1, A1, A1, q, wk, wv, 0, N, W, d_h, d_h, d_h, BASE)
    np.testing.assert_allclose(o[0, 0], _textbook(q[0, 0], keys, vals, N - 1, d_h, BASE),
                               rtol=1e-11, atol=1e-12)


def _brute(lat, A, Bm, q, wk, wv, t0, N, W, r_k, r_v, d_h, base):
    """eqs. 3-4 with Python scalars: every sum and rotation spelled out."""
    nt, H = len(q), len(q[0])
    i = N - 1
    m = r_k // d_h if r_k >= d_h else None
    Wcap = len(wk[0])

    def rot_latent(x, pos):
        x = list(x)
        out = [0.0] * r_k
        for p in range(r_k // 2):
            f = p // m if m else p * (d_h // r_k)     # m pairs per frequency
            th = base ** (-2.0 * f / d_h)
            z = complex(x[2 * p], x[2 * p + 1]) * cmath.exp(1j * pos * th)
            out[2 * p], out[2 * p + 1] = z.real, z.imag
        return out

    def rot_head(x, pos):
        out = [0.0] * d_h
        for f in range(d_h // 2):
            z = complex(x[2 * f], x[2 * f + 1]) * cmath.exp(1j * pos * base ** (-2.0 * f / d_h))
            out[2 * f], out[2 * f + 1] = z.real, z.imag
        return out

    res = np.zeros((nt, H, d_h))
    for tt in range(nt):
        for h in range(H):
            qt = [sum(A[tt][h][d][c] * q[tt][h][d] for d in range(d_h)) for c in range(r_k)]
            qt = rot_latent(qt, i)
            qw = rot_head(q[tt][h], i)
            scores, kinds = [], []
            for j in range(N):
                if j < i - W:
                    scores.append(sum(qt[c] * lat[j][c] for c in range(r_k)) / math.sqrt(d_h))
                    kinds.append(("lat", j))
                else:
                    kk = wk[t0 + tt][j % Wcap][h]
                    scores.append(sum(qw[d] * kk[d] for d in range(d_h)) / math.sqrt(d_h))
                    kinds.append(("win", j))
            mx = max(scores)
            w = [math.exp(s - mx) for s in scores]
            tot = sum(w)
            ylat = [0.0] * r_v
            out = [0.0] * d_h
            for wt, (kind, j) in zip(w, kinds):
                if kind == "lat":
                    for c in range(r_v):
                        ylat[c] += wt / tot * lat[j][r_k + c]
                else:
                    for d in range(d_h):
                        out[d] += wt / tot * wv[t0 + tt][j % Wcap][h][d]
            for d in range(d_h):
                out[d] += sum(Bm[tt][h][c][d] * ylat[c] for c in range(r_v))
            res[tt, h] = out
    return res


@pytest.mark.parametrize("T,N,W,r_k", [(2, 6, 2, 16), (3, 12, 3, 8), (4, 9, 0, 16), (4, 5, 8, 8)])
def test_brute_force_agrees(T, N, W, r_k):
    rng = np.random.default_rng(T * 100 + N)
    H, d_h, r_v = 2, 8, 6
    lat = rng.standard_normal((N, r_k + r_v))
    A = rng.standard_normal((T - 1, H, d_h, r_k)) / 2
    Bm = rng.standard_normal((T - 1, H, r_v, d_h))
    q = rng.standard_normal((T - 1, H, d_h))
    Wcap = W + 2
    wk = rng.standard_normal((T, Wcap, H, d_h))
    wv = rng.standard_normal((T, Wcap, H, d_h))
    args = (lat, A, Bm, q, wk, wv, 1, N, W, r_k, r_v, d_h, BASE)
    np.testing.assert_allclose(hla.decode(*args), _brute(*args), rtol=1e-11, atol=1e-12)


def test_writer_sum_ranges_and_loop_index():
    """eq. 2: loop 1 feeds only c^(1) through E_1; loop t >= 2 feeds only c
    through E_t (checked loop by loop, with rotation off)."""
    rng = np.random.default_rng(9)
    n, T, D, r_k, r_v, r_1, d_h = 3, 4, 6, 8, 4, 4, 4
    E = rng.standard_normal((T - 1, r_k + r_v, D))
    E1 = rng.standard_normal((2 * r_1, D))
    for t in range(1, T + 1):
        h = np.zeros((n, T, D))
        h[:, t - 1] = rng.standard_normal((n, D))
        c, c1 = hla.write(h, E, E1, 0, r_k, r_v, r_1, d_h, BASE, rotate_keys=False)
        if t == 1:
            np.testing.assert_array_equal(c, 0)
            np.testing.assert_allclose(c1, h[:, 0] @ E1.T, rtol=1e-14)
        else:
            np.testing.assert_array_equal(c1, 0)
            np.testing.assert_allclose(c, h[:, t - 1] @ E[t - 2].T, rtol=1e-14)


def test_writer_rotates_key_part_only_at_token_position():
    rng = np.random.default_rng(10)
    n, T, D, r_k, r_v, r_1, d_h, pos0 = 4, 2, 6, 8, 4, 4, 4, 100
    h = rng.standard_normal((n, T, D))
    E = rng.standard_normal((T - 1, r_k + r_v, D))
    E1 = rng.standard_normal((2 * r_1, D))
    c0, c10 = hla.write(h, E, E1, pos0, r_k, r_v, r_1, d_h, BASE, rotate_keys=False)
    c, c1 = hla.write(h, E, E1, pos0, r_k, r_v, r_1, d_h, BASE)
    np.testing.assert_array_equal(c[:, r_k:], c0[:, r_k:])
    np.testing.assert_array_equal(c1[:, r_1:], c10[:, r_1:])
    for j in range(n):
        np.testing.assert_allclose(c[j, :r_k], rope.matrix(pos0 + j, r_k, d_h, BASE) @ c0[j, :r_k],
                                   atol=1e-12)


def test_printed_cache_sizes():
    """The HLA summary prints 768 KiB -> 72 KiB per token (10.7x) for
    Ouro-1.4B; the writer's row layout (r_k + r_v + 2 r_1 numbers per layer,
    eq. 2's storage line) with the Ouro-shaped ranks must reproduce them."""
    with open(os.path.join(GOLDEN, "printed_sizes.json")) as fh:
        g = json.load(fh)
    L, T, H, d_h, r_k, r_v, r_1 = 24, 4, 16, 128, 512, 512, 256
    full = L * 2 * T * H * d_h * 2
    lat = L * (r_k + r_v + 2 * r_1) * 2
    assert full == g["ouro_full_cache_kib_per_token"] * 1024
    assert lat == g["ouro_hla_cache_kib_per_token"] * 1024
    assert round(full / lat, 1) == g["ouro_hla_reduction"]
    # LLA abstract: 32x on Huginn-3.5B.  Count the numbers one token occupies
    # through the oracle's own per-head writer at the Huginn-like shapes (32
    # loops, 55 heads, d_h = 96, rank 96): its per-loop K and V in, the
    # per-head K and V latent rows out.
    T_h, H_h, dh_h, r_h = 32, 55, 96, 96
    rng = np.random.default_rng(5)
    k = rng.standard_normal((1, T_h, H_h, dh_h))
    v = rng.standard_normal((1, T_h, H_h, dh_h))
    EK = rng.standard_normal((T_h, H_h, r_h, dh_h))
    EV = rng.standard_normal((T_h, H_h, r_h, dh_h))
    cK, cV = lla.write_perhead(k, v, EK, EV)
    assert cK.shape == (H_h, 1, r_h) and cV.shape == (H_h, 1, r_h)
    assert (k.size + v.size) / (cK.size + cV.size) == g["huginn_lla_compression"]


def test_several_positions_with_full_window_are_causal_exact_attention():
    """decode_positions with W >= N: every position p reads only the exact ring,
    so each must equal textbook causal rotary attention over tokens 0..i_p with
    i_p = N - nq + p (pins the positions, the ring slots j mod Wcap and the
    per-position rotation against an independent formula)."""
    rng = np.random.default_rng(21)
    N, nq, T, H, d_h, W = 12, 4, 3, 2, 8, 20
    Wcap = 13
    k = rng.standard_normal((N, T, H, d_h))
    v = rng.standard_normal((N, T, H, d_h))
    q = rng.standard_normal((nq, 2, H, d_h))
    ring_k = np.zeros((T, Wcap, H, d_h))
    ring_v = np.zeros((T, Wcap, H, d_h))
    for j in range(N):
        ring_k[:, j % Wcap] = rope.rotate(k[j], j, d_h, BASE)
        ring_v[:, j % Wcap] = v[j]
    A = rng.standard_normal((2, H, d_h, 16))
    Bm = rng.standard_normal((2, H, 16, d_h))
    lat = rng.standard_normal((N, 32))
    got = hla.decode_positions(lat, A, Bm, q, ring_k, ring_v, 1, N, W, 16, 16, d_h, BASE)
    for p in range(nq):
        i = N - nq + p
        ref = exact.attention(q[p], k[:i + 1], v[:i + 1], 1, d_h, BASE)
        np.testing.assert_allclose(got[p], ref, atol=1e-12)
