"""Pins for the LLA oracle (per-head, LLA-2D, LLA-D); CPU only."""

import math

import numpy as np
import pytest

from oracle import codec, exact, lla


def _data(seed, N, T, H, d_h, rank=3):
    """Keys/values with a low-rank loop trajectory plus noise."""
    rng = np.random.default_rng(seed)
    P = rng.standard_normal((T, rank))
    u = rng.standard_normal((N, rank, H, d_h))
    k = np.einsum("ts,nshd->nthd", P, u) + 0.05 * rng.standard_normal((N, T, H, d_h))
    u = rng.standard_normal((N, rank, H, d_h))
    v = np.einsum("ts,nshd->nthd", P, u) + 0.05 * rng.standard_normal((N, T, H, d_h))
    q = rng.standard_normal((T, H, d_h))
    return k, v, q


def _ring(k, v, N, W, Wcap):
    _, T, H, d_h = k.shape
    wk = np.full((T, Wcap, H, d_h), np.nan)
    wv = np.full((T, Wcap, H, d_h), np.nan)
    for j in range(max(0, N - 1 - W), N):
        wk[:, j % Wcap] = k[j]
        wv[:, j % Wcap] = v[j]
    return wk, wv


@pytest.mark.parametrize("N,W", [(15, 0), (15, 4), (3, 0)])
def test_perhead_full_rank_reconstruct_is_exact(N, W):
    """Invariant: r = T d_h with the SVD codec reconstructs every per-loop key
    and value, so reconstruct-on-read equals exact per-loop attention
    (keys here are post-rotary, so no rotation is applied)."""
    T, H, d_h = 3, 2, 4
    k, v, q = _data(N + W, N, T, H, d_h)
    EK, EV, UK, UV = codec.lla_perhead(k, v, T * d_h)
    cK, cV = lla.write_perhead(k, v, EK, EV)
    wk, wv = _ring(k, v, N, W, W + 1)
    o = lla.decode_reconstruct(cK, cV, UK, UV, q, wk, wv, 0, N, W)
    ref = exact.attention(q, k, v, 0, d_h, 10000.0, rotary=False)
    np.testing.assert_allclose(o, ref, rtol=1e-10, atol=1e-12)


def test_perhead_low_rank_is_close_but_not_exact():
    """Control, and the pages' premise: a rank-3 trajectory plus small noise
    is captured well by a small rank, but not exactly."""
    N, W, T, H, d_h = 30, 0, 4, 2, 8
    k, v, q = _data(1, N, T, H, d_h, rank=3)
    EK, EV, UK, UV = codec.lla_perhead(k, v, 3 * d_h)
    cK, cV = lla.write_perhead(k, v, EK, EV)
    wk, wv = _ring(k, v, N, W, 1)
    o = lla.decode_reconstruct(cK, cV, UK, UV, q, wk, wv, 0, N, W)
    ref = exact.attention(q, k, v, 0, d_h, 10000.0, rotary=False)
    err = np.linalg.norm(o - ref) / np.linalg.norm(ref)
    assert 1e-6 < err < 0.1


@pytest.mark.parametrize("N,W", [(12, 0), (12, 3)])
def test_folded_full_rank_absorbed_is_exact(N, W):
    """Invariant: LLA-2D at r_K = r_V = T H d_h with the SVD codec, read by
    LLA-D (no reconstruction), equals exact per-loop attention."""
    T, H, d_h = 2, 2, 4
    k, v, q = _data(7 + N + W, N, T, H, d_h)
    r = T * H * d_h
    EK, EV, UK, UV = codec.lla_folded(k, v, r, r)
    lat = lla.write_folded(k, v, EK, EV)
    wk, wv = _ring(k, v, N, W, W + 1)
    o = lla.decode_absorbed(lat, UK, UV, q, wk, wv, 0, N, W, r, r)
    ref = exact.attention(q, k, v, 0, d_h, 10000.0, rotary=False)
    np.testing.assert_allclose(o, ref, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("W", [0, 2])
def test_absorbed_read_equals_reconstruct_on_read(W):
    """Invariant: q^T (U c) = (U^T q)^T c.  Per-head latents embedded
    block-diagonally into one folded latent, read by LLA-D, must equal the
    per-head reconstruct-on-read with arbitrary (non-SVD) decoders."""
    rng = np.random.default_rng(40 + W)
    N, T, H, d_h, r = 11, 3, 2, 4, 5
    cK = rng.standard_normal((H, N, r))
    cV = rng.standard_normal((H, N, r))
    UK = rng.standard_normal((T, H, d_h, r))
    UV = rng.standard_normal((T, H, d_h, r))
    q = rng.standard_normal((T, H, d_h))
    wk = rng.standard_normal((T, W + 1, H, d_h))
    wv = rng.standard_normal((T, W + 1, H, d_h))
    rec = lla.decode_reconstruct(cK, cV, UK, UV, q, wk, wv, 0, N, W)
    lat = np.concatenate([np.concatenate(list(cK), axis=1), np.concatenate(list(cV), axis=1)], axis=1)
    UKf = np.zeros((T, H, d_h, H * r))
    UVf = np.zeros((T, H, d_h, H * r))
    for h in range(H):
        UKf[:, h, :, h * r:(h + 1) * r] = UK[:, h]
        UVf[:, h, :, h * r:(h + 1) * r] = UV[:, h]
    absd = lla.decode_absorbed(lat, UKf, UVf, q, wk, wv, 0, N, W, H * r, H * r)
    np.testing.assert_allclose(absd, rec, rtol=1e-11, atol=1e-12)


def test_writers_are_linear_sums_over_loops_and_heads():
    """Per-head: c_{j,h} = sum_t E_{t,h} k_{j,t,h}; folded sums heads too."""
    rng = np.random.default_rng(5)
    n, T, H, d_h, r = 4, 3, 2, 4, 3
    EK = rng.standard_normal((T, H, r, d_h))
    EV = rng.standard_normal((T, H, r, d_h))
    for t in range(T):
        for h in range(H):
            k = np.zeros((n, T, H, d_h))
            v = np.zeros((n, T, H, d_h))
            k[:, t, h] = rng.standard_normal((n, d_h))
            v[:, t, h] = rng.standard_normal((n, d_h))
            cK, cV = lla.write_perhead(k, v, EK, EV)
            for hh in range(H):
                expect_k = k[:, t, h] @ EK[t, h].T if hh == h else np.zeros((n, r))
                np.testing.assert_allclose(cK[hh], expect_k, atol=1e-14)
            row = lla.write_folded(k, v, EK, EV)
            np.testing.assert_allclose(row[:, :r], k[:, t, h] @ EK[t, h].T, atol=1e-14)
            np.testing.assert_allclose(row[:, r:], v[:, t, h] @ EV[t, h].T, atol=1e-14)


def test_reconstruct_brute_force_tiny():
    """Python-scalar restatement of reconstruct-on-read on a tiny case."""
    rng = np.random.default_rng(6)
    N, W, T, H, d_h, r = 6, 1, 2, 1, 3, 2
    cK = rng.standard_normal((H, N, r))
    cV = rng.standard_normal((H, N, r))
    UK = rng.standard_normal((T, H, d_h, r))
    UV = rng.standard_normal((T, H, d_h, r))
    q = rng.standard_normal((T, H, d_h))
    wk = rng.standard_normal((T, W + 1, H, d_h))
    wv = rng.standard_normal((T, W + 1, H, d_h))
    o = lla.decode_reconstruct(cK, cV, UK, UV, q, wk, wv, 0, N, W)
    i = N - 1
    for t in range(T):
        keys, vals = [], []
        for j in range(N):
            if j < i - W:
                keys.append([sum(UK[t, 0, d, c] * cK[0, j, c] for c in range(r)) for d in range(d_h)])
                vals.append([sum(UV[t, 0, d, c] * cV[0, j, c] for c in range(r)) for d in range(d_h)])
            else:
                keys.append(list(wk[t, j % (W + 1), 0]))
                vals.append(list(wv[t, j % (W + 1), 0]))
        s = [sum(q[t, 0, d] * kk[d] for d in range(d_h)) / math.sqrt(d_h) for kk in keys]
        w = [math.exp(x - max(s)) for x in s]
        expect = [sum(w[j] * vals[j][d] for j in range(N)) / sum(w) for d in range(d_h)]
        np.testing.assert_allclose(o[t, 0], expect, rtol=1e-12)
