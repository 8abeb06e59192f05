"""Seeded generators: configuration shapes, activations, codecs, queries, rings."""

import math
from dataclasses import dataclass

import numpy as np
import torch

TRAJ_RANK = 8        # rank of the per-loop trajectory of the synthetic activations
NOISE = 0.05         # std of the noise added to each loop's activation


@dataclass(frozen=True)
class ConfigShape:
    name: str
    kind: str            # 'hla' | 'lla' (per-head reconstruct) | 'lla2d' (folded, absorbed)
    B: int
    L: int
    T: int
    H: int
    d_h: int
    D: int
    N: int
    W: int
    r_k: int
    r_v: int
    r_1: int
    lat_dtype: str       # 'bf16' | 'f32' | 'fp8' (e4m3 rows with per-token scales)
    base: float = 10000.0


CONFIGS = {
    # tiny fp32 HLA layer that the oracle finishes in seconds
    "tiny_hla": ConfigShape("tiny_hla", "hla", B=1, L=1, T=4, H=2, d_h=64, D=128, N=256, W=16,
                            r_k=128, r_v=128, r_1=32, lat_dtype="f32"),
    # Ouro-1.4B-shaped HLA decode, all 24 layers, 4k context, batch 32
    "ouro_hla_4k": ConfigShape("ouro_hla_4k", "hla", B=32, L=24, T=4, H=16, d_h=128, D=2048,
                               N=4096, W=128, r_k=512, r_v=512, r_1=256, lat_dtype="bf16"),
    # Huginn-3.5B-like LLA per-head reconstruct-on-read, 32 loops, rank 96
    "huginn_lla_4k": ConfigShape("huginn_lla_4k", "lla", B=16, L=1, T=32, H=55, d_h=96, D=0,
                                 N=4096, W=0, r_k=96, r_v=96, r_1=0, lat_dtype="bf16"),
    # the same under the served semantics: an exact window of the last 64 tokens
    # (plus the current one), latents for older tokens only
    "huginn_lla_4k_w64": ConfigShape("huginn_lla_4k_w64", "lla", B=16, L=1, T=32, H=55, d_h=96, D=0,
                                     N=4096, W=64, r_k=96, r_v=96, r_1=0, lat_dtype="bf16"),
    # capacity regime: Ouro-shaped LLA-2D, batch 768, absorbed read, no window
    "ouro_lla2d_768": ConfigShape("ouro_lla2d_768", "lla2d", B=768, L=24, T=4, H=16, d_h=128, D=0,
                                  N=4096, W=0, r_k=576, r_v=576, r_1=0, lat_dtype="bf16"),
    # the same at the printed 21.3x compression: 768 numbers per token and
    # layer (r_K = r_V = 384) instead of the configured 1152
    "ouro_lla2d_768_r384": ConfigShape("ouro_lla2d_768_r384", "lla2d", B=768, L=24, T=4, H=16, d_h=128,
                                       D=0, N=4096, W=0, r_k=384, r_v=384, r_1=0, lat_dtype="bf16"),
    # the gate workload with fp8 (e4m3) latent rows and per-token scales
    "ouro_lla2d_768_fp8": ConfigShape("ouro_lla2d_768_fp8", "lla2d", B=768, L=24, T=4, H=16, d_h=128,
                                      D=0, N=4096, W=0, r_k=576, r_v=576, r_1=0, lat_dtype="fp8"),
    # long-context HLA, 16k, batch 64
    "ouro_hla_16k": ConfigShape("ouro_hla_16k", "hla", B=64, L=24, T=4, H=16, d_h=128, D=2048,
                                N=16384, W=128, r_k=512, r_v=512, r_1=256, lat_dtype="bf16"),
}


def _gen(seed, device="cpu"):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


# ---------------------------------------------------------------- tiny --
def tiny_hla(seed=0):
    """Tiny fp32 HLA layer: every tensor ~ N(0, 1/d) with d = d_model = 128.

    Draw order from numpy default_rng(seed): h [N,T,D], E_1 [2r_1,D],
    E_2..T [T-1,r_k+r_v,D], A_1 [1,H,d_h,r_1], A_2..T [T-1,H,d_h,r_k],
    B_1 [1,H,r_1,d_h], B_2..T [T-1,H,r_v,d_h], q [T,H,d_h], then the ring
    K, V [T,W+1,H,d_h] (slot j mod (W+1) holds token j).  fp64 draws cast to
    fp32; the fp32 values are the shared input.
    """
    c = CONFIGS["tiny_hla"]
    rng = np.random.default_rng(seed)
    sd = 1.0 / math.sqrt(c.D)

    def draw(*shape):
        return (rng.standard_normal(shape) * sd).astype(np.float32)

    out = {}
    out["h"] = draw(c.N, c.T, c.D)
    out["E_1"] = draw(2 * c.r_1, c.D)
    out["E_main"] = draw(c.T - 1, c.r_k + c.r_v, c.D)
    out["A_1"] = draw(1, c.H, c.d_h, c.r_1)
    out["A"] = draw(c.T - 1, c.H, c.d_h, c.r_k)
    out["B_1"] = draw(1, c.H, c.r_1, c.d_h)
    out["Bm"] = draw(c.T - 1, c.H, c.r_v, c.d_h)
    out["q"] = draw(c.T, c.H, c.d_h)
    out["win_k"] = draw(c.T, c.W + 1, c.H, c.d_h)
    out["win_v"] = draw(c.T, c.W + 1, c.H, c.d_h)
    return out


# ---------------------------------------------------- HLA activations --
def hla_hidden(P, n, seed, D, device="cpu", dtype=torch.float32):
    """Hidden states [n, T, D]: h_{j,t} = sum_s P[t,s] u_{j,s} + NOISE * eps,
    u_{j,s}, eps ~ N(0, I_D): a rank-8 trajectory across loops plus noise."""
    g = _gen(seed, device)
    T, R = P.shape
    P = P.to(device=device, dtype=dtype)
    u = torch.randn(n, R, D, generator=g, device=device, dtype=dtype)
    h = torch.einsum("ts,nsd->ntd", P, u).contiguous()
    h += NOISE * torch.randn(n, T, D, generator=g, device=device, dtype=dtype)
    return h


def _top_right_singular(x, k):
    """First k right singular vectors of x (rows = samples), fp64."""
    _, _, vh = torch.linalg.svd(x, full_matrices=False)
    if vh.shape[0] < k:
        raise ValueError("not enough calibration samples for the requested rank")
    return vh[:k]


def _pair_freq(r, d_h):
    return [(p * d_h) // r for p in range(r // 2)]


def _fit_hla_group(k, v, W_K, W_V, r_k, r_v):
    """Codec of one loop group from calibration keys/values k, v [n, G, H, d_h].

    Keys: frequency-aligned, latent pair p serves frequency floor(p d_h / r_k);
    the pairs of frequency f take the top singular vectors of that frequency's
    (loop, head) samples.  Values: plain SVD of [G*H*d_h] samples.
    """
    n, G, H, d_h = k.shape
    D = W_K.shape[2]
    E = torch.zeros(G, r_k + r_v, D, dtype=torch.float64)
    A = torch.zeros(G, H, d_h, r_k, dtype=torch.float64)
    Bm = torch.zeros(G, H, r_v, d_h, dtype=torch.float64)
    freq = _pair_freq(r_k, d_h)
    pairs_of = {}
    for p, f in enumerate(freq):
        pairs_of.setdefault(f, []).append(p)
    for f, plist in pairs_of.items():
        samples = torch.cat([k[..., 2 * f].reshape(n, G * H), k[..., 2 * f + 1].reshape(n, G * H)], 0)
        u = _top_right_singular(samples, len(plist)).reshape(len(plist), G, H)
        for s, p in enumerate(plist):
            # E rows: sum over heads of u * (head-h projection rows of this pair)
            E[:, 2 * p] = torch.einsum("gh,hd->gd", u[s], W_K[:, 2 * f])
            E[:, 2 * p + 1] = torch.einsum("gh,hd->gd", u[s], W_K[:, 2 * f + 1])
            A[:, :, 2 * f, 2 * p] = u[s]
            A[:, :, 2 * f + 1, 2 * p + 1] = u[s]
    bv = _top_right_singular(v.reshape(n, G * H * d_h), r_v).reshape(r_v, G, H, d_h)
    E[:, r_k:] = torch.einsum("sghd,hdD->gsD", bv, W_V)
    Bm[:] = bv.permute(1, 2, 0, 3)
    return E, A, Bm


def hla_codec(shape, seed, n_cal=1024):
    """Model and codec of one HLA layer, fitted on n_cal calibration tokens.

    Returns float32 CPU tensors: W_K, W_V [H,d_h,D], P [T,8], E_main
    [T-1,r_k+r_v,D], E_1 [2r_1,D], A [T-1,H,d_h,r_k], A_1 [1,H,d_h,r_1],
    Bm [T-1,H,r_v,d_h], B_1 [1,H,r_1,d_h].
    """
    c = shape
    g = _gen(seed)
    P = torch.randn(c.T, TRAJ_RANK, generator=g, dtype=torch.float64) / math.sqrt(TRAJ_RANK)
    W_K = torch.randn(c.H, c.d_h, c.D, generator=g, dtype=torch.float64) / math.sqrt(c.D)
    W_V = torch.randn(c.H, c.d_h, c.D, generator=g, dtype=torch.float64) / math.sqrt(c.D)
    h = hla_hidden(P, n_cal, seed + 1, c.D, dtype=torch.float64)
    k = torch.einsum("hdD,ntD->nthd", W_K, h)
    v = torch.einsum("hdD,ntD->nthd", W_V, h)
    E, A, Bm = _fit_hla_group(k[:, 1:], v[:, 1:], W_K, W_V, c.r_k, c.r_v)
    E1, A1, B1 = _fit_hla_group(k[:, :1], v[:, :1], W_K, W_V, c.r_1, c.r_1)
    f32 = lambda t: t.to(torch.float32).contiguous()  # noqa: E731
    return dict(P=f32(P), W_K=f32(W_K), W_V=f32(W_V), E_main=f32(E), E_1=f32(E1[0]), A=f32(A),
                A_1=f32(A1), Bm=f32(Bm), B_1=f32(B1))


# ---------------------------------------------------- LLA activations --
def lla_kv(P, n, d_h, seed, device="cpu", dtype=torch.float32):
    """Per-loop keys and values [n, T, H, d_h] with per-head rank-8 loop
    trajectories: k_{j,t,h} = sum_s P[h,t,s] u_{j,h,s} + NOISE * eps."""
    g = _gen(seed, device)
    H, T, R = P.shape
    P = P.to(device=device, dtype=dtype)
    out = []
    for _ in range(2):
        u = torch.randn(n, H, R, d_h, generator=g, device=device, dtype=dtype)
        x = torch.einsum("hts,nhsd->nthd", P, u).contiguous()
        x += NOISE * torch.randn(n, T, H, d_h, generator=g, device=device, dtype=dtype)
        out.append(x)
    return out[0], out[1]


def _lla_model(shape, seed):
    g = _gen(seed)
    return torch.randn(shape.H, shape.T, TRAJ_RANK, generator=g, dtype=torch.float64) / math.sqrt(TRAJ_RANK)


def lla_perhead_codec(shape, seed, n_cal=256):
    """Per-head SVD codec: E_K, E_V [T,H,r,d_h] and U_K, U_V [T,H,d_h,r] (float32)."""
    c = shape
    P = _lla_model(c, seed)
    k, v = lla_kv(P, n_cal, c.d_h, seed + 1, dtype=torch.float64)
    r = c.r_k
    EK = torch.zeros(c.T, c.H, r, c.d_h, dtype=torch.float64)
    EV = torch.zeros_like(EK)
    for h in range(c.H):
        bk = _top_right_singular(k[:, :, h].reshape(n_cal, c.T * c.d_h), r).reshape(r, c.T, c.d_h)
        bv = _top_right_singular(v[:, :, h].reshape(n_cal, c.T * c.d_h), r).reshape(r, c.T, c.d_h)
        EK[:, h] = bk.permute(1, 0, 2)
        EV[:, h] = bv.permute(1, 0, 2)
    f32 = lambda t: t.to(torch.float32).contiguous()  # noqa: E731
    return dict(P=f32(P), E_K=f32(EK), E_V=f32(EV), U_K=f32(EK.transpose(2, 3)), U_V=f32(EV.transpose(2, 3)))


def lla_folded_codec(shape, seed, n_cal=1024):
    """LLA-2D SVD codec: E_K [T,H,r_K,d_h], E_V [T,H,r_V,d_h], U_K [T,H,d_h,r_K],
    U_V [T,H,d_h,r_V] (float32)."""
    c = shape
    P = _lla_model(c, seed)
    k, v = lla_kv(P, n_cal, c.d_h, seed + 1, dtype=torch.float64)
    bk = _top_right_singular(k.reshape(n_cal, -1), c.r_k).reshape(c.r_k, c.T, c.H, c.d_h)
    bv = _top_right_singular(v.reshape(n_cal, -1), c.r_v).reshape(c.r_v, c.T, c.H, c.d_h)
    f32 = lambda t: t.to(torch.float32).contiguous()  # noqa: E731
    return dict(P=f32(P), E_K=f32(bk.permute(1, 2, 0, 3)), E_V=f32(bv.permute(1, 2, 0, 3)),
                U_K=f32(bk.permute(1, 2, 3, 0)), U_V=f32(bv.permute(1, 2, 3, 0)))


# ---------------------------------------------------------- per call --
def queries(B, nt, H, d_h, seed, device="cpu"):
    """Queries q ~ N(0, 1) [B, nt, H, d_h] float32."""
    return torch.randn(B, nt, H, d_h, generator=_gen(seed, device), device=device)


def window_ring(k_last, v_last, N, Wcap, dtype=torch.bfloat16):
    """Ring [B, T, Wcap, H, d_h] holding the tokens N-n..N-1 given as
    k_last, v_last [B, n, T, H, d_h] (token N-n+x in slot (N-n+x) mod Wcap).
    Unfilled slots are zero."""
    B, n, T, H, d_h = k_last.shape
    rk = torch.zeros(B, T, Wcap, H, d_h, dtype=dtype, device=k_last.device)
    rv = torch.zeros_like(rk)
    for x in range(n):
        slot = (N - n + x) % Wcap
        rk[:, :, slot] = k_last[:, x].to(dtype)
        rv[:, :, slot] = v_last[:, x].to(dtype)
    return rk, rv


def random_latents(B, n, width, seed, dtype=torch.bfloat16, std=1.0, device="cpu"):
    """Latent rows drawn directly ~ N(0, std^2) [B, n, width]."""
    x = torch.randn(B, n, width, generator=_gen(seed, device), device=device) * std
    return x.to(dtype)


def random_fp8_rows(B, n, r_k, r_v, seed, device="cpu"):
    """fp8 latent rows [B, n, r_k + r_v + 16] (uint8): e4m3 codes of N(0, 100^2)
    draws clipped to +-448 (torch's float32 -> float8_e4m3fn conversion), then
    per-token scales s^K, s^V ~ U(0.002, 0.02) as fp32 bytes, then 8 zero
    bytes."""
    g = _gen(seed)
    w = r_k + r_v
    x = (torch.randn(B, n, w, generator=g) * 100).clamp(-448, 448)
    codes = x.to(torch.float8_e4m3fn).view(torch.uint8)
    sc = (torch.rand(B, n, 2, generator=g) * 0.018 + 0.002).to(torch.float32)
    rows = torch.zeros(B, n, w + 16, dtype=torch.uint8)
    rows[:, :, :w] = codes
    rows[:, :, w:w + 8] = sc.view(torch.uint8).reshape(B, n, 8)
    return rows.to(device)
