"""Full-size parity: every workload at its benchmark shape (same batch, context,
ranks, rows per call -- hence the same split plan and kernel launch configuration
bench.py times), checked against the oracle on sampled outputs.

A handful of distinct sequences are generated on the host and repeated across
the batch with plain device copies; queries differ for every sequence, so every
sampled output is a separate check.  Tolerance: relative L2 <= 2e-2 for bf16
latents (fp32 accumulation), pooled over each sampled sequence and for every
(loop, head) row of it, plus a per-element bound (parity_check)."""

import math

import numpy as np
import pytest
import torch

import looped_transformer_latent_b200 as L
import synth
from oracle import hla, lla
from parity_check import assert_rows_close

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2
BASE = 10000.0


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def _tile_batch(distinct, B, dev):
    """[B, ...] device tensor whose sequence b is distinct[b % len(distinct)]."""
    k = distinct.shape[0]
    out = torch.empty((B,) + tuple(distinct.shape[1:]), dtype=distinct.dtype, device=dev)
    d = distinct.to(dev)
    for b0 in range(0, B, k):
        n = min(k, B - b0)
        out[b0:b0 + n] = d[:n]
    return out


def _absorbed_full(dev, seed, B, N, W, H, nt, t0, T, d_h, r_k, r_v, rotate, samples):
    g = torch.Generator().manual_seed(seed)
    ndist = 3
    lat_d = (torch.randn(ndist, N, r_k + r_v, generator=g) * math.sqrt(d_h / r_k)).to(torch.bfloat16)
    A = torch.randn(nt, H, d_h, r_k, generator=g) / math.sqrt(d_h)
    Bm = torch.randn(nt, H, r_v, d_h, generator=g) / math.sqrt(r_v)
    q = torch.randn(B, nt, H, d_h, generator=g)
    Wcap = W + 1
    wk_d = torch.randn(ndist, T, Wcap, H, d_h, generator=g).to(torch.bfloat16)
    wv_d = torch.randn(ndist, T, Wcap, H, d_h, generator=g).to(torch.bfloat16)
    lat = _tile_batch(lat_d, B, dev)
    wk = _tile_batch(wk_d, B, dev)
    wv = _tile_batch(wv_d, B, dev)
    out = torch.full((B, nt, H, d_h), float("nan"), device=dev)
    L.hla_decode_attn(lat=lat, A=A.to(dev), Bm=Bm.to(dev), q=q.to(dev), win_k=wk, win_v=wv, out=out,
                      N=N, W=W, t0=t0, rotate_query=rotate, rope_base=BASE)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    errs = []
    for b in samples:
        k = b % ndist
        ref = hla.decode(f64(lat_d[k]), f64(A), f64(Bm), f64(q[b]), f64(wk_d[k]), f64(wv_d[k]), t0, N, W,
                         r_k, r_v, d_h, BASE, rotate_query=rotate)
        errs.append(assert_rows_close(out[b], ref, TOL_BF16, f"sequence {b}"))
    return errs


@pytest.mark.parametrize("group", ["main", "loop1"])
def test_ouro_hla_4k_reads(cuda_device, group):
    c = synth.CONFIGS["ouro_hla_4k"]
    if group == "main":
        args = dict(nt=c.T - 1, t0=1, r_k=c.r_k, r_v=c.r_v)
    else:
        args = dict(nt=1, t0=0, r_k=c.r_1, r_v=c.r_1)
    errs = _absorbed_full(cuda_device, 11, c.B, c.N, c.W, c.H, T=c.T, d_h=c.d_h, rotate=True,
                          samples=[0, 13, c.B - 1], **args)
    print(f"ouro_hla_4k {group}: rel L2 (pooled, worst row) {errs}")


@pytest.mark.parametrize("group", ["main", "loop1"])
def test_ouro_hla_16k_reads(cuda_device, group):
    c = synth.CONFIGS["ouro_hla_16k"]
    if group == "main":
        args = dict(nt=c.T - 1, t0=1, r_k=c.r_k, r_v=c.r_v)
    else:
        args = dict(nt=1, t0=0, r_k=c.r_1, r_v=c.r_1)
    errs = _absorbed_full(cuda_device, 12, c.B, c.N, c.W, c.H, T=c.T, d_h=c.d_h, rotate=True,
                          samples=[1, c.B - 1], **args)
    print(f"ouro_hla_16k {group}: rel L2 (pooled, worst row) {errs}")


@pytest.mark.parametrize("name", ["ouro_lla2d_768", "ouro_lla2d_768_r384"])
def test_ouro_lla2d_768_absorbed_read(cuda_device, name):
    c = synth.CONFIGS[name]
    errs = _absorbed_full(cuda_device, 13, c.B, c.N, 0, c.H, nt=c.T, t0=0, T=c.T, d_h=c.d_h, r_k=c.r_k,
                          r_v=c.r_v, rotate=False, samples=[0, 400, c.B - 1])
    print(f"{name}: rel L2 (pooled, worst row) {errs}")


@pytest.mark.parametrize("name", ["huginn_lla_4k", "huginn_lla_4k_w64"])
def test_huginn_lla_4k_reconstruct(cuda_device, name):
    c = synth.CONFIGS[name]
    B, H, N, r, T, d_h, W = c.B, c.H, c.N, c.r_k, c.T, c.d_h, c.W
    g = torch.Generator().manual_seed(14)
    ndist = 2
    cK_d = torch.randn(ndist, H, N, r, generator=g).to(torch.bfloat16)
    cV_d = torch.randn(ndist, H, N, r, generator=g).to(torch.bfloat16)
    UK = torch.randn(T, H, d_h, r, generator=g) / math.sqrt(r)
    UV = torch.randn(T, H, d_h, r, generator=g) / math.sqrt(r)
    q = torch.randn(B, T, H, d_h, generator=g)
    wk_d = torch.randn(ndist, T, W + 1, H, d_h, generator=g).to(torch.bfloat16)
    wv_d = torch.randn(ndist, T, W + 1, H, d_h, generator=g).to(torch.bfloat16)
    dev = cuda_device
    out = torch.full((B, T, H, d_h), float("nan"), device=dev)
    L.lla_decode_attn(cK=_tile_batch(cK_d, B, dev), cV=_tile_batch(cV_d, B, dev), UK=UK.to(dev),
                      UV=UV.to(dev), q=q.to(dev), win_k=_tile_batch(wk_d, B, dev),
                      win_v=_tile_batch(wv_d, B, dev), out=out, N=N, W=W, t0=0)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    errs = []
    for b, h in [(0, 0), (7, 31), (B - 1, H - 1)]:
        k = b % ndist
        ref = lla.decode_reconstruct(f64(cK_d[k][h:h + 1]), f64(cV_d[k][h:h + 1]), f64(UK[:, h:h + 1]),
                                     f64(UV[:, h:h + 1]), f64(q[b][:, h:h + 1]), f64(wk_d[k][:, :, h:h + 1]),
                                     f64(wv_d[k][:, :, h:h + 1]), 0, N, W)
        errs.append(assert_rows_close(out[b][:, h:h + 1], ref, TOL_BF16, f"sequence {b} head {h}"))
    print(f"{name}: rel L2 (pooled, worst row) {errs}")


def test_decode_step_writers_at_full_batch(cuda_device):
    """The writer as the decode step calls it: one token per sequence at row N-1,
    for each workload's mode and batch."""
    dev = cuda_device
    g = torch.Generator().manual_seed(15)
    # HLA (Ouro-shaped): E_main [3, 1024, 2048], E_1 [512, 2048]
    c = synth.CONFIGS["ouro_hla_4k"]
    h = torch.randn(c.B, 1, c.T, c.D, generator=g)
    E = torch.randn(c.T - 1, c.r_k + c.r_v, c.D, generator=g) / math.sqrt(c.D)
    E1 = torch.randn(2 * c.r_1, c.D, generator=g) / math.sqrt(c.D)
    lat = torch.zeros(c.B, c.N, c.r_k + c.r_v, dtype=torch.bfloat16, device=dev)
    lat1 = torch.zeros(c.B, c.N, 2 * c.r_1, dtype=torch.bfloat16, device=dev)
    L.lla_write_latents(L.LLA_WRITE_HLA, x=h.to(dev), E_main=E.to(dev), E_1=E1.to(dev), out0=lat, out1=lat1,
                        r_k=c.r_k, d_h=c.d_h, pos0=c.N - 1, rope_base=c.base)
    torch.cuda.synchronize()
    for b in (0, c.B - 1):
        cm, c1 = hla.write(f64(h[b]), f64(E), f64(E1), c.N - 1, c.r_k, c.r_v, c.r_1, c.d_h, c.base)
        assert_rows_close(lat[b, c.N - 1:], cm, 1e-2, "HLA main row")
        assert_rows_close(lat1[b, c.N - 1:], c1, 1e-2, "HLA loop-1 row")
    assert not lat[:, :c.N - 1].any()
    # LLA-2D (folded): batch 768, E [4, 16, 576, 128]
    c = synth.CONFIGS["ouro_lla2d_768"]
    k = torch.randn(c.B, 1, c.T, c.H, c.d_h, generator=g)
    v = torch.randn(c.B, 1, c.T, c.H, c.d_h, generator=g)
    EK = torch.randn(c.T, c.H, c.r_k, c.d_h, generator=g) / math.sqrt(c.T * c.H * c.d_h)
    EV = torch.randn(c.T, c.H, c.r_v, c.d_h, generator=g) / math.sqrt(c.T * c.H * c.d_h)
    rows = torch.zeros(c.B, 8, c.r_k + c.r_v, dtype=torch.bfloat16, device=dev)
    L.lla_write_latents(L.LLA_WRITE_FOLDED, x=k.to(dev), xv=v.to(dev), E_K=EK.to(dev), E_V=EV.to(dev),
                        out0=rows, pos0=7)
    torch.cuda.synchronize()
    for b in (0, 511, c.B - 1):
        ref = lla.write_folded(f64(k[b]), f64(v[b]), f64(EK), f64(EV))
        assert_rows_close(rows[b, 7:], ref, 1e-2, "LLA-2D row")
    # LLA per-head (Huginn-like): 55 heads, 32 loops, rank 96
    c = synth.CONFIGS["huginn_lla_4k"]
    k = torch.randn(c.B, 1, c.T, c.H, c.d_h, generator=g)
    v = torch.randn(c.B, 1, c.T, c.H, c.d_h, generator=g)
    EK = torch.randn(c.T, c.H, c.r_k, c.d_h, generator=g) / math.sqrt(c.T * c.d_h)
    EV = torch.randn(c.T, c.H, c.r_k, c.d_h, generator=g) / math.sqrt(c.T * c.d_h)
    cK = torch.zeros(c.B, c.H, 4, c.r_k, dtype=torch.bfloat16, device=dev)
    cV = torch.zeros(c.B, c.H, 4, c.r_k, dtype=torch.bfloat16, device=dev)
    L.lla_write_latents(L.LLA_WRITE_PERHEAD, x=k.to(dev), xv=v.to(dev), E_K=EK.to(dev), E_V=EV.to(dev),
                        out0=cK, out1=cV, pos0=3)
    torch.cuda.synchronize()
    for b in (0, c.B - 1):
        rk, rv = lla.write_perhead(f64(k[b]), f64(v[b]), f64(EK), f64(EV))
        assert_rows_close(cK[b, :, 3:], rk, 1e-2, "per-head K rows")
        assert_rows_close(cV[b, :, 3:], rv, 1e-2, "per-head V rows")


def test_ouro_lla2d_768_fp8_read(cuda_device):
    """The gate workload's shapes with fp8 rows (e4m3 codes, per-token scales)
    at batch 768, sampled sequences against the oracle's read of the same rows."""
    from oracle import quant
    c = synth.CONFIGS["ouro_lla2d_768_fp8"]
    B, N, H, T, d_h, r_k, r_v = c.B, c.N, c.H, c.T, c.d_h, c.r_k, c.r_v
    g = torch.Generator().manual_seed(17)
    ndist = 3
    rows_d = synth.random_fp8_rows(ndist, N, r_k, r_v, 18)
    A = torch.randn(T, H, d_h, r_k, generator=g) / math.sqrt(d_h)
    Bm = torch.randn(T, H, r_v, d_h, generator=g) / math.sqrt(r_v)
    q = torch.randn(B, T, H, d_h, generator=g)
    wk_d = torch.randn(ndist, T, 1, H, d_h, generator=g).to(torch.bfloat16)
    wv_d = torch.randn(ndist, T, 1, H, d_h, generator=g).to(torch.bfloat16)
    dev = cuda_device
    out = torch.full((B, T, H, d_h), float("nan"), device=dev)
    L.hla_decode_attn(lat=_tile_batch(rows_d, B, dev), A=A.to(dev), Bm=Bm.to(dev), q=q.to(dev),
                      win_k=_tile_batch(wk_d, B, dev), win_v=_tile_batch(wv_d, B, dev), out=out, N=N, W=0, t0=0,
                      rotate_query=False)
    torch.cuda.synchronize()
    errs = []
    for b in (0, 400, B - 1):
        k = b % ndist
        vals = quant.from_row_bytes(rows_d[k].numpy(), r_k, r_v)
        ref = hla.decode(vals, f64(A), f64(Bm), f64(q[b]), f64(wk_d[k]), f64(wv_d[k]), 0, N, 0, r_k, r_v, d_h,
                         BASE, rotate_query=False)
        errs.append(assert_rows_close(out[b], ref, TOL_BF16, f"sequence {b}"))
    print(f"ouro_lla2d_768_fp8: rel L2 (pooled, worst row) {errs}")
