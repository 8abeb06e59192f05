"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
identical seeded inputs.  Tolerances: relative L2 <= 1e-4 for fp32 latents,
<= 2e-2 for bf16-stored latents (fp32 accumulate), pooled over the call AND for
every (sequence, loop, head) output row, plus a per-element bound relative to
the row's largest magnitude (parity_check.assert_rows_close); writer layout
bit-exact."""

import math

import numpy as np
import pytest
import torch

import looped_transformer_latent_b200 as L
import synth
from oracle import hla, lla, quant, rounding
from parity_check import assert_rows_close

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
TOL_BF16 = 2e-2
BASE = 10000.0


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def _gen(seed):
    g = torch.Generator()
    g.manual_seed(seed)
    return g


# ------------------------------------------------------------- tiny HLA --
def test_tiny_hla_layer_matches_oracle(cuda_device):
    """Tiny fp32 HLA layer: writer (eq. 2) then both reads (loop 1 with
    c^(1), loops 2..4 with c) through the C ABI, against the oracle."""
    c = synth.CONFIGS["tiny_hla"]
    x = synth.tiny_hla(0)
    # oracle
    lat_o, lat1_o = hla.write(x["h"], x["E_main"], x["E_1"], 0, c.r_k, c.r_v, c.r_1, c.d_h, c.base)
    lat_o, lat1_o = rounding.to_f32(lat_o), rounding.to_f32(lat1_o)
    o1 = hla.decode(lat1_o, x["A_1"], x["B_1"], x["q"][:1], x["win_k"], x["win_v"], 0, c.N, c.W,
                    c.r_1, c.r_1, c.d_h, c.base)
    om = hla.decode(lat_o, x["A"], x["Bm"], x["q"][1:], x["win_k"], x["win_v"], 1, c.N, c.W,
                    c.r_k, c.r_v, c.d_h, c.base)
    # CUDA path
    dev = cuda_device
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)  # noqa: E731
    h = T(x["h"])[None]
    lat = torch.full((1, c.N, c.r_k + c.r_v), float("nan"), device=dev)
    lat1 = torch.full((1, c.N, 2 * c.r_1), float("nan"), device=dev)
    L.lla_write_latents(L.LLA_WRITE_HLA, x=h, E_main=T(x["E_main"]), E_1=T(x["E_1"]), out0=lat,
                        out1=lat1, r_k=c.r_k, d_h=c.d_h, pos0=0, rope_base=c.base)
    q = T(x["q"])[None]
    wk, wv = T(x["win_k"])[None], T(x["win_v"])[None]
    out1 = torch.empty(1, 1, c.H, c.d_h, device=dev)
    outm = torch.empty(1, c.T - 1, c.H, c.d_h, device=dev)
    L.hla_decode_attn(lat=lat1, A=T(x["A_1"]), Bm=T(x["B_1"]), q=q[:, :1].contiguous(), win_k=wk,
                      win_v=wv, out=out1, N=c.N, W=c.W, t0=0, rope_base=c.base)
    L.hla_decode_attn(lat=lat, A=T(x["A"]), Bm=T(x["Bm"]), q=q[:, 1:].contiguous(), win_k=wk,
                      win_v=wv, out=outm, N=c.N, W=c.W, t0=1, rope_base=c.base)
    torch.cuda.synchronize()
    # fp32 rows: the writer's fp32 accumulation over (T-1) D = 384 terms moves
    # single elements by ~1e-6 of the row's largest value
    assert_rows_close(lat[0], lat_o, 1e-6, "tiny HLA main latent rows", elem_tol=1e-5)
    assert_rows_close(lat1[0], lat1_o, 1e-6, "tiny HLA loop-1 latent rows", elem_tol=1e-5)
    e1 = assert_rows_close(out1[0], o1, TOL_F32, "tiny HLA loop 1")
    em = assert_rows_close(outm[0], om, TOL_F32, "tiny HLA loops 2..4")
    print(f"tiny HLA rel L2 (pooled, worst row): loop1 {e1} main {em}")


# ------------------------------------------------- absorbed read, bf16 --
def _absorbed_case(seed, B, N, W, H, nt, d_h, r_k, r_v, Wcap, t0=1, lat_dtype=torch.bfloat16,
                   rotate=True):
    g = _gen(seed)
    T = t0 + nt
    lat = (torch.randn(B, max(N, 1), r_k + r_v, generator=g) * math.sqrt(d_h / r_k)).to(lat_dtype)
    A = torch.randn(nt, H, d_h, r_k, generator=g) / math.sqrt(d_h)
    Bm = torch.randn(nt, H, r_v, d_h, generator=g) / math.sqrt(r_v)
    q = torch.randn(B, nt, H, d_h, generator=g)
    wk = torch.randn(B, T, Wcap, H, d_h, generator=g).to(torch.bfloat16)
    wv = torch.randn(B, T, Wcap, H, d_h, generator=g).to(torch.bfloat16)
    return dict(lat=lat, A=A, Bm=Bm, q=q, wk=wk, wv=wv, t0=t0, T=T)


def _absorbed_oracle(cs, N, W, r_k, r_v, d_h, rotate):
    B = cs["q"].shape[0]
    out = []
    for b in range(B):
        out.append(hla.decode(f64(cs["lat"][b]), f64(cs["A"]), f64(cs["Bm"]), f64(cs["q"][b]),
                              f64(cs["wk"][b]), f64(cs["wv"][b]), cs["t0"], N, W, r_k, r_v, d_h,
                              BASE, rotate_query=rotate))
    return np.stack(out)


def _absorbed_gpu(cs, dev, N, W, rotate, **extra):
    out = torch.full(tuple(cs["q"].shape), float("nan"), device=dev)
    L.hla_decode_attn(lat=cs["lat"].to(dev), A=cs["A"].to(dev), Bm=cs["Bm"].to(dev),
                      q=cs["q"].to(dev), win_k=cs["wk"].to(dev), win_v=cs["wv"].to(dev), out=out,
                      N=N, W=W, t0=cs["t0"], rotate_query=rotate, rope_base=BASE, **extra)
    torch.cuda.synchronize()
    return f64(out)


ABSORBED_CASES = [
    # B, N, W, H, nt, d_h, r_k, r_v, Wcap
    (3, 301, 16, 4, 3, 64, 128, 96, 17),      # several tiles, ragged tail
    (2, 1, 8, 2, 1, 64, 64, 64, 9),           # N = 1: only the current token
    (2, 10, 16, 2, 2, 64, 64, 64, 17),        # W >= i: no latent token
    (2, 18, 16, 2, 1, 64, 64, 64, 17),        # exactly one latent token
    (2, 700, 128, 16, 3, 128, 512, 512, 129), # Ouro-shaped main latent (48 rows)
    (2, 650, 128, 16, 1, 128, 256, 256, 129), # Ouro-shaped loop-1 latent (16 rows)
    (1, 1100, 0, 16, 4, 128, 576, 576, 1),    # LLA-2D-shaped: 64 rows, no window
    (5, 257, 4, 3, 2, 32, 32, 40, 7),         # small ranks, ring larger than needed
]


@pytest.mark.parametrize("case", ABSORBED_CASES)
@pytest.mark.parametrize("rotate", [True, False])
def test_absorbed_read_bf16(cuda_device, case, rotate):
    B, N, W, H, nt, d_h, r_k, r_v, Wcap = case
    cs = _absorbed_case(1000 + N + H, B, N, W, H, nt, d_h, r_k, r_v, Wcap)
    ref = _absorbed_oracle(cs, N, W, r_k, r_v, d_h, rotate)
    got = _absorbed_gpu(cs, cuda_device, N, W, rotate)
    err = assert_rows_close(got, ref, TOL_BF16, f"absorbed {case} rotate={rotate}")
    print(f"absorbed {case} rotate={rotate}: rel L2 (pooled, worst row) {err}")


@pytest.mark.parametrize("splits", [1, 2, 5, 16])
def test_absorbed_read_split_count(cuda_device, monkeypatch, splits):
    """The tensor-core read with the planner's split count forced: one split
    (no merge of partials), a few, and more than the context has tiles (the
    count is capped at one tile per split)."""
    monkeypatch.setenv("LLA_READ_SPLITS", str(splits))
    for case in (ABSORBED_CASES[0], ABSORBED_CASES[4]):
        B, N, W, H, nt, d_h, r_k, r_v, Wcap = case
        cs = _absorbed_case(1000 + N + H, B, N, W, H, nt, d_h, r_k, r_v, Wcap)
        ref = _absorbed_oracle(cs, N, W, r_k, r_v, d_h, True)
        got = _absorbed_gpu(cs, cuda_device, N, W, True)
        err = assert_rows_close(got, ref, TOL_BF16, f"absorbed {case}, {splits} splits")
        print(f"absorbed {case}, {splits} splits: rel L2 (pooled, worst row) {err}")


def test_absorbed_read_fp32_latents(cuda_device):
    B, N, W, H, nt, d_h, r_k, r_v, Wcap = 2, 333, 16, 4, 2, 64, 128, 64, 20
    cs = _absorbed_case(77, B, N, W, H, nt, d_h, r_k, r_v, Wcap, lat_dtype=torch.float32)
    cs["wk"], cs["wv"] = cs["wk"].float(), cs["wv"].float()
    assert_rows_close(_absorbed_gpu(cs, cuda_device, N, W, True),
                      _absorbed_oracle(cs, N, W, r_k, r_v, d_h, True), TOL_F32, "fp32 latents")


def test_explicit_scale(cuda_device):
    B, N, W, H, nt, d_h, r_k, r_v, Wcap = 2, 90, 8, 2, 1, 64, 64, 64, 9
    cs = _absorbed_case(5, B, N, W, H, nt, d_h, r_k, r_v, Wcap)
    ref = np.stack([hla.decode(f64(cs["lat"][b]), f64(cs["A"]), f64(cs["Bm"]), f64(cs["q"][b]),
                               f64(cs["wk"][b]), f64(cs["wv"][b]), cs["t0"], N, W, r_k, r_v, d_h,
                               BASE, scale=0.3) for b in range(B)])
    got = _absorbed_gpu(cs, cuda_device, N, W, True, scale=0.3)
    assert_rows_close(got, ref, TOL_BF16, "explicit scale")


def test_strided_latent_view(cuda_device):
    """A latent view with padded rows and a batch stride larger than dense."""
    B, N, W, H, nt, d_h, r_k, r_v, Wcap = 2, 200, 8, 2, 2, 64, 64, 64, 9
    cs = _absorbed_case(9, B, N, W, H, nt, d_h, r_k, r_v, Wcap)
    big = torch.zeros(B, N + 7, r_k + r_v + 64, dtype=torch.bfloat16)
    big[:, :N, :r_k + r_v] = cs["lat"]
    ref = _absorbed_oracle(cs, N, W, r_k, r_v, d_h, True)
    cs["lat"] = big[:, :, :r_k + r_v]
    dev = cuda_device
    out = torch.empty(tuple(cs["q"].shape), device=dev)
    L.hla_decode_attn(lat=big.to(dev)[:, :, :r_k + r_v], A=cs["A"].to(dev), Bm=cs["Bm"].to(dev),
                      q=cs["q"].to(dev), win_k=cs["wk"].to(dev), win_v=cs["wv"].to(dev), out=out,
                      N=N, W=W, t0=cs["t0"], rope_base=BASE)
    torch.cuda.synchronize()
    assert_rows_close(out, ref, TOL_BF16, "strided latent view")


# ------------------------------------------------ writer: exact layout --
def _int_tensor(g, shape, lo, hi):
    return torch.randint(lo, hi + 1, shape, generator=g).to(torch.float32)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_writer_hla_layout_bit_exact(cuda_device, dtype):
    """Small integers in h and E make every latent exactly representable, so
    the stored rows (and the untouched ones) must equal the oracle's bits."""
    g = _gen(3)
    B, n, pos0, Ncap, T, D, r_k, r_v, r_1, d_h = 3, 7, 5, 16, 4, 32, 16, 24, 8, 8
    h = _int_tensor(g, (B, n, T, D), -2, 2)
    E = (_int_tensor(g, (T - 1, r_k + r_v, D), -1, 1) * (torch.rand(T - 1, r_k + r_v, D, generator=g) < 0.15))
    E1 = (_int_tensor(g, (2 * r_1, D), -1, 1) * (torch.rand(2 * r_1, D, generator=g) < 0.15))
    sentinel = 1234.0
    dev = cuda_device
    lat = torch.full((B, Ncap, r_k + r_v), sentinel, dtype=dtype, device=dev)
    lat1 = torch.full((B, Ncap, 2 * r_1), sentinel, dtype=dtype, device=dev)
    L.lla_write_latents(L.LLA_WRITE_HLA, x=h.to(dev), E_main=E.to(dev), E_1=E1.to(dev), out0=lat,
                        out1=lat1, r_k=r_k, d_h=d_h, pos0=pos0, rotate_keys=False)
    torch.cuda.synchronize()
    exp = torch.full((B, Ncap, r_k + r_v), sentinel, dtype=torch.float64)
    exp1 = torch.full((B, Ncap, 2 * r_1), sentinel, dtype=torch.float64)
    for b in range(B):
        c, c1 = hla.write(h[b].double().numpy(), E.double().numpy(), E1.double().numpy(), pos0,
                          r_k, r_v, r_1, d_h, BASE, rotate_keys=False)
        exp[b, pos0:pos0 + n] = torch.from_numpy(c)
        exp1[b, pos0:pos0 + n] = torch.from_numpy(c1)
    assert torch.equal(lat.cpu(), exp.to(dtype))
    assert torch.equal(lat1.cpu(), exp1.to(dtype))


@pytest.mark.parametrize("d_h", [16, 32])     # 16: SIMT writer; 32: tensor-core writer (tensor-map view)
@pytest.mark.parametrize("mode", [L.LLA_WRITE_PERHEAD, L.LLA_WRITE_FOLDED])
def test_writer_lla_layout_bit_exact(cuda_device, mode, d_h):
    g = _gen(4 + mode + d_h)
    B, n, pos0, Ncap, T, H = 2, 5, 3, 12, 3, 3
    r = 16 if mode == L.LLA_WRITE_PERHEAD else 24
    rV = r if mode == L.LLA_WRITE_PERHEAD else 40
    k = _int_tensor(g, (B, n, T, H, d_h), -2, 2)
    v = _int_tensor(g, (B, n, T, H, d_h), -2, 2)
    EK = _int_tensor(g, (T, H, r, d_h), -1, 1) * (torch.rand(T, H, r, d_h, generator=g) < 0.2)
    EV = _int_tensor(g, (T, H, rV, d_h), -1, 1) * (torch.rand(T, H, rV, d_h, generator=g) < 0.2)
    dev = cuda_device
    sentinel = -77.0
    if mode == L.LLA_WRITE_PERHEAD:
        cK = torch.full((B, H, Ncap, r), sentinel, dtype=torch.bfloat16, device=dev)
        cV = torch.full((B, H, Ncap, r), sentinel, dtype=torch.bfloat16, device=dev)
        L.lla_write_latents(mode, x=k.to(dev), xv=v.to(dev), E_K=EK.to(dev), E_V=EV.to(dev),
                            out0=cK, out1=cV, pos0=pos0)
        torch.cuda.synchronize()
        eK = torch.full((B, H, Ncap, r), sentinel, dtype=torch.float64)
        eV = eK.clone()
        for b in range(B):
            ck, cv = lla.write_perhead(k[b].double().numpy(), v[b].double().numpy(),
                                       EK.double().numpy(), EV.double().numpy())
            eK[b, :, pos0:pos0 + n] = torch.from_numpy(ck)
            eV[b, :, pos0:pos0 + n] = torch.from_numpy(cv)
        assert torch.equal(cK.cpu(), eK.to(torch.bfloat16))
        assert torch.equal(cV.cpu(), eV.to(torch.bfloat16))
    else:
        lat = torch.full((B, Ncap, r + rV), sentinel, dtype=torch.bfloat16, device=dev)
        L.lla_write_latents(mode, x=k.to(dev), xv=v.to(dev), E_K=EK.to(dev), E_V=EV.to(dev),
                            out0=lat, pos0=pos0)
        torch.cuda.synchronize()
        e = torch.full((B, Ncap, r + rV), sentinel, dtype=torch.float64)
        for b in range(B):
            e[b, pos0:pos0 + n] = torch.from_numpy(lla.write_folded(
                k[b].double().numpy(), v[b].double().numpy(), EK.double().numpy(), EV.double().numpy()))
        assert torch.equal(lat.cpu(), e.to(torch.bfloat16))


def _accumulation_bound(x_blocks, e_blocks):
    """Bound on the fp32 accumulation error of each written value: the sum of
    the magnitudes of its K products times sqrt(K) 2^-22 (a few fp32 roundings
    per product, random-walk growth), widened over each rotated pair (a
    rotation mixes the two members with |cos| + |sin| <= 2)."""
    ax = np.abs(np.concatenate([np.asarray(b, np.float64) for b in x_blocks], axis=1))
    ae = np.abs(np.concatenate([np.asarray(b, np.float64) for b in e_blocks], axis=1))
    s = ax @ ae.T
    s = np.maximum(s[:, 0::2], s[:, 1::2]).repeat(2, axis=1) * 2.0
    return np.sqrt(ax.shape[1]) * 2.0 ** -22 * s


def test_writer_rotation_and_rounding(cuda_device):
    """Rotated bf16 writes: each value within one bf16 ulp of the oracle's plus
    the fp32 accumulation error bound (where a value cancels to far below its
    terms, fp32 summation alone can move it by more than one bf16 ulp), and
    at least 95 % of the values equal to the oracle's rounded value."""
    c = synth.CONFIGS["tiny_hla"]
    x = synth.tiny_hla(1)
    dev = cuda_device
    pos0 = 100
    n = 64
    h = torch.from_numpy(x["h"][:n])[None].to(dev)
    lat = torch.zeros(1, pos0 + n, c.r_k + c.r_v, dtype=torch.bfloat16, device=dev)
    lat1 = torch.zeros(1, pos0 + n, 2 * c.r_1, dtype=torch.bfloat16, device=dev)
    L.lla_write_latents(L.LLA_WRITE_HLA, x=h, E_main=torch.from_numpy(x["E_main"]).to(dev),
                        E_1=torch.from_numpy(x["E_1"]).to(dev), out0=lat, out1=lat1, r_k=c.r_k,
                        d_h=c.d_h, pos0=pos0, rope_base=c.base)
    torch.cuda.synchronize()
    ce, c1e = hla.write(x["h"][:n], x["E_main"], x["E_1"], pos0, c.r_k, c.r_v, c.r_1, c.d_h, c.base)
    hx = x["h"][:n]
    acc_main = _accumulation_bound([hx[:, t] for t in range(1, c.T)], list(x["E_main"]))
    acc_1 = _accumulation_bound([hx[:, 0]], [x["E_1"]])
    for got, exact, acc in ((f64(lat[0, pos0:]), ce, acc_main), (f64(lat1[0, pos0:]), c1e, acc_1)):
        ulp = np.abs(rounding.to_bf16(exact)) * 2.0 ** -7 + 1e-30
        assert np.all(np.abs(got - exact) <= ulp + acc)
        assert np.mean(got == rounding.to_bf16(exact)) > 0.95


# --------------------------------------------- LLA reconstruct-on-read --
LLA_CASES = [
    # B, H, d_h, r, T, t0, nt, N, W, Wcap
    (2, 3, 32, 32, 4, 0, 4, 200, 0, 1),
    (2, 2, 96, 96, 8, 2, 3, 77, 5, 6),
    (1, 1, 64, 64, 1, 0, 1, 1, 0, 1),        # N = 1
    (3, 2, 64, 32, 2, 0, 2, 129, 3, 4),      # r < d_h, ragged tile
    (1, 2, 128, 128, 2, 0, 2, 300, 2, 3),    # largest tensor-core layout (d_h = r = 128), ragged tile
    (3, 2, 96, 96, 8, 1, 5, 400, 0, 1),      # 5 loops: a group of 3 and a group of 2, 4 tiles
    (2, 1, 64, 80, 2, 0, 2, 260, 1, 2),      # rank 80: last 32-element chunk half zero-padded
    (2, 1, 32, 88, 3, 0, 3, 150, 0, 1),      # rank 88: last 16-element MMA step half zero-padded
]


def _lla_case(case, seed):
    B, H, d_h, r, T, t0, nt, N, W, Wcap = case
    g = _gen(seed)
    cK = torch.randn(B, H, N, r, generator=g).to(torch.bfloat16)
    cV = torch.randn(B, H, N, r, generator=g).to(torch.bfloat16)
    UK = torch.randn(nt, H, d_h, r, generator=g) / math.sqrt(r)
    UV = torch.randn(nt, H, d_h, r, generator=g) / math.sqrt(r)
    q = torch.randn(B, nt, H, d_h, generator=g)
    wk = torch.randn(B, T, Wcap, H, d_h, generator=g).to(torch.bfloat16)
    wv = torch.randn(B, T, Wcap, H, d_h, generator=g).to(torch.bfloat16)
    ref = np.stack([lla.decode_reconstruct(f64(cK[b]), f64(cV[b]), f64(UK), f64(UV), f64(q[b]),
                                           f64(wk[b]), f64(wv[b]), t0, N, W) for b in range(B)])
    return dict(cK=cK, cV=cV, UK=UK, UV=UV, q=q, wk=wk, wv=wv), ref


def _lla_gpu(x, case, dev):
    B, H, d_h, r, T, t0, nt, N, W, Wcap = case
    out = torch.full((B, nt, H, d_h), float("nan"), device=dev)
    L.lla_decode_attn(cK=x["cK"].to(dev), cV=x["cV"].to(dev), UK=x["UK"].to(dev), UV=x["UV"].to(dev),
                      q=x["q"].to(dev), win_k=x["wk"].to(dev), win_v=x["wv"].to(dev), out=out, N=N, W=W,
                      t0=t0)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("seq_per_cta", [2, 3, 8])
def test_lla_reconstruct_sequences_per_cta(cuda_device, monkeypatch, seq_per_cta):
    """One CTA walking several sequences with the same decoders in shared
    memory (the planner's choice forced): state must restart per sequence."""
    monkeypatch.setenv("LLA_RECON_SEQ_PER_CTA", str(seq_per_cta))
    case = (5, 2, 96, 96, 4, 0, 4, 300, 0, 1)
    x, ref = _lla_case(case, 71)
    out = _lla_gpu(x, case, cuda_device)
    err = assert_rows_close(out, ref, TOL_BF16, f"reconstruct, {seq_per_cta} sequences per CTA")
    print(f"reconstruct {seq_per_cta} sequences per CTA: rel L2 (pooled, worst row) {err}")


@pytest.mark.parametrize("case", LLA_CASES)
def test_lla_reconstruct_bf16(cuda_device, case):
    B, H, d_h, r, T, t0, nt, N, W, Wcap = case
    g = _gen(50 + N)
    cK = torch.randn(B, H, N, r, generator=g).to(torch.bfloat16)
    cV = torch.randn(B, H, N, r, generator=g).to(torch.bfloat16)
    UK = torch.randn(nt, H, d_h, r, generator=g) / math.sqrt(r)
    UV = torch.randn(nt, H, d_h, r, generator=g) / math.sqrt(r)
    q = torch.randn(B, nt, H, d_h, generator=g)
    wk = torch.randn(B, T, Wcap, H, d_h, generator=g).to(torch.bfloat16)
    wv = torch.randn(B, T, Wcap, H, d_h, generator=g).to(torch.bfloat16)
    ref = np.stack([lla.decode_reconstruct(f64(cK[b]), f64(cV[b]), f64(UK), f64(UV), f64(q[b]),
                                           f64(wk[b]), f64(wv[b]), t0, N, W) for b in range(B)])
    dev = cuda_device
    out = torch.full((B, nt, H, d_h), float("nan"), device=dev)
    L.lla_decode_attn(cK=cK.to(dev), cV=cV.to(dev), UK=UK.to(dev), UV=UV.to(dev), q=q.to(dev),
                      win_k=wk.to(dev), win_v=wv.to(dev), out=out, N=N, W=W, t0=t0)
    torch.cuda.synchronize()
    err = assert_rows_close(out, ref, TOL_BF16, f"lla reconstruct {case}")
    print(f"lla reconstruct {case}: rel L2 (pooled, worst row) {err}")


# ------------------------------------------ LLA-2D: writer + absorbed --
def test_lla2d_writer_then_absorbed_read(cuda_device):
    """End to end on LLA-2D: folded writer on both sides, then LLA-D (absorbed,
    no rotation) on each side's own latents."""
    g = _gen(60)
    B, T, H, d_h, rK, rV, N, W = 2, 2, 4, 32, 64, 64, 50, 0
    k = torch.randn(B, N, T, H, d_h, generator=g)
    v = torch.randn(B, N, T, H, d_h, generator=g)
    EK = torch.randn(T, H, rK, d_h, generator=g) / math.sqrt(T * H * d_h)
    EV = torch.randn(T, H, rV, d_h, generator=g) / math.sqrt(T * H * d_h)
    UK = torch.randn(T, H, d_h, rK, generator=g) / math.sqrt(rK)
    UV = torch.randn(T, H, d_h, rV, generator=g) / math.sqrt(rV)
    q = torch.randn(B, T, H, d_h, generator=g)
    Wcap = 1
    wk = torch.zeros(B, T, Wcap, H, d_h)
    wv = torch.zeros(B, T, Wcap, H, d_h)
    wk[:, :, (N - 1) % Wcap] = k[:, N - 1]
    wv[:, :, (N - 1) % Wcap] = v[:, N - 1]
    dev = cuda_device
    lat = torch.zeros(B, N, rK + rV, dtype=torch.bfloat16, device=dev)
    L.lla_write_latents(L.LLA_WRITE_FOLDED, x=k.to(dev), xv=v.to(dev), E_K=EK.to(dev),
                        E_V=EV.to(dev), out0=lat, pos0=0)
    out = torch.empty(B, T, H, d_h, device=dev)
    L.hla_decode_attn(lat=lat, A=UK.to(dev), Bm=UV.transpose(2, 3).contiguous().to(dev), q=q.to(dev),
                      win_k=wk.to(torch.bfloat16).to(dev), win_v=wv.to(torch.bfloat16).to(dev),
                      out=out, N=N, W=W, t0=0, rotate_query=False)
    torch.cuda.synchronize()
    ref = []
    for b in range(B):
        row = rounding.to_bf16(lla.write_folded(f64(k[b]), f64(v[b]), f64(EK), f64(EV)))
        ref.append(lla.decode_absorbed(row, f64(UK), f64(UV), f64(q[b]),
                                       f64(wk[b].to(torch.bfloat16)), f64(wv[b].to(torch.bfloat16)),
                                       0, N, W, rK, rV))
    err = assert_rows_close(out, np.stack(ref), TOL_BF16, "lla2d end to end")
    print(f"lla2d end to end rel L2 (pooled, worst row) {err}")


# ------------------------------------- streaming store = prefill rows --
STREAM_CASES = [
    # mode, dtype
    (L.LLA_WRITE_PERHEAD, torch.bfloat16),
    (L.LLA_WRITE_PERHEAD, torch.float32),
    (L.LLA_WRITE_FOLDED, torch.bfloat16),
    (L.LLA_WRITE_HLA, torch.bfloat16),
]


@pytest.mark.parametrize("mode,dtype", STREAM_CASES)
def test_streaming_store_matches_prefill_rows(cuda_device, mode, dtype):
    """Served semantics (LLA abstract, streaming latent store): the latent of
    a token written alone when it leaves the exact window -- one call with
    n = 1 at pos0 = j -- must be bit-identical to the row the prefill writer
    stored for it in a call over many tokens, since the read cannot tell which
    of the two wrote it."""
    g = _gen(90 + mode)
    dev = cuda_device
    B, n, T, H, d_h = 3, 200, 4, 5, 64
    if mode == L.LLA_WRITE_HLA:
        D, r_k, r_v, r_1 = 256, 128, 96, 64
        h = torch.randn(B, n, T, D, generator=g)
        E = torch.randn(T - 1, r_k + r_v, D, generator=g) / math.sqrt(D)
        E1 = torch.randn(2 * r_1, D, generator=g) / math.sqrt(D)
        kw = dict(E_main=E.to(dev), E_1=E1.to(dev), r_k=r_k, d_h=d_h, rope_base=BASE)
        outs = lambda: (torch.zeros(B, n, r_k + r_v, dtype=dtype, device=dev),  # noqa: E731
                        torch.zeros(B, n, 2 * r_1, dtype=dtype, device=dev))
        args = lambda j0, j1: dict(x=h[:, j0:j1].contiguous().to(dev))  # noqa: E731
    else:
        r = 96 if mode == L.LLA_WRITE_PERHEAD else 160
        k = torch.randn(B, n, T, H, d_h, generator=g)
        v = torch.randn(B, n, T, H, d_h, generator=g)
        EK = torch.randn(T, H, r, d_h, generator=g) / math.sqrt(T * d_h)
        EV = torch.randn(T, H, r, d_h, generator=g) / math.sqrt(T * d_h)
        kw = dict(E_K=EK.to(dev), E_V=EV.to(dev))
        if mode == L.LLA_WRITE_PERHEAD:
            outs = lambda: (torch.zeros(B, H, n, r, dtype=dtype, device=dev),  # noqa: E731
                            torch.zeros(B, H, n, r, dtype=dtype, device=dev))
        else:
            outs = lambda: (torch.zeros(B, n, 2 * r, dtype=dtype, device=dev), None)  # noqa: E731
        args = lambda j0, j1: dict(x=k[:, j0:j1].contiguous().to(dev),  # noqa: E731
                                   xv=v[:, j0:j1].contiguous().to(dev))
    pre0, pre1 = outs()
    L.lla_write_latents(mode, out0=pre0, out1=pre1, pos0=0, **args(0, n), **kw)
    one0, one1 = outs()
    picks = [0, 1, 77, n - 1]
    for j in picks:
        L.lla_write_latents(mode, out0=one0, out1=one1, pos0=j, **args(j, j + 1), **kw)
    torch.cuda.synchronize()
    tok = (lambda t, j: t[:, :, j]) if mode == L.LLA_WRITE_PERHEAD else (lambda t, j: t[:, j])
    for j in picks:
        assert torch.equal(tok(one0, j), tok(pre0, j)), f"row {j} differs"
        if one1 is not None:
            assert torch.equal(tok(one1, j), tok(pre1, j)), f"row {j} (second latent) differs"


# -------------------------------------- several query positions at once --
MQ_CASES = [
    # B, N, W, H, nt, nq, d_h, r_k, r_v, rotate, fp8
    (2, 700, 128, 16, 1, 4, 128, 256, 256, True, False),   # loop-1 latent, 4 positions x 16 rows
    (2, 500, 16, 8, 3, 2, 128, 512, 512, True, False),     # main latent, 2 positions x 24 rows
    (1, 900, 0, 8, 4, 2, 128, 576, 576, False, False),     # LLA-D folded, 2 positions x 32 rows
    (3, 20, 16, 4, 2, 4, 64, 128, 64, True, False),        # first positions have no latent token yet
    (2, 700, 128, 16, 1, 4, 128, 256, 256, True, True),    # fp8 rows, 4 positions
]


@pytest.mark.parametrize("case", MQ_CASES)
def test_several_query_positions(cuda_device, case):
    """Multi-query read: the last nq positions of the context in one call
    (prefill chunk / two-pass second pass), every latent tile shared by all
    positions' rows; each position must match its own decode read."""
    B, N, W, H, nt, nq, d_h, r_k, r_v, rotate, fp8 = case
    g = _gen(80 + N + nq)
    t0 = 1 if rotate else 0
    T = t0 + nt
    Wcap = min(N, W + nq) + 1
    if fp8:
        lat = synth.random_fp8_rows(B, N, r_k, r_v, 81 + N)
        lat_vals = [quant.from_row_bytes(lat[b].numpy(), r_k, r_v) for b in range(B)]
    else:
        lat = (torch.randn(B, N, r_k + r_v, generator=g) * math.sqrt(d_h / r_k)).to(torch.bfloat16)
        lat_vals = [f64(lat[b]) for b in range(B)]
    A = torch.randn(nt, H, d_h, r_k, generator=g) / math.sqrt(d_h)
    Bm = torch.randn(nt, H, r_v, d_h, generator=g) / math.sqrt(r_v)
    q = torch.randn(B, nq, nt, H, d_h, generator=g)
    wk = torch.randn(B, T, Wcap, H, d_h, generator=g).to(torch.bfloat16)
    wv = torch.randn(B, T, Wcap, H, d_h, generator=g).to(torch.bfloat16)
    dev = cuda_device
    out = torch.full(tuple(q.shape), float("nan"), device=dev)
    L.hla_decode_attn(lat=lat.to(dev), A=A.to(dev), Bm=Bm.to(dev), q=q.to(dev), win_k=wk.to(dev),
                      win_v=wv.to(dev), out=out, N=N, W=W, t0=t0, rotate_query=rotate, rope_base=BASE)
    torch.cuda.synchronize()
    ref = np.stack([hla.decode_positions(lat_vals[b], f64(A), f64(Bm), f64(q[b]), f64(wk[b]), f64(wv[b]), t0,
                                         N, W, r_k, r_v, d_h, BASE, rotate_query=rotate) for b in range(B)])
    err = assert_rows_close(out, ref, TOL_BF16, f"multi-query {case}")
    print(f"multi-query {case}: rel L2 (pooled, worst row) {err}")


# ------------------------------------------ window on a second stream --
@pytest.mark.parametrize("W,N", [(128, 700), (16, 300), (0, 200)])
def test_window_stream_bit_identical(cuda_device, W, N):
    """The exact window on the caller's second stream (fork and join events)
    gives the bits of the single-stream call, eagerly and replayed from a
    captured graph."""
    g = _gen(90 + W)
    B, H, nt, t0, d_h, r_k, r_v = 3, 16, 3, 1, 128, 512, 512
    T = t0 + nt
    dev = cuda_device
    lat = (torch.randn(B, N, r_k + r_v, generator=g) * math.sqrt(d_h / r_k)).to(torch.bfloat16).to(dev)
    A = (torch.randn(nt, H, d_h, r_k, generator=g) / math.sqrt(d_h)).to(dev)
    Bm = (torch.randn(nt, H, r_v, d_h, generator=g) / math.sqrt(r_v)).to(dev)
    q = torch.randn(B, nt, H, d_h, generator=g).to(dev)
    wk = torch.randn(B, T, W + 1, H, d_h, generator=g).to(torch.bfloat16).to(dev)
    wv = torch.randn(B, T, W + 1, H, d_h, generator=g).to(torch.bfloat16).to(dev)
    kw = dict(lat=lat, A=A, Bm=Bm, q=q, win_k=wk, win_v=wv, N=N, W=W, t0=t0, rotate_query=True, rope_base=BASE)
    ref = torch.full((B, nt, H, d_h), float("nan"), device=dev)
    L.hla_decode_attn(out=ref, **kw)
    side = torch.cuda.Stream(dev)
    evs = (torch.cuda.Event(), torch.cuda.Event())
    for ev in evs:
        ev.record()
    out = torch.full_like(ref, float("nan"))
    L.hla_decode_attn(out=out, win_stream=side, win_events=evs, **kw)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    # the same call captured and replayed (fork and join become graph edges)
    s = torch.cuda.Stream(dev)
    ws = torch.empty(L.hla_decode_workspace_bytes(out=out, **kw), dtype=torch.uint8, device=dev)
    out2 = torch.full_like(ref, float("nan"))
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        L.hla_decode_attn(out=out2, workspace=ws, stream=s, win_stream=side, win_events=evs, **kw)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out2, ref)
    del graph
