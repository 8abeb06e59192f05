"""fp8 latent rows (e4m3 codes with per-token, per-part scales; HLA summary,
"Conclusion / Future directions": latents combined with quantisation):
the writer's bytes against the oracle's quantiser, and the tensor-core read of
such rows against the oracle's read of the same rows.

Row format: [codes of c^K | codes of c^V | s^K fp32 | s^V fp32 | 8 zero bytes].
Tolerances: bytes bit-exact where the latents are exact in fp32 (integer
inputs); otherwise each stored value within one e4m3 step of the oracle's and
the read within 2e-2 relative L2 (pooled, per row and per element, as the bf16
latents; the codes are exact f16 operands, the query and probabilities f16)."""

import math

import numpy as np
import pytest
import torch

import looped_transformer_latent_b200 as L
import synth
from oracle import hla, lla, quant
from parity_check import assert_rows_close

pytestmark = pytest.mark.gpu

TOL = 2e-2
BASE = 10000.0


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def _gen(seed):
    return torch.Generator().manual_seed(seed)


def _int_tensor(g, shape, lo, hi):
    return torch.randint(lo, hi + 1, shape, generator=g).to(torch.float32)


@pytest.mark.parametrize("mode", [L.LLA_WRITE_HLA, L.LLA_WRITE_FOLDED])
def test_fp8_writer_bytes_bit_exact(cuda_device, mode):
    """Integer inputs and sparse integer codecs make every latent exact in
    fp32, so the scales (fp32 max / 448), the quotients (fp32 division) and
    their e4m3 codes are determined: the stored bytes must equal the oracle's."""
    g = _gen(20 + mode)
    dev = cuda_device
    B, n, pos0, Ncap, T = 2, 9, 3, 14, 3
    if mode == L.LLA_WRITE_HLA:
        D, r_k, r_v, r_1, d_h = 64, 32, 48, 16, 16
        h = _int_tensor(g, (B, n, T, D), -3, 3)
        E = _int_tensor(g, (T - 1, r_k + r_v, D), -2, 2) * (torch.rand(T - 1, r_k + r_v, D, generator=g) < 0.2)
        E1 = _int_tensor(g, (2 * r_1, D), -2, 2) * (torch.rand(2 * r_1, D, generator=g) < 0.2)
        lat = torch.full((B, Ncap, r_k + r_v + 16), 0xAB, dtype=torch.uint8, device=dev)
        lat1 = torch.full((B, Ncap, 2 * r_1 + 16), 0xAB, dtype=torch.uint8, device=dev)
        L.lla_write_latents(L.LLA_WRITE_HLA, x=h.to(dev), E_main=E.to(dev), E_1=E1.to(dev), out0=lat,
                            out1=lat1, r_k=r_k, d_h=d_h, pos0=pos0, rotate_keys=False)
        torch.cuda.synchronize()
        for b in range(B):
            c, c1 = hla.write(f64(h[b]), f64(E), f64(E1), pos0, r_k, r_v, r_1, d_h, BASE, rotate_keys=False)
            exp = quant.row_bytes(*quant.quantize_rows(c, r_k, r_v))
            exp1 = quant.row_bytes(*quant.quantize_rows(c1, r_1, r_1))
            assert np.array_equal(lat[b, pos0:pos0 + n].cpu().numpy(), exp)
            assert np.array_equal(lat1[b, pos0:pos0 + n].cpu().numpy(), exp1)
            assert torch.all(lat[b, :pos0] == 0xAB) and torch.all(lat[b, pos0 + n:] == 0xAB)
    else:
        H, d_h, r_k, r_v = 3, 32, 48, 80
        k = _int_tensor(g, (B, n, T, H, d_h), -2, 2)
        v = _int_tensor(g, (B, n, T, H, d_h), -2, 2)
        EK = _int_tensor(g, (T, H, r_k, d_h), -1, 1) * (torch.rand(T, H, r_k, d_h, generator=g) < 0.2)
        EV = _int_tensor(g, (T, H, r_v, d_h), -1, 1) * (torch.rand(T, H, r_v, d_h, generator=g) < 0.2)
        lat = torch.full((B, Ncap, r_k + r_v + 16), 0xAB, dtype=torch.uint8, device=dev)
        L.lla_write_latents(L.LLA_WRITE_FOLDED, x=k.to(dev), xv=v.to(dev), E_K=EK.to(dev), E_V=EV.to(dev),
                            out0=lat, pos0=pos0)
        torch.cuda.synchronize()
        for b in range(B):
            c = lla.write_folded(f64(k[b]), f64(v[b]), f64(EK), f64(EV))
            exp = quant.row_bytes(*quant.quantize_rows(c, r_k, r_v))
            assert np.array_equal(lat[b, pos0:pos0 + n].cpu().numpy(), exp)


def test_fp8_writer_rotated_rows_within_one_step(cuda_device):
    """Random inputs with rotation: fp32 summation order can move a quotient
    across an e4m3 rounding boundary, so each stored value must lie within one
    e4m3 step (relative 2^-3, or 2^-9 of the scale) of the oracle's value, at
    least 98 % of the codes must equal the oracle's, and the scales must agree
    within 1e-5 relative."""
    g = _gen(31)
    dev = cuda_device
    B, n, T, D, r_k, r_v, r_1, d_h = 2, 40, 4, 128, 64, 64, 32, 32
    h = torch.randn(B, n, T, D, generator=g)
    E = torch.randn(T - 1, r_k + r_v, D, generator=g) / math.sqrt(D)
    E1 = torch.randn(2 * r_1, D, generator=g) / math.sqrt(D)
    pos0 = 500
    lat = torch.zeros(B, pos0 + n, r_k + r_v + 16, dtype=torch.uint8, device=dev)
    lat1 = torch.zeros(B, pos0 + n, 2 * r_1 + 16, dtype=torch.uint8, device=dev)
    L.lla_write_latents(L.LLA_WRITE_HLA, x=h.to(dev), E_main=E.to(dev), E_1=E1.to(dev), out0=lat, out1=lat1,
                        r_k=r_k, d_h=d_h, pos0=pos0, rope_base=BASE)
    torch.cuda.synchronize()
    for b in range(B):
        c, c1 = hla.write(f64(h[b]), f64(E), f64(E1), pos0, r_k, r_v, r_1, d_h, BASE)
        for got_rows, exact, rk, rv in ((lat[b, pos0:], c, r_k, r_v), (lat1[b, pos0:], c1, r_1, r_1)):
            got_rows = got_rows.cpu().numpy()
            codes, sK, sV = quant.quantize_rows(exact, rk, rv)
            w = rk + rv
            gK = got_rows[:, w:w + 4].copy().view(np.float32)[:, 0]
            gV = got_rows[:, w + 4:w + 8].copy().view(np.float32)[:, 0]
            dK = np.max(np.abs(gK / sK - 1)) if np.all(sK > 0) else np.inf
            dV = np.max(np.abs(gV / sV - 1)) if np.all(sV > 0) else np.inf
            assert dK <= 1e-5 and dV <= 1e-5, f"scales off by {dK:.2e} / {dV:.2e} (rk {rk})"
            got = quant.from_row_bytes(got_rows, rk, rv)
            ref = quant.dequantize_rows(codes, sK, sV, rk)
            s = np.concatenate([np.repeat(sK[:, None], rk, 1), np.repeat(sV[:, None], rv, 1)], 1)
            viol = np.abs(got - ref) - (2.0 ** -3 * np.abs(ref) + s * 2.0 ** -9 + 1e-12)
            # the codes themselves (the scales differ in their last bits, so the
            # dequantised values are compared by the bound above only)
            frac_eq = np.mean(got_rows[:, :w] == quant.e4m3_bits(codes))
            assert np.all(viol <= 0), (f"rk {rk}: {np.sum(viol > 0)} values beyond one step, worst "
                                       f"{np.max(viol):.3e}")
            assert frac_eq > 0.98, f"rk {rk}: equal code fraction {frac_eq:.4f}"


FP8_READS = [
    # B, N, W, H, nt, d_h, r_k, r_v, Wcap, rotate
    (2, 700, 128, 16, 3, 128, 512, 512, 129, True),    # Ouro-shaped main latent, 48 rows
    (2, 650, 128, 16, 1, 128, 256, 256, 129, True),    # Ouro-shaped loop-1 latent, 16 rows
    (1, 1100, 0, 16, 4, 128, 576, 576, 1, False),      # LLA-2D-shaped, 64 rows, no window
    (3, 301, 16, 4, 3, 64, 128, 192, 17, True),        # ragged tail, odd value chunk count
    (2, 300, 0, 4, 2, 64, 64, 64, 1, False),           # one score chain and one value chain, 8 rows
    (1, 520, 0, 16, 4, 128, 768, 768, 1, False),       # widest rows: one slot per ring, 64 rows
]


@pytest.mark.parametrize("case", FP8_READS)
def test_fp8_read_matches_oracle(cuda_device, case):
    B, N, W, H, nt, d_h, r_k, r_v, Wcap, rotate = case
    g = _gen(40 + N)
    t0 = 1 if rotate else 0
    T = t0 + nt
    rows = synth.random_fp8_rows(B, N, r_k, r_v, 41 + N)
    A = torch.randn(nt, H, d_h, r_k, generator=g) / math.sqrt(d_h)
    Bm = torch.randn(nt, H, r_v, d_h, generator=g) / math.sqrt(r_v)
    q = torch.randn(B, nt, H, d_h, generator=g)
    wk = torch.randn(B, T, Wcap, H, d_h, generator=g).to(torch.bfloat16)
    wv = torch.randn(B, T, Wcap, H, d_h, generator=g).to(torch.bfloat16)
    dev = cuda_device
    out = torch.full((B, nt, H, d_h), float("nan"), device=dev)
    L.hla_decode_attn(lat=rows.to(dev), A=A.to(dev), Bm=Bm.to(dev), q=q.to(dev), win_k=wk.to(dev),
                      win_v=wv.to(dev), out=out, N=N, W=W, t0=t0, rotate_query=rotate, rope_base=BASE)
    torch.cuda.synchronize()
    ref = []
    for b in range(B):
        vals = quant.from_row_bytes(rows[b].numpy(), r_k, r_v)
        ref.append(hla.decode(vals, f64(A), f64(Bm), f64(q[b]), f64(wk[b]), f64(wv[b]), t0, N, W, r_k, r_v,
                              d_h, BASE, rotate_query=rotate))
    err = assert_rows_close(out, np.stack(ref), TOL, f"fp8 read {case}")
    print(f"fp8 read {case}: rel L2 (pooled, worst row) {err}")


def test_fp8_lla2d_writer_then_read(cuda_device):
    """LLA-2D end to end with fp8 rows: the folded writer quantises on the GPU,
    the absorbed read reads the bytes; the oracle writes, quantises and reads."""
    g = _gen(61)
    B, T, H, d_h, rK, rV, N = 2, 2, 4, 32, 128, 128, 300
    k = torch.randn(B, N, T, H, d_h, generator=g)
    v = torch.randn(B, N, T, H, d_h, generator=g)
    EK = torch.randn(T, H, rK, d_h, generator=g) / math.sqrt(T * H * d_h)
    EV = torch.randn(T, H, rV, d_h, generator=g) / math.sqrt(T * H * d_h)
    UK = torch.randn(T, H, d_h, rK, generator=g) / math.sqrt(rK)
    UV = torch.randn(T, H, d_h, rV, generator=g) / math.sqrt(rV)
    q = torch.randn(B, T, H, d_h, generator=g)
    wk = k[:, N - 1].reshape(B, T, 1, H, d_h)
    wv = v[:, N - 1].reshape(B, T, 1, H, d_h)
    dev = cuda_device
    lat = torch.zeros(B, N, rK + rV + 16, dtype=torch.uint8, device=dev)
    L.lla_write_latents(L.LLA_WRITE_FOLDED, x=k.to(dev), xv=v.to(dev), E_K=EK.to(dev), E_V=EV.to(dev),
                        out0=lat, pos0=0)
    out = torch.empty(B, T, H, d_h, device=dev)
    L.hla_decode_attn(lat=lat, A=UK.to(dev), Bm=UV.transpose(2, 3).contiguous().to(dev), q=q.to(dev),
                      win_k=wk.to(torch.bfloat16).to(dev), win_v=wv.to(torch.bfloat16).to(dev), out=out,
                      N=N, W=0, t0=0, rotate_query=False)
    torch.cuda.synchronize()
    ref = []
    for b in range(B):
        c = lla.write_folded(f64(k[b]), f64(v[b]), f64(EK), f64(EV))
        rows = quant.to_storage_fp8(c, rK, rV)
        ref.append(lla.decode_absorbed(rows, f64(UK), f64(UV), f64(q[b]), f64(wk[b].to(torch.bfloat16)),
                                       f64(wv[b].to(torch.bfloat16)), 0, N, 0, rK, rV))
    err = assert_rows_close(out, np.stack(ref), TOL, "fp8 LLA-2D end to end")
    print(f"fp8 LLA-2D end to end: rel L2 (pooled, worst row) {err}")
