"""The exact decode step the benchmark times, checked against the oracle.

bench.py builds each workload from writer-produced latents: synthetic hidden
states (HLA) or per-loop keys and values (LLA-2D) with a low-rank loop
trajectory, encoded by the SVD codecs of synth.hla_codec /
synth.lla_folded_codec through lla_write_latents.  These tests build that same
step object, run it once exactly as the benchmark's captured graph does (all
layers, the M1 two-stream schedule for HLA), and compare sampled sequences
with the oracle row by row.

The oracle never sees a value the CUDA path produced: it regenerates the
sequence's prefill inputs from the same seeded generator, writes its own
latents (eq. 2 for HLA, the folded encoder for LLA-2D), rounds them to bf16
(the storage format) and reads them with its own decode.  The GPU latents are
compared with the oracle's too.  Tolerance: 2e-2 relative L2 for bf16 latents,
pooled and per (loop, head) row, plus the per-element bound of parity_check.
"""

import numpy as np
import pytest
import torch

import bench
import synth
from oracle import hla, lla, quant, rounding
from parity_check import assert_rows_close

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def _run_eager(step, dev):
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))   # the prefill ran on the current stream
    with torch.cuda.stream(s):
        step.run()
    torch.cuda.synchronize()


def test_ouro_hla_4k_bench_step_matches_oracle(cuda_device):
    c = synth.CONFIGS["ouro_hla_4k"]
    step = bench.HlaStep(c, cuda_device, "m1")
    _run_eager(step, cuda_device)
    cod = {k: v.double().numpy() for k, v in step.codec_host.items()}
    n_lat = c.N - 1 - c.W
    for b in (0, 13, c.B - 1):
        h = step.prefill_hidden(b).double().numpy()
        lat, lat1 = hla.write(h, cod["E_main"], cod["E_1"], 0, c.r_k, c.r_v, c.r_1, c.d_h, c.base)
        lat, lat1 = rounding.to_bf16(lat), rounding.to_bf16(lat1)
        lay0 = step.layers[0]
        # the GPU writer's rows (read by the decode below) against the oracle's
        assert_rows_close(lay0["lat"][b, :n_lat], lat[:n_lat], 1e-2, f"sequence {b} main latent rows")
        assert_rows_close(lay0["lat1"][b, :n_lat], lat1[:n_lat], 1e-2, f"sequence {b} loop-1 latent rows")
        for layer in (0, c.L - 1):
            lay = step.layers[layer]
            q, wk, wv = f64(lay["q"][b]), f64(lay["wk"][b]), f64(lay["wv"][b])
            o1 = hla.decode(lat1, cod["A_1"], cod["B_1"], q[:1], wk, wv, 0, c.N, c.W, c.r_1, c.r_1,
                            c.d_h, c.base)
            om = hla.decode(lat, cod["A"], cod["Bm"], q[1:], wk, wv, 1, c.N, c.W, c.r_k, c.r_v,
                            c.d_h, c.base)
            err = assert_rows_close(lay["out"][b], np.concatenate([o1, om]), TOL_BF16,
                                    f"layer {layer} sequence {b}")
            print(f"ouro_hla_4k bench step, layer {layer} sequence {b}: rel L2 (pooled, worst row) {err}")


def test_ouro_lla2d_768_bench_step_matches_oracle(cuda_device):
    c = synth.CONFIGS["ouro_lla2d_768"]
    step = bench.Lla2dStep(c, cuda_device, "m1")
    _run_eager(step, cuda_device)
    cod = {k: v.double().numpy() for k, v in step.codec_host.items()}
    n_lat = c.N - 1
    for b in (0, 400, c.B - 1):
        k, v = step.prefill_kv(b)
        lat = rounding.to_bf16(lla.write_folded(k.double().numpy(), v.double().numpy(), cod["E_K"], cod["E_V"]))
        assert_rows_close(step.layers[0]["lat"][b, :n_lat], lat, 1e-2, f"sequence {b} latent rows")
        for layer in (0, c.L - 1):
            lay = step.layers[layer]
            out = lla.decode_absorbed(lat, cod["U_K"], cod["U_V"], f64(lay["q"][b]), f64(lay["wk"][b]),
                                      f64(lay["wv"][b]), 0, c.N, 0, c.r_k, c.r_v)
            err = assert_rows_close(lay["out"][b], out, TOL_BF16, f"layer {layer} sequence {b}")
            print(f"ouro_lla2d_768 bench step, layer {layer} sequence {b}: rel L2 (pooled, worst row) {err}")


def test_ouro_lla2d_768_fp8_bench_step_matches_oracle(cuda_device):
    """The fp8-row variant of the gate step: the GPU writer quantises its rows
    (e4m3 codes, per-token scales); the oracle quantises its own fp64 rows and
    reads those.  The codes are compared byte for byte (a code may differ by
    one step where the exact value sits on a rounding boundary, so 98 % equal
    is required) and the outputs at the bf16 tolerance."""
    c = synth.CONFIGS["ouro_lla2d_768_fp8"]
    step = bench.Lla2dStep(c, cuda_device, "m1")
    _run_eager(step, cuda_device)
    cod = {k: v.double().numpy() for k, v in step.codec_host.items()}
    n_lat, w = c.N - 1, c.r_k + c.r_v
    for b in (0, 400, c.B - 1):
        k, v = step.prefill_kv(b)
        exact = lla.write_folded(k.double().numpy(), v.double().numpy(), cod["E_K"], cod["E_V"])
        codes, sK, sV = quant.quantize_rows(exact, c.r_k, c.r_v)
        got = step.layers[0]["lat"][b, :n_lat].cpu().numpy()
        frac_eq = np.mean(got[:, :w] == quant.e4m3_bits(codes))
        assert frac_eq > 0.98, f"sequence {b}: equal code fraction {frac_eq:.4f}"
        rows = quant.dequantize_rows(codes, sK, sV, c.r_k)
        for layer in (0, c.L - 1):
            lay = step.layers[layer]
            out = lla.decode_absorbed(rows, cod["U_K"], cod["U_V"], f64(lay["q"][b]), f64(lay["wk"][b]),
                                      f64(lay["wv"][b]), 0, c.N, 0, c.r_k, c.r_v)
            err = assert_rows_close(lay["out"][b], out, TOL_BF16, f"layer {layer} sequence {b}")
            print(f"ouro_lla2d_768_fp8 bench step, layer {layer} sequence {b}: rel L2 (pooled, worst row) {err}")
