"""Programmatic dependent launch (LLA_PDL=1) must not change any result.

With the attribute every kernel may be scheduled while its predecessor on
the stream drains and waits (griddepcontrol.wait) before touching global
memory.  The same writer-then-read sequences run in two child processes,
one with LLA_PDL=1 and one with LLA_PDL=0 (the switch is read once per
process), and their outputs must be bit-identical: the tensor-core read of
bf16 and fp8 rows, the window, the maps and the writer all take part.
"""

import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import math, sys
import numpy as np
import torch
sys.path.insert(0, sys.argv[1])
import looped_transformer_latent_b200 as L
dev = torch.device("cuda", 0)
g = torch.Generator().manual_seed(5)
outs = []
for fp8 in (False, True):
    B, n, T, H, d_h, r = 3, 700, 4, 16, 128, 256
    k = torch.randn(B, n, T, H, d_h, generator=g)
    v = torch.randn(B, n, T, H, d_h, generator=g)
    EK = torch.randn(T, H, r, d_h, generator=g) / math.sqrt(T * H * d_h)
    EV = torch.randn(T, H, r, d_h, generator=g) / math.sqrt(T * H * d_h)
    UK = torch.randn(T, H, d_h, r, generator=g) / math.sqrt(r)
    UV = torch.randn(T, H, d_h, r, generator=g) / math.sqrt(r)
    q = torch.randn(B, T, H, d_h, generator=g)
    W = 16
    wk = torch.randn(B, T, W + 1, H, d_h, generator=g).to(torch.bfloat16)
    wv = torch.randn(B, T, W + 1, H, d_h, generator=g).to(torch.bfloat16)
    if fp8:
        lat = torch.zeros(B, n, 2 * r + 16, dtype=torch.uint8, device=dev)
    else:
        lat = torch.zeros(B, n, 2 * r, dtype=torch.bfloat16, device=dev)
    s = torch.cuda.Stream(dev)
    with torch.cuda.stream(s):
        L.lla_write_latents(L.LLA_WRITE_FOLDED, x=k.to(dev), xv=v.to(dev), E_K=EK.to(dev), E_V=EV.to(dev),
                            out0=lat, pos0=0, stream=s)
        out = torch.empty(B, T, H, d_h, device=dev)
        for _ in range(3):   # back-to-back calls: each kernel follows another of this library
            L.hla_decode_attn(lat=lat, A=UK.to(dev), Bm=UV.transpose(2, 3).contiguous().to(dev), q=q.to(dev),
                              win_k=wk.to(dev), win_v=wv.to(dev), out=out, N=n, W=W, t0=0, rotate_query=False,
                              stream=s)
    torch.cuda.synchronize()
    outs += [lat.view(torch.uint8).cpu().numpy(), out.cpu().numpy()]
np.savez(sys.argv[2], *outs)
'''


def _run(tmp_path, pdl):
    f = tmp_path / f"out_pdl{pdl}.npz"
    env = dict(os.environ, LLA_PDL=str(pdl))
    subprocess.run([sys.executable, "-c", CHILD, ROOT, str(f)], env=env, check=True, timeout=600)
    d = np.load(f)
    return [d[k] for k in sorted(d.files, key=lambda s: int(s.split("_")[1]))]


def test_pdl_outputs_bit_identical(cuda_device, tmp_path):
    on, off = _run(tmp_path, 1), _run(tmp_path, 0)
    assert len(on) == len(off) == 4
    for a, b in zip(on, off):
        assert a.shape == b.shape
        assert np.array_equal(a.view(np.uint8), b.view(np.uint8))
    assert np.all(np.isfinite(on[1])) and np.all(np.isfinite(on[3]))
