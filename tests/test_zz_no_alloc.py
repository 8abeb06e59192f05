"""hla_decode_attn_noalloc: the absorbed read for callers that cannot allocate
device memory (a plugin handed only input/output buffers, or an engine that has
reserved all device memory for its cache).  It takes no workspace; its scratch
is a static device array inside the library.  Its output must match the
workspace entry point, hla_decode_attn, on the same inputs bit for bit (both
run the same deterministic kernels; only the scratch address differs) --
checked on three calls in a row with different inputs, so that anything one
call leaves in the shared scratch cannot leak into the next: a SIMT-read case,
then a tensor-core case with 48 query rows and r_k = 512, then a tensor-core
case with fewer rows (16) and a smaller r_k (128), whose query operand and split
partials occupy less of the scratch than the previous call left behind.

This file is collected last (its name sorts after the other test files), so a
run that stops at the first failure has already run every other test.
"""

import ctypes
import math

import pytest
import torch

import looped_transformer_latent_b200 as L
from looped_transformer_latent_b200 import _abi

pytestmark = pytest.mark.gpu


def _case(seed, B, N, W, H, nt, d_h, r_k, r_v, Wcap, dev):
    g = torch.Generator().manual_seed(seed)
    t0 = 1
    T = t0 + nt
    c = dict(
        lat=(torch.randn(B, N, r_k + r_v, generator=g) * math.sqrt(d_h / r_k)).to(torch.bfloat16),
        A=torch.randn(nt, H, d_h, r_k, generator=g) / math.sqrt(d_h),
        Bm=torch.randn(nt, H, r_v, d_h, generator=g) / math.sqrt(r_v),
        q=torch.randn(B, nt, H, d_h, generator=g),
        win_k=torch.randn(B, T, Wcap, H, d_h, generator=g).to(torch.bfloat16),
        win_v=torch.randn(B, T, Wcap, H, d_h, generator=g).to(torch.bfloat16),
    )
    c = {k: v.to(dev) for k, v in c.items()}
    c.update(N=N, W=W, t0=t0)
    return c


def _noalloc(case, out):
    """Call the no-allocation entry point through the C ABI."""
    p = L._hla_params(lat=case["lat"], A=case["A"], Bm=case["Bm"], q=case["q"],
                      win_k=case["win_k"], win_v=case["win_v"], out=out, N=case["N"],
                      W=case["W"], t0=case["t0"], r_k=None, rotate_query=True,
                      rope_base=10000.0, scale=0.0)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.lib().hla_decode_attn_noalloc(ctypes.byref(p), stream)


def _with_workspace(case, out):
    L.hla_decode_attn(lat=case["lat"], A=case["A"], Bm=case["Bm"], q=case["q"],
                      win_k=case["win_k"], win_v=case["win_v"], out=out, N=case["N"],
                      W=case["W"], t0=case["t0"])


def test_noalloc_matches_workspace_entry_point_on_three_calls(cuda_device):
    first = _case(11, 3, 301, 16, 4, 3, 64, 128, 96, 17, cuda_device)       # SIMT read (r_v = 96)
    second = _case(12, 2, 700, 128, 16, 3, 128, 512, 512, 129, cuda_device)  # tensor cores, 48 rows
    third = _case(14, 3, 500, 16, 8, 2, 128, 128, 256, 17, cuda_device)      # tensor cores, 16 rows
    for case in (first, second, third):
        ref = torch.empty(tuple(case["q"].shape), device=cuda_device)
        got = torch.full(tuple(case["q"].shape), float("nan"), device=cuda_device)
        _with_workspace(case, ref)
        assert _noalloc(case, got) == _abi.LLA_OK
        torch.cuda.synchronize()
        assert torch.isfinite(got).all()
        assert torch.equal(got, ref)


def test_noalloc_refuses_problems_larger_than_its_scratch(cuda_device):
    # Needs far more than the static scratch: rejected before any launch.
    case = _case(13, 2, 40, 8, 2, 1, 64, 64, 64, 9, cuda_device)
    p = L._hla_params(lat=case["lat"], A=case["A"], Bm=case["Bm"], q=case["q"],
                      win_k=case["win_k"], win_v=case["win_v"],
                      out=torch.empty(tuple(case["q"].shape), device=cuda_device),
                      N=case["N"], W=case["W"], t0=case["t0"], r_k=None, rotate_query=True,
                      rope_base=10000.0, scale=0.0)
    p.B = 200000
    p.q_stride_b = p.out_stride_b = 128
    need = L.lib().hla_decode_workspace_bytes(ctypes.byref(p))
    assert need > _abi.NOALLOC_SCRATCH_BYTES
    st = L.lib().hla_decode_attn_noalloc(ctypes.byref(p), None)
    assert st == _abi.LLA_ERR_WORKSPACE
