"""The C ABI library loads, exports every declared symbol, and validates its
arguments on the host (no GPU needed: invalid calls return before any CUDA
call)."""

import ctypes
import os
import re

import pytest

import looped_transformer_latent_b200 as L
from looped_transformer_latent_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from looped_transformer_latent_b200 import build
    build.build()
    return _abi.load()


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "lla.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return set(re.findall(r"\b([a-z_][a-z0-9_]*)\s*\([^;{]*\)\s*;", src))


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for n in ["lla_write_latents", "lla_decode_attn", "hla_decode_attn", "lla_status_str",
              "lla_write_workspace_bytes", "lla_decode_workspace_bytes",
              "hla_decode_workspace_bytes", "lla_abi_version", "lla_last_cuda_error", "lla_cuda_error_name"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert names, "no declarations parsed"
    for n in names:
        assert hasattr(lib, n), f"liblla.so does not export {n}"
    assert set(_abi.PROTOTYPES) >= names - set(), "binding lacks a prototype"


def test_status_strings(lib):
    for s in range(8):
        assert L.lla_status_str(s) != "unknown status"
    assert L.lla_status_str(99) == "unknown status"
    assert L.lla_abi_version() >= 1
    assert L.lib().lla_last_cuda_error() == 0
    assert L.lib().lla_cuda_error_name(0).decode() == "cudaSuccess"


def test_struct_sizes_match_c_layout(lib):
    # offsets of the last field: any mismatch with the header shows up here
    assert ctypes.sizeof(_abi.WriteParams) == _abi.WriteParams.out1_stride_n.offset + 8
    assert _abi.WriteParams.rope_base.offset == 48
    assert _abi.HlaDecodeParams.rope_base.offset % 8 == 0


def _hla(**over):
    p = _abi.HlaDecodeParams()
    vals = dict(B=2, H=2, d_h=64, T=4, t0=1, nt=3, N=100, W=16, r_k=128, r_v=128,
                lat=0x10000, lat_dtype=1, lat_stride_b=100 * 256, lat_stride_n=256,
                A=0x20000, Bm=0x30000, q=0x40000, q_stride_b=3 * 2 * 64, rotate_query=1,
                rope_base=10000.0, win_k=0x50000, win_v=0x60000, win_dtype=1, Wcap=17,
                win_stride_b=4 * 17 * 2 * 64, out=0x70000, out_stride_b=3 * 2 * 64, scale=0.0)
    vals.update(over)
    for k, v in vals.items():
        setattr(p, k, v)
    return p


def _call_hla(lib, p, ws=0x100000, nbytes=1 << 30):
    return lib.hla_decode_attn(ctypes.byref(p), ctypes.c_void_p(ws), nbytes, None)


@pytest.mark.parametrize("over,status", [
    (dict(lat=0), _abi.LLA_ERR_NULL),
    (dict(A=0), _abi.LLA_ERR_NULL),
    (dict(out=0), _abi.LLA_ERR_NULL),
    (dict(win_stream=0x1234), _abi.LLA_ERR_NULL),  # a window stream needs its fork/join events
    (dict(lat_dtype=7), _abi.LLA_ERR_DTYPE),
    (dict(win_dtype=-1), _abi.LLA_ERR_DTYPE),
    (dict(t0=2), _abi.LLA_ERR_SHAPE),            # t0 + nt > T
    (dict(N=0), _abi.LLA_ERR_SHAPE),
    (dict(W=-1), _abi.LLA_ERR_SHAPE),
    (dict(Wcap=16), _abi.LLA_ERR_SHAPE),          # ring smaller than W+1
    (dict(r_k=127), _abi.LLA_ERR_SHAPE),          # odd rank has no rotary pairs
    (dict(d_h=256), _abi.LLA_ERR_UNSUPPORTED),
    (dict(lat=0x10008), _abi.LLA_ERR_ALIGN),
    (dict(lat_stride_n=260), _abi.LLA_ERR_ALIGN),
    (dict(q_stride_b=10), _abi.LLA_ERR_SHAPE),
    (dict(scale=-1.0), _abi.LLA_ERR_SHAPE),
])
def test_hla_validation(lib, over, status):
    assert _call_hla(lib, _hla(**over)) == status


def test_hla_workspace_checks(lib):
    p = _hla()
    need = lib.hla_decode_workspace_bytes(ctypes.byref(p))
    assert need > 0
    assert _call_hla(lib, p, ws=0, nbytes=need) == _abi.LLA_ERR_WORKSPACE
    assert _call_hla(lib, p, ws=0x100000, nbytes=need - 1) == _abi.LLA_ERR_WORKSPACE
    assert _call_hla(lib, p, ws=0x100010, nbytes=need) == _abi.LLA_ERR_WORKSPACE  # misaligned
    assert lib.hla_decode_workspace_bytes(ctypes.byref(_hla(N=0))) == 0


def test_read_split_override_sizes_the_workspace(lib, monkeypatch):
    # LLA_READ_SPLITS fixes the latent read's context splits: each split keeps
    # (max, sum) and an r_V-wide partial per (sequence, row) in fp32, and the
    # count is capped at one 64-token tile per split (here 83 latent tokens: 2)
    p = _hla()
    rows = p.nt * p.H
    per_split = p.B * rows * p.r_v * 4      # the r_V-wide partials (the (max, sum) pairs share an aligned block)
    need = {}
    for v in ("1", "2", "50"):
        monkeypatch.setenv("LLA_READ_SPLITS", v)
        need[v] = lib.hla_decode_workspace_bytes(ctypes.byref(p))
    monkeypatch.delenv("LLA_READ_SPLITS")
    assert need["2"] - need["1"] >= per_split
    assert need["50"] == need["2"]
    assert lib.hla_decode_workspace_bytes(ctypes.byref(p)) > 0


def test_empty_batch_is_a_no_op(lib):
    # B = 0 or nt = 0: nothing to do, null pointers allowed, no workspace
    p = _hla(B=0, lat=0, A=0, Bm=0, q=0, win_k=0, win_v=0, out=0)
    assert lib.hla_decode_attn(ctypes.byref(p), None, 0, None) == _abi.LLA_OK
    p = _hla(nt=0, lat=0, A=0, Bm=0, q=0, win_k=0, win_v=0, out=0)
    assert lib.hla_decode_attn(ctypes.byref(p), None, 0, None) == _abi.LLA_OK


def test_null_params(lib):
    assert lib.hla_decode_attn(None, None, 0, None) == _abi.LLA_ERR_NULL
    assert lib.lla_decode_attn(None, None, 0, None) == _abi.LLA_ERR_NULL
    assert lib.lla_write_latents(None, None, 0, None) == _abi.LLA_ERR_NULL
    assert lib.hla_decode_workspace_bytes(None) == 0


def _lla(**over):
    p = _abi.LlaDecodeParams()
    vals = dict(B=2, H=3, d_h=32, r=32, T=4, t0=0, nt=4, N=50, W=0, cK=0x10000, cV=0x20000,
                lat_dtype=1, lat_stride_b=3 * 64 * 32, lat_stride_h=64 * 32, UK=0x30000,
                UV=0x40000, q=0x50000, q_stride_b=4 * 3 * 32, win_k=0x60000, win_v=0x70000,
                win_dtype=1, Wcap=1, win_stride_b=4 * 1 * 3 * 32, out=0x80000,
                out_stride_b=4 * 3 * 32, scale=0.0)
    vals.update(over)
    for k, v in vals.items():
        setattr(p, k, v)
    return p


@pytest.mark.parametrize("over,status", [
    (dict(cK=0), _abi.LLA_ERR_NULL),
    (dict(UV=0), _abi.LLA_ERR_NULL),
    (dict(lat_dtype=3), _abi.LLA_ERR_DTYPE),
    (dict(nt=5), _abi.LLA_ERR_SHAPE),
    (dict(r=256), _abi.LLA_ERR_UNSUPPORTED),
    (dict(lat_stride_h=10), _abi.LLA_ERR_ALIGN),
    (dict(lat_stride_h=40 * 32), _abi.LLA_ERR_SHAPE),   # fewer rows than latent tokens
    (dict(Wcap=0), _abi.LLA_ERR_SHAPE),
])
def test_lla_validation(lib, over, status):
    p = _lla(**over)
    assert lib.lla_decode_attn(ctypes.byref(p), ctypes.c_void_p(0x100000), 1 << 30, None) == status


def _write(**over):
    p = _abi.WriteParams()
    vals = dict(mode=0, B=2, n=5, pos0=3, T=4, H=2, d_h=64, D=128, r_k=128, r_v=128, r_1=32,
                rotate_keys=1, rope_base=10000.0, x=0x10000, xv=0, x_stride_b=5 * 4 * 128,
                x_stride_n=4 * 128, x_stride_t=128, E_main=0x20000, E_1=0x30000, E_K=0, E_V=0,
                out0=0x40000, out1=0x50000, out_dtype=1, Ncap=16, out_stride_b=16 * 256,
                out_stride_h=0, out_stride_n=256, out1_stride_b=16 * 64, out1_stride_n=64)
    vals.update(over)
    for k, v in vals.items():
        setattr(p, k, v)
    return p


@pytest.mark.parametrize("over,status", [
    (dict(E_1=0), _abi.LLA_ERR_NULL),
    (dict(mode=9), _abi.LLA_ERR_UNSUPPORTED),
    (dict(out_dtype=5), _abi.LLA_ERR_DTYPE),
    (dict(pos0=12), _abi.LLA_ERR_SHAPE),          # pos0 + n > Ncap
    (dict(D=100), _abi.LLA_ERR_SHAPE),
    (dict(T=1), _abi.LLA_ERR_SHAPE),               # eq. 2 needs loops 2..T
    (dict(r_k=130), _abi.LLA_ERR_ALIGN),           # bf16 row of 258 is not 16-byte sized
    (dict(out0=0x40004), _abi.LLA_ERR_ALIGN),
])
def test_write_validation(lib, over, status):
    p = _write(**over)
    assert lib.lla_write_latents(ctypes.byref(p), ctypes.c_void_p(0x100000), 1 << 30, None) == status


def test_write_workspace(lib):
    p = _write()
    need = lib.lla_write_workspace_bytes(ctypes.byref(p))
    assert need > 0 and need % 256 == 0
    assert lib.lla_write_latents(ctypes.byref(p), None, 0, None) == _abi.LLA_ERR_WORKSPACE


def test_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros(1, 2, 4, 128)
    with pytest.raises(ValueError, match="CUDA"):
        L.lla_write_latents(L.LLA_WRITE_HLA, x=x, E_main=torch.zeros(3, 256, 128),
                            E_1=torch.zeros(64, 128), out0=torch.zeros(1, 4, 256),
                            out1=torch.zeros(1, 4, 64), r_k=128, d_h=64)
