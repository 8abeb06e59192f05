"""B200-native decode-time latent attention for looped (weight-tied) Transformers.

Thin Python binding over the C ABI in ``include/lla.h`` (``liblla.so``): the
functions below only turn torch tensors into pointers, sizes and strides and
call the library entry points of the same names.  Every step of the
computation runs in the library's CUDA kernels; there is no CPU path.  Tensors
must be CUDA tensors; PyTorch provides device memory and streams only.

Entry points (names as in the C ABI):

* ``lla_write_latents``  -- HLA latent writer (eq. 2), LLA per-head and LLA-2D
  encoders; appends rows to a caller-owned latent cache.
* ``lla_decode_attn``    -- LLA reconstruct-on-read decode attention.
* ``hla_decode_attn``    -- absorbed latent read: HLA (eqs. 3-4) and LLA-D.
"""

import ctypes

from . import _abi
from ._abi import (LLA_BF16, LLA_ERR_CUDA, LLA_F32, LLA_FP8_E4M3, LLA_WRITE_FOLDED, LLA_WRITE_HLA,  # noqa: F401
                   LLA_WRITE_PERHEAD, LibraryMissing)

__all__ = [
    "LLAError", "lla_status_str", "lla_abi_version",
    "lla_write_latents", "lla_write_workspace_bytes",
    "lla_decode_attn", "lla_decode_workspace_bytes",
    "hla_decode_attn", "hla_decode_workspace_bytes",
    "LLA_WRITE_HLA", "LLA_WRITE_PERHEAD", "LLA_WRITE_FOLDED",
]


class LLAError(RuntimeError):
    """A non-zero lla_status returned by the library."""

    def __init__(self, status, where):
        self.status = status
        msg = f"{where}: status {status} ({lla_status_str(status)})"
        self.cuda_error = None
        if status == LLA_ERR_CUDA:
            self.cuda_error = lib().lla_last_cuda_error()
            msg += f": {lib().lla_cuda_error_name(self.cuda_error).decode()} ({self.cuda_error})"
        super().__init__(msg)


def lib():
    return _abi.load()


def lla_status_str(status):
    return lib().lla_status_str(int(status)).decode()


def lla_abi_version():
    return lib().lla_abi_version()


# ---------------------------------------------------------------- helpers --
def _torch():
    import torch
    return torch


def _dtype_code(t):
    torch = _torch()
    if t.dtype == torch.float32:
        return LLA_F32
    if t.dtype == torch.bfloat16:
        return LLA_BF16
    if t.dtype == torch.uint8:
        return LLA_FP8_E4M3          # byte rows: e4m3 codes, then the two fp32 scales and 8 zero bytes
    raise TypeError(f"unsupported dtype {t.dtype}; use float32, bfloat16 or uint8 (fp8 rows)")


FP8_ROW_EXTRA = 16   # bytes after the codes of an fp8 row: s^K, s^V (fp32), 8 zero bytes


def _row_width(t):
    """Elements of one latent row: the codes only, for fp8 byte rows."""
    return t.shape[-1] - (FP8_ROW_EXTRA if t.dtype == _torch().uint8 else 0)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _cuda(*ts):
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("every tensor must be a CUDA tensor (this library has no CPU path)")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError("tensors are on different devices")
    if dev is None:
        raise ValueError("no tensor given")
    return dev


def _dense_inner(t, ndim_inner, name):
    """Check that the last ``ndim_inner`` axes of t are dense row-major."""
    exp = 1
    for ax in range(t.dim() - 1, t.dim() - 1 - ndim_inner, -1):
        if t.shape[ax] != 1 and t.stride(ax) != exp:
            raise ValueError(f"{name}: inner axes must be dense (axis {ax} stride {t.stride(ax)}, want {exp})")
        exp *= t.shape[ax]


def _stream_handle(stream, device):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _workspace(nbytes, device, workspace):
    torch = _torch()
    if nbytes == 0:
        return None, 0
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
    if workspace.numel() * workspace.element_size() < nbytes:
        raise ValueError(f"workspace too small: {workspace.numel()} < {nbytes} bytes")
    return ctypes.c_void_p(workspace.data_ptr()), workspace.numel() * workspace.element_size()


def _call(fn, params, ws, nbytes, stream, where):
    st = fn(ctypes.byref(params), ws, nbytes, stream)
    if st != 0:
        raise LLAError(st, where)


# ----------------------------------------------------------------- writer --
def _write_params(mode, x, xv, E_main, E_1, E_K, E_V, out0, out1, pos0, d_h, r_k, r_v, r_1,
                  rotate_keys, rope_base):
    p = _abi.WriteParams()
    p.mode = mode
    p.pos0 = pos0
    p.rope_base = float(rope_base)
    p.rotate_keys = int(bool(rotate_keys))
    if mode == LLA_WRITE_HLA:
        B, n, T, D = x.shape
        _dense_inner(x, 1, "h")
        p.B, p.n, p.T, p.D, p.H, p.d_h = B, n, T, D, 1, d_h
        p.r_k, p.r_v, p.r_1 = r_k, _row_width(out0) - r_k, _row_width(out1) // 2
        p.out_stride_b, p.out_stride_n = out0.stride(0), out0.stride(1)
        p.out1_stride_b, p.out1_stride_n = out1.stride(0), out1.stride(1)
        p.Ncap = min(out0.shape[1], out1.shape[1])
        _dense_inner(out0, 1, "out0")
        _dense_inner(out1, 1, "out1")
    else:
        B, n, T, H, dh = x.shape
        _dense_inner(x, 2, "k")
        _dense_inner(xv, 2, "v")
        if xv.stride() != x.stride() or xv.shape != x.shape:
            raise ValueError("k and v must have the same shape and strides")
        p.B, p.n, p.T, p.H, p.d_h, p.D = B, n, T, H, dh, 0
        if mode == LLA_WRITE_PERHEAD:
            r = out0.shape[-1]
            p.r_k = p.r_v = r
            _dense_inner(out0, 1, "cK")
            _dense_inner(out1, 1, "cV")
            if out1.stride() != out0.stride():
                raise ValueError("cK and cV must share strides")
            p.out_stride_b, p.out_stride_h, p.out_stride_n = out0.stride(0), out0.stride(1), out0.stride(2)
            p.Ncap = out0.shape[2]
        else:
            p.r_k = E_K.shape[2]
            p.r_v = E_V.shape[2]
            _dense_inner(out0, 1, "lat")
            p.out_stride_b, p.out_stride_n = out0.stride(0), out0.stride(1)
            p.Ncap = out0.shape[1]
    p.x, p.xv = _ptr(x), _ptr(xv)
    p.x_stride_b, p.x_stride_n, p.x_stride_t = x.stride(0), x.stride(1), x.stride(2)
    p.E_main, p.E_1, p.E_K, p.E_V = _ptr(E_main), _ptr(E_1), _ptr(E_K), _ptr(E_V)
    p.out0, p.out1 = _ptr(out0), _ptr(out1)
    p.out_dtype = _dtype_code(out0)
    for t in (x, xv, E_main, E_1, E_K, E_V):
        if t is not None and t.dtype != _torch().float32:
            raise TypeError("writer inputs and codecs are float32")
    for t in (E_main, E_1, E_K, E_V):
        if t is not None and not t.is_contiguous():
            raise ValueError("codec tensors must be contiguous")
    return p


def lla_write_workspace_bytes(mode, **kw):
    p = _write_params(mode, **_write_kw(kw))
    return lib().lla_write_workspace_bytes(ctypes.byref(p))


def _write_kw(kw):
    keys = ["x", "xv", "E_main", "E_1", "E_K", "E_V", "out0", "out1", "pos0", "d_h", "r_k",
            "r_v", "r_1", "rotate_keys", "rope_base"]
    d = {k: None for k in keys}
    d.update(pos0=0, d_h=0, r_k=0, r_v=0, r_1=0, rotate_keys=True, rope_base=10000.0)
    unknown = set(kw) - set(keys) - {"workspace", "stream"}
    if unknown:
        raise TypeError(f"unknown arguments {sorted(unknown)}")
    d.update({k: v for k, v in kw.items() if k in keys})
    return d


def lla_write_latents(mode, *, workspace=None, stream=None, **kw):
    """Append latents of n tokens per sequence at rows pos0..pos0+n-1.

    HLA:     x=h [B,n,T,D], E_main [T-1,r_k+r_v,D], E_1 [2r_1,D],
             out0 [B,Ncap,r_k+r_v], out1 [B,Ncap,2r_1], r_k=..., d_h=...
    PERHEAD: x=k, xv=v [B,n,T,H,d_h], E_K, E_V [T,H,r,d_h], out0=cK, out1=cV [B,H,Ncap,r]
    FOLDED:  x=k, xv=v, E_K [T,H,r_K,d_h], E_V [T,H,r_V,d_h], out0 [B,Ncap,r_K+r_V]
    """
    args = _write_kw(kw)
    dev = _cuda(args["x"], args["xv"], args["E_main"], args["E_1"], args["E_K"], args["E_V"],
                args["out0"], args["out1"])
    p = _write_params(mode, **args)
    L = lib()
    need = L.lla_write_workspace_bytes(ctypes.byref(p))
    ws, nb = _workspace(need, dev, workspace)
    _call(L.lla_write_latents, p, ws, nb, _stream_handle(stream, dev), "lla_write_latents")


# ----------------------------------------------------------------- decode --
def _ring_fields(p, win_k, win_v):
    if win_k.shape != win_v.shape or win_k.stride() != win_v.stride() or win_k.dtype != win_v.dtype:
        raise ValueError("win_k and win_v must match in shape, strides and dtype")
    _dense_inner(win_k, 4, "win_k")
    p.win_k, p.win_v = _ptr(win_k), _ptr(win_v)
    p.win_dtype = _dtype_code(win_k)
    p.Wcap = win_k.shape[2]
    p.win_stride_b = win_k.stride(0)


def _events(p, timing_events):
    """Attach the optional (begin, end) torch.cuda.Event pair (timing hook)."""
    if timing_events is None:
        p.timing_events = None
        return
    ev0, ev1 = timing_events
    for ev in (ev0, ev1):
        if ev.cuda_event == 0:
            raise ValueError("record each timing event once before passing it (creates the handle)")
    arr = (ctypes.c_void_p * 2)(ev0.cuda_event, ev1.cuda_event)
    p._keep = arr
    p.timing_events = ctypes.cast(arr, ctypes.c_void_p)


def _win_side(p, win_stream, win_events):
    """Attach the optional window stream and its (fork, join) torch.cuda.Event pair."""
    if win_stream is None:
        p.win_stream = None
        p.win_events = None
        return
    if win_events is None:
        raise ValueError("win_stream needs win_events: a (fork, join) pair of torch.cuda.Event")
    ev0, ev1 = win_events
    for ev in (ev0, ev1):
        if ev.cuda_event == 0:
            raise ValueError("record each window event once before passing it (creates the handle)")
    arr = (ctypes.c_void_p * 2)(ev0.cuda_event, ev1.cuda_event)
    p._keep_win = arr
    p.win_stream = ctypes.c_void_p(win_stream.cuda_stream)
    p.win_events = ctypes.cast(arr, ctypes.c_void_p)


def _hla_params(lat, A, Bm, q, win_k, win_v, out, N, W, t0, r_k, rotate_query, rope_base, scale,
                timing_events=None, win_stream=None, win_events=None):
    p = _abi.HlaDecodeParams()
    if q.dim() == 5:                       # [B, nq, nt, H, d_h]: the last nq positions at once
        B, nq, nt, H, d_h = q.shape
        _dense_inner(q, 4, "q")
        _dense_inner(out, 4, "out")
    else:
        B, nt, H, d_h = q.shape
        nq = 1
        _dense_inner(q, 3, "q")
        _dense_inner(out, 3, "out")
    if tuple(out.shape) != tuple(q.shape):
        raise ValueError("out must have q's shape")
    p.nq = nq
    for t, nm in ((A, "A"), (Bm, "Bm")):
        if not t.is_contiguous() or t.dtype != _torch().float32:
            raise ValueError(f"{nm} must be a contiguous float32 tensor")
    if tuple(A.shape[:3]) != (nt, H, d_h) or tuple(Bm.shape[:2]) != (nt, H) or Bm.shape[3] != d_h:
        raise ValueError("A is [nt,H,d_h,r_k], Bm is [nt,H,r_v,d_h]")
    r_k = A.shape[3] if r_k is None else r_k
    p.B, p.H, p.d_h, p.nt, p.t0 = B, H, d_h, nt, t0
    p.T = win_k.shape[1]
    p.N, p.W = N, W
    p.r_k, p.r_v = r_k, Bm.shape[2]
    if lat is not None:
        _dense_inner(lat, 1, "lat")
        p.lat = _ptr(lat)
        p.lat_dtype = _dtype_code(lat)
        p.lat_stride_b, p.lat_stride_n = lat.stride(0), lat.stride(1)
    p.A, p.Bm, p.q = _ptr(A), _ptr(Bm), _ptr(q)
    p.q_stride_b = q.stride(0)
    p.rotate_query = int(bool(rotate_query))
    p.rope_base = float(rope_base)
    _ring_fields(p, win_k, win_v)
    p.out = _ptr(out)
    p.out_stride_b = out.stride(0)
    p.scale = float(scale)
    _events(p, timing_events)
    _win_side(p, win_stream, win_events)
    return p


def hla_decode_workspace_bytes(**kw):
    p = _hla_params(**_hla_kw(kw))
    return lib().hla_decode_workspace_bytes(ctypes.byref(p))


def _hla_kw(kw):
    d = dict(lat=None, A=None, Bm=None, q=None, win_k=None, win_v=None, out=None, N=None, W=None,
             t0=0, r_k=None, rotate_query=True, rope_base=10000.0, scale=0.0, timing_events=None,
             win_stream=None, win_events=None)
    unknown = set(kw) - set(d) - {"workspace", "stream"}
    if unknown:
        raise TypeError(f"unknown arguments {sorted(unknown)}")
    d.update({k: v for k, v in kw.items() if k in d})
    return d


def hla_decode_attn(*, workspace=None, stream=None, **kw):
    """Absorbed latent read (HLA eqs. 3-4, or LLA-D with rotate_query=False).

    lat [B,Ncap,r_k+r_v] (key part stored as R~_j c^K_j; bf16, float32, or
    uint8 fp8 rows of r_k+r_v+16 bytes), A [nt,H,d_h,r_k], Bm [nt,H,r_v,d_h],
    q [B,nt,H,d_h] (or [B,nq,nt,H,d_h]: the last nq positions of the context
    at once), ring win_k/win_v [B,T,Wcap,H,d_h], out shaped like q, float32;
    N = context length, W = exact window, t0 = first loop served.  Optional
    win_stream (torch.cuda.Stream) with win_events (a (fork, join) pair of
    torch.cuda.Event, each recorded once beforehand): the window runs on
    win_stream beside the query map and the latent read.
    """
    args = _hla_kw(kw)
    dev = _cuda(args["lat"], args["A"], args["Bm"], args["q"], args["win_k"], args["win_v"], args["out"])
    p = _hla_params(**args)
    L = lib()
    need = L.hla_decode_workspace_bytes(ctypes.byref(p))
    ws, nb = _workspace(need, dev, workspace)
    _call(L.hla_decode_attn, p, ws, nb, _stream_handle(stream, dev), "hla_decode_attn")


def _lla_params(cK, cV, UK, UV, q, win_k, win_v, out, N, W, t0, scale, timing_events=None):
    p = _abi.LlaDecodeParams()
    B, nt, H, d_h = q.shape
    _dense_inner(q, 3, "q")
    _dense_inner(out, 3, "out")
    for t, nm in ((UK, "UK"), (UV, "UV")):
        if not t.is_contiguous() or t.dtype != _torch().float32:
            raise ValueError(f"{nm} must be a contiguous float32 tensor")
    r = UK.shape[3]
    p.B, p.H, p.d_h, p.r, p.nt, p.t0 = B, H, d_h, r, nt, t0
    p.T = win_k.shape[1]
    p.N, p.W = N, W
    if cK is not None:
        _dense_inner(cK, 2, "cK")
        if cK.stride() != cV.stride() or cK.dtype != cV.dtype:
            raise ValueError("cK and cV must share strides and dtype")
        p.cK, p.cV = _ptr(cK), _ptr(cV)
        p.lat_dtype = _dtype_code(cK)
        p.lat_stride_b, p.lat_stride_h = cK.stride(0), cK.stride(1)
    p.UK, p.UV, p.q = _ptr(UK), _ptr(UV), _ptr(q)
    p.q_stride_b = q.stride(0)
    _ring_fields(p, win_k, win_v)
    p.out = _ptr(out)
    p.out_stride_b = out.stride(0)
    p.scale = float(scale)
    _events(p, timing_events)
    return p


def _lla_kw(kw):
    d = dict(cK=None, cV=None, UK=None, UV=None, q=None, win_k=None, win_v=None, out=None,
             N=None, W=0, t0=0, scale=0.0, timing_events=None)
    unknown = set(kw) - set(d) - {"workspace", "stream"}
    if unknown:
        raise TypeError(f"unknown arguments {sorted(unknown)}")
    d.update({k: v for k, v in kw.items() if k in d})
    return d


def lla_decode_workspace_bytes(**kw):
    p = _lla_params(**_lla_kw(kw))
    return lib().lla_decode_workspace_bytes(ctypes.byref(p))


def lla_decode_attn(*, workspace=None, stream=None, **kw):
    """LLA reconstruct-on-read decode attention.

    cK, cV [B,H,Ncap,r], UK, UV [nt,H,d_h,r], q [B,nt,H,d_h] post-rotary,
    ring win_k/win_v [B,T,Wcap,H,d_h], out [B,nt,H,d_h] float32.
    """
    args = _lla_kw(kw)
    dev = _cuda(args["cK"], args["cV"], args["UK"], args["UV"], args["q"], args["win_k"],
                args["win_v"], args["out"])
    p = _lla_params(**args)
    L = lib()
    need = L.lla_decode_workspace_bytes(ctypes.byref(p))
    ws, nb = _workspace(need, dev, workspace)
    _call(L.lla_decode_attn, p, ws, nb, _stream_handle(stream, dev), "lla_decode_attn")
