"""Run one call of the hot path on synthetic inputs of a configuration's shapes.

    python -m looped_transformer_latent_b200.profile_call --config ouro_hla_4k \
        --group main --batch 16 --iters 3
    python -m looped_transformer_latent_b200.profile_call --op write \
        --config ouro_lla2d_768 --batch 768 --iters 3

A small, self-contained workload for profilers (ncu).  `--op read` (default)
builds random bf16 latents and fp32 codecs/queries on the device and calls
hla_decode_attn `iters` times: `--group main` reads the main latent (loops
2..T share it), `--group loop1` the loop-1 latent, `--group folded` an LLA-2D
latent (no rotation); `--nq n` reads the last n positions in one call
(multi-query), `--fp8` reads e4m3 rows with per-token scales instead of bf16
rows.  `--op write` calls lla_write_latents for one decode token per sequence
in the configuration's writer mode (HLA, LLA-2D folded or LLA per-head).
`--time` brackets each call with CUDA events on the launching stream and
prints the median time and the latent bytes per second (reads whose latent is
larger than the 126 MB L2 stream from HBM on every call).
"""

import argparse
import math
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main():
    import looped_transformer_latent_b200 as L
    import synth

    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="ouro_hla_4k", choices=sorted(synth.CONFIGS))
    ap.add_argument("--group", default="main", choices=["main", "loop1", "folded"])
    ap.add_argument("--batch", type=int, default=16)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--op", default="read", choices=["read", "write", "recon"])
    ap.add_argument("--context", type=int, default=0, help="override the context length N (read)")
    ap.add_argument("--nq", type=int, default=1, help="query positions per call (read)")
    ap.add_argument("--fp8", action="store_true", help="e4m3 latent rows with per-token scales (read)")
    ap.add_argument("--time", action="store_true", help="time each call with CUDA events")
    args = ap.parse_args()
    c = synth.CONFIGS[args.config]
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(7)
    B = args.batch
    if args.op == "write":
        return write(L, c, B, args.iters, g, dev)
    if args.op == "recon":
        return recon(L, c, B, args.iters, g, dev, args.context or c.N)
    if args.group == "main":
        t0, nt, r_k, r_v, rotate = 1, c.T - 1, c.r_k, c.r_v, True
    elif args.group == "loop1":
        t0, nt, r_k, r_v, rotate = 0, 1, c.r_1, c.r_1, True
    else:
        t0, nt, r_k, r_v, rotate = 0, c.T, c.r_k, c.r_v, False
    H, d_h, N, W, nq = c.H, c.d_h, (args.context or c.N), c.W, args.nq
    Wcap = (min(N, W + nq) if nq > 1 else W) + 1
    if args.fp8:
        # codes uniform over the finite e4m3 patterns, scales of the bf16 rows' magnitude
        w = r_k + r_v
        lat = torch.zeros(B, N, w + 16, dtype=torch.uint8, device=dev)
        codes = torch.randint(0, 256, (B, N, w), generator=g, device=dev, dtype=torch.int32)
        codes = torch.where((codes & 0x7F) == 0x7F, codes - 1, codes)   # no NaN pattern
        lat[..., :w] = codes.to(torch.uint8)
        scale = torch.full((B, N, 2), math.sqrt(d_h / r_k) / 64.0, device=dev)
        lat[..., w:w + 8] = scale.view(torch.uint8).reshape(B, N, 8)
    else:
        lat = (torch.randn(B, N, r_k + r_v, generator=g, device=dev) * math.sqrt(d_h / r_k)).to(torch.bfloat16)
    A = torch.randn(nt, H, d_h, r_k, generator=g, device=dev) / math.sqrt(d_h)
    Bm = torch.randn(nt, H, r_v, d_h, generator=g, device=dev) / math.sqrt(r_v)
    qshape = (B, nt, H, d_h) if nq == 1 else (B, nq, nt, H, d_h)
    q = torch.randn(qshape, generator=g, device=dev)
    wk = torch.randn(B, c.T, Wcap, H, d_h, generator=g, device=dev).to(torch.bfloat16)
    wv = torch.randn(B, c.T, Wcap, H, d_h, generator=g, device=dev).to(torch.bfloat16)
    out = torch.empty(qshape, device=dev)
    kw = dict(lat=lat, A=A, Bm=Bm, q=q, win_k=wk, win_v=wv, out=out, N=N, W=W, t0=t0,
              rotate_query=rotate, rope_base=c.base)
    ws = torch.empty(max(256, L.hla_decode_workspace_bytes(**kw)), dtype=torch.uint8, device=dev)
    nbytes = lat[:, :max(0, N - 1 - W)].numel() * lat.element_size()
    times = _timed(lambda: L.hla_decode_attn(workspace=ws, **kw), args.iters, args.time)
    print(f"ok: {args.config} {args.group} B={B} N={N} nq={nq} rows={nq * nt * H} r_k={r_k} r_v={r_v} "
          f"{'fp8' if args.fp8 else 'bf16'}, latent bytes per call {nbytes / 1e6:.1f} MB")
    _report(times, nbytes)


def _timed(call, iters, timed):
    """Run call iters times; with timed, bracket each with CUDA events on the
    current stream and return the durations in ms."""
    if not timed:
        for _ in range(iters):
            call()
        torch.cuda.synchronize()
        return []
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
    torch.cuda.synchronize()
    for a, b in ev:
        a.record()
        call()
        b.record()
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def _report(times, nbytes):
    if not times:
        return
    t = sorted(times[1:] if len(times) > 1 else times)   # the first call also pays the first-touch costs
    med = t[len(t) // 2]
    print(f"time: median {med:.4f} ms (min {t[0]:.4f}, max {t[-1]:.4f}) over {len(t)} calls; "
          f"{nbytes / 1e9 / (med / 1e3):.1f} GB/s of latent bytes")


def recon(L, c, B, iters, g, dev, N):
    """LLA per-head reconstruct-on-read: all T loops of every head, W = 0."""
    r, T, H, d_h = c.r_k, c.T, c.H, c.d_h
    cK = torch.randn(B, H, N, r, generator=g, device=dev).to(torch.bfloat16)
    cV = torch.randn(B, H, N, r, generator=g, device=dev).to(torch.bfloat16)
    UK = torch.randn(T, H, d_h, r, generator=g, device=dev) / math.sqrt(r)
    UV = torch.randn(T, H, d_h, r, generator=g, device=dev) / math.sqrt(r)
    q = torch.randn(B, T, H, d_h, generator=g, device=dev)
    wk = torch.randn(B, T, 1, H, d_h, generator=g, device=dev).to(torch.bfloat16)
    wv = torch.randn(B, T, 1, H, d_h, generator=g, device=dev).to(torch.bfloat16)
    out = torch.empty(B, T, H, d_h, device=dev)
    kw = dict(cK=cK, cV=cV, UK=UK, UV=UV, q=q, win_k=wk, win_v=wv, out=out, N=N, W=0, t0=0)
    ws = torch.empty(max(256, L.lla_decode_workspace_bytes(**kw)), dtype=torch.uint8, device=dev)
    for _ in range(iters):
        L.lla_decode_attn(workspace=ws, **kw)
    torch.cuda.synchronize()
    print(f"ok: recon {c.name} B={B} N={N} H={H} T={T} r={r}")


def write(L, c, B, iters, g, dev):
    pos = 0   # the row written does not change the work; row 0 keeps the buffers small
    if c.kind == "hla":
        h = torch.randn(B, 1, c.T, c.D, generator=g, device=dev)
        E = torch.randn(c.T - 1, c.r_k + c.r_v, c.D, generator=g, device=dev) / math.sqrt(c.D)
        E1 = torch.randn(2 * c.r_1, c.D, generator=g, device=dev) / math.sqrt(c.D)
        out0 = torch.empty(B, pos + 1, c.r_k + c.r_v, dtype=torch.bfloat16, device=dev)
        out1 = torch.empty(B, pos + 1, 2 * c.r_1, dtype=torch.bfloat16, device=dev)
        kw = dict(x=h, E_main=E, E_1=E1, out0=out0, out1=out1, r_k=c.r_k, d_h=c.d_h, pos0=pos, rope_base=c.base)
        mode = L.LLA_WRITE_HLA
    else:
        k = torch.randn(B, 1, c.T, c.H, c.d_h, generator=g, device=dev)
        v = torch.randn(B, 1, c.T, c.H, c.d_h, generator=g, device=dev)
        EK = torch.randn(c.T, c.H, c.r_k, c.d_h, generator=g, device=dev) / math.sqrt(c.d_h)
        EV = torch.randn(c.T, c.H, c.r_v, c.d_h, generator=g, device=dev) / math.sqrt(c.d_h)
        if c.kind == "lla2d":
            out0 = torch.empty(B, pos + 1, c.r_k + c.r_v, dtype=torch.bfloat16, device=dev)
            kw = dict(x=k, xv=v, E_K=EK, E_V=EV, out0=out0, pos0=pos)
            mode = L.LLA_WRITE_FOLDED
        else:
            out0 = torch.empty(B, c.H, pos + 1, c.r_k, dtype=torch.bfloat16, device=dev)
            out1 = torch.empty(B, c.H, pos + 1, c.r_v, dtype=torch.bfloat16, device=dev)
            kw = dict(x=k, xv=v, E_K=EK, E_V=EV, out0=out0, out1=out1, pos0=pos)
            mode = L.LLA_WRITE_PERHEAD
    ws = torch.empty(max(256, L.lla_write_workspace_bytes(mode, **kw)), dtype=torch.uint8, device=dev)
    for _ in range(iters):
        L.lla_write_latents(mode, workspace=ws, **kw)
    torch.cuda.synchronize()
    print(f"ok: write {c.name} B={B} mode={mode}")


if __name__ == "__main__":
    main()
