"""Run one absorbed-read call of a configuration's latent on synthetic inputs.

    python -m looped_transformer_latent_b200.profile_call --config ouro_hla_4k \
        --group main --batch 16 --iters 3

A small, self-contained workload for profilers (ncu): it builds random bf16
latents and fp32 codecs/queries of the configuration's shapes on the device,
then calls hla_decode_attn `iters` times on one stream and synchronises.
`--group main` reads the main latent (loops 2..T share it), `--group loop1`
the loop-1 latent, `--group folded` an LLA-2D latent (no rotation).
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
    args = ap.parse_args()
    c = synth.CONFIGS[args.config]
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(7)
    B = args.batch
    if args.group == "main":
        t0, nt, r_k, r_v, rotate = 1, c.T - 1, c.r_k, c.r_v, True
    elif args.group == "loop1":
        t0, nt, r_k, r_v, rotate = 0, 1, c.r_1, c.r_1, True
    else:
        t0, nt, r_k, r_v, rotate = 0, c.T, c.r_k, c.r_v, False
    H, d_h, N, W = c.H, c.d_h, c.N, c.W
    Wcap = W + 1
    lat = (torch.randn(B, N, r_k + r_v, generator=g, device=dev) * math.sqrt(d_h / r_k)).to(torch.bfloat16)
    A = torch.randn(nt, H, d_h, r_k, generator=g, device=dev) / math.sqrt(d_h)
    Bm = torch.randn(nt, H, r_v, d_h, generator=g, device=dev) / math.sqrt(r_v)
    q = torch.randn(B, nt, H, d_h, generator=g, device=dev)
    wk = torch.randn(B, c.T, Wcap, H, d_h, generator=g, device=dev).to(torch.bfloat16)
    wv = torch.randn(B, c.T, Wcap, H, d_h, generator=g, device=dev).to(torch.bfloat16)
    out = torch.empty(B, nt, H, d_h, device=dev)
    kw = dict(lat=lat, A=A, Bm=Bm, q=q, win_k=wk, win_v=wv, out=out, N=N, W=W, t0=t0,
              rotate_query=rotate, rope_base=c.base)
    ws = torch.empty(max(256, L.hla_decode_workspace_bytes(**kw)), dtype=torch.uint8, device=dev)
    for _ in range(args.iters):
        L.hla_decode_attn(workspace=ws, **kw)
    torch.cuda.synchronize()
    print(f"ok: {args.config} {args.group} B={B} N={N} rows={nt * H} r_k={r_k} r_v={r_v}, "
          f"latent bytes per call {lat[:, :max(0, N - 1 - W)].numel() * 2 / 1e6:.1f} MB")


if __name__ == "__main__":
    main()
