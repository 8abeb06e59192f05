"""Concurrent kernel timeline of one graph-replayed decode step.

    python -m looped_transformer_latent_b200.profile_timeline --config ouro_hla_4k \
        --replays 3 --out timeline.json.gz
    python -m looped_transformer_latent_b200.profile_timeline --config ouro_hla_4k \
        --replays 3 --from-trace timeline.json.gz      # summarise a saved trace (no GPU)

Builds the step `bench.py` times (same inputs, same streams), captures it in
a CUDA graph, replays it a few times under the PyTorch profiler with CUDA
activity only, and writes the Chrome trace.  The activity records carry each
kernel's start and end on the GPU while the streams overlap, which a
serialising profiler (ncu) cannot show.  Printed: per kernel and grid the
launches and mean duration, the step time over the replays, and the kernels
of one layer (`--layer`) with their start offsets and streams.  Durations
taken under a profiler are diagnostics, not bench numbers.
"""

import argparse
import gzip
import json
import os
import re
import sys
from collections import defaultdict

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _short(name):
    name = re.sub(r"void |lla::|\(anonymous namespace\)::", "", name)
    return name.split("(")[0][:32]


def summarise(events, replays, layer_window):
    ev = sorted((e for e in events if e.get("ph") == "X" and e.get("cat") in ("kernel", "gpu_memset", "gpu_memcpy")),
                key=lambda e: e["ts"])
    if not ev:
        print("no GPU activity recorded")
        return
    t0 = ev[0]["ts"]
    agg = defaultdict(list)
    for e in ev:
        agg[(_short(e["name"]), str(e["args"].get("grid")))].append(e["dur"])
    print(f"{'kernel':34s} {'grid':14s} {'launches':>8s} {'mean us':>8s}")
    for (k, g), v in sorted(agg.items(), key=lambda kv: -sum(kv[1])):
        print(f"{k:34s} {g:14s} {len(v):8d} {sum(v) / len(v):8.1f}")
    span = ev[-1]["ts"] + ev[-1]["dur"] - t0
    print(f"step: {span / replays:.1f} us (span of {replays} replays / {replays})")
    if layer_window is not None:
        lo, hi = layer_window
        print(f"{'start us':>9s} {'dur us':>7s} stream kernel")
        for e in ev:
            if lo <= e["ts"] - t0 <= hi:
                print(f"{e['ts'] - t0:9.1f} {e['dur']:7.1f} s{e['args'].get('stream')} {_short(e['name'])} "
                      f"grid={e['args'].get('grid')}")


def main():
    import bench
    import synth
    from looped_transformer_latent_b200 import build

    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="ouro_hla_4k", choices=sorted(synth.CONFIGS))
    ap.add_argument("--mode", default="m1", choices=["m1", "m2"])
    ap.add_argument("--replays", type=int, default=3)
    ap.add_argument("--layer", type=int, default=8, help="print the kernels of this layer of the first replay")
    ap.add_argument("--out", default="timeline.json.gz")
    ap.add_argument("--from-trace", default=None, help="summarise this saved trace instead of profiling")
    args = ap.parse_args()
    cfg = synth.CONFIGS[args.config]
    if args.from_trace:
        opener = gzip.open if args.from_trace.endswith(".gz") else open
        with opener(args.from_trace, "rt") as f:
            return report(json.load(f)["traceEvents"], args.replays, cfg.L, args.layer)
    build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    step = bench.make_step(cfg, dev, args.mode)
    stream = torch.cuda.Stream(dev)
    with torch.cuda.stream(stream):
        step.run()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step.run()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for _ in range(5):
            graph.replay()
    torch.cuda.synchronize()
    from torch.profiler import ProfilerActivity, profile
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        with torch.cuda.stream(stream):
            for _ in range(args.replays):
                graph.replay()
        torch.cuda.synchronize()
    tmp = args.out[:-3] if args.out.endswith(".gz") else args.out
    prof.export_chrome_trace(tmp)
    with open(tmp) as f:
        trace = json.load(f)
    if args.out.endswith(".gz"):
        with gzip.open(args.out, "wt") as f:
            json.dump(trace, f)
        os.remove(tmp)
    report(trace["traceEvents"], args.replays, cfg.L, args.layer)


def report(events, replays, layers, layer):
    """Summary of a trace of `replays` steps of `layers` layers each."""
    kern = sorted(e["ts"] for e in events if e.get("ph") == "X" and e.get("cat") == "kernel")
    window = None
    if kern:
        per_layer = (kern[-1] - kern[0]) / max(1, replays * layers)
        window = (layer * per_layer, (layer + 1) * per_layer)
    summarise(events, replays, window)


if __name__ == "__main__":
    main()
