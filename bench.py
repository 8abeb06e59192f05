"""Decode-step benchmark: tokens/s and achieved HBM bandwidth on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--mode m1|m2]
    python bench.py --impl reference ...      # the fp64 CPU oracle, bounded sample

One step = one decode token for every sequence of the batch through every
layer and loop of the hot path: per layer, the absorbed latent reads (loop-1
latent c^(1) and main latent c, eqs. 3-4, with the exact window) or the LLA
read, plus the latent writer (eq. 2) for the token.  The step is captured once
into a CUDA graph and replayed; timing is CUDA events on the replay stream.
Multi-GPU runs are independent replicas (the path shards by sequence with no
collective); the time is the max over ranks.
"""

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "decode tokens/s (all layers×loops) and achieved HBM GB/s vs roofline, 1×B200"


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            p = json.load(fh)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# ------------------------------------------------------------ clocks --
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ----------------------------------------------------------- workloads --
class HlaStep:
    """One decode step of an HLA model (absorbed reads + writer), all layers."""

    def __init__(self, cfg, dev, mode, seed=1234):
        import looped_transformer_latent_b200 as L
        self.L = L
        self.cfg, self.dev, self.mode = cfg, dev, mode
        c = cfg
        B, N, T, H, d_h, D = c.B, c.N, c.T, c.H, c.d_h, c.D
        self.i = N - 1
        Wcap = c.W + 1
        codec = synth.hla_codec(c, seed)
        g = torch.Generator(device=dev)
        g.manual_seed(seed + 7)
        self.layers = []
        self.ws_bytes = 0
        for layer in range(c.L):
            lay = {}
            for k in ("E_main", "E_1", "A", "A_1", "Bm", "B_1"):
                lay[k] = codec[k].to(dev).clone()
            lay["lat"] = torch.empty(B, N, c.r_k + c.r_v, dtype=torch.bfloat16, device=dev)
            lay["lat1"] = torch.empty(B, N, 2 * c.r_1, dtype=torch.bfloat16, device=dev)
            self._prefill(lay, codec["P"], seed + 100 * layer)
            lay["wk"] = torch.randn(B, T, Wcap, H, d_h, generator=g, device=dev).to(torch.bfloat16)
            lay["wv"] = torch.randn(B, T, Wcap, H, d_h, generator=g, device=dev).to(torch.bfloat16)
            lay["q"] = torch.randn(B, T, H, d_h, generator=g, device=dev)
            lay["h"] = synth.hla_hidden(codec["P"], B, seed + 100 * layer + 1, D, device=dev).reshape(B, 1, T, D)
            lay["out"] = torch.empty(B, T, H, d_h, device=dev)
            self.layers.append(lay)
        self.calls = self._calls()
        for kind, kw in self.calls:
            nb = (L.hla_decode_workspace_bytes(**kw) if kind == "hla"
                  else L.lla_write_workspace_bytes(L.LLA_WRITE_HLA, **kw))
            self.ws_bytes = max(self.ws_bytes, nb)
        self.ws = torch.empty(max(self.ws_bytes, 256), dtype=torch.uint8, device=dev)

    def _prefill(self, lay, P, seed):
        c = self.cfg
        L = self.L
        chunk = max(1, (1 << 28) // (c.N * c.T * c.D))  # ~1 GiB of fp32 hidden states
        for b0 in range(0, c.B, chunk):
            nb = min(chunk, c.B - b0)
            h = synth.hla_hidden(P, nb * (c.N - 1), seed + b0, c.D, device=self.dev).reshape(nb, c.N - 1, c.T, c.D)
            L.lla_write_latents(L.LLA_WRITE_HLA, x=h, E_main=lay["E_main"], E_1=lay["E_1"],
                                out0=lay["lat"][b0:b0 + nb], out1=lay["lat1"][b0:b0 + nb], r_k=c.r_k,
                                d_h=c.d_h, pos0=0, rope_base=c.base)
            del h

    def _calls(self):
        c = self.cfg
        calls = []
        for lay in self.layers:
            common = dict(win_k=lay["wk"], win_v=lay["wv"], N=c.N, W=c.W, rope_base=c.base)
            if self.mode == "m1":
                groups = [(0, 1), (1, c.T - 1)]
            else:
                groups = [(t, 1) for t in range(c.T)]
            for t0, nt in groups:
                if t0 == 0:
                    kw = dict(lat=lay["lat1"], A=lay["A_1"], Bm=lay["B_1"], r_k=c.r_1)
                else:
                    a = t0 - 1
                    kw = dict(lat=lay["lat"], A=lay["A"][a:a + nt], Bm=lay["Bm"][a:a + nt], r_k=c.r_k)
                kw.update(common, q=lay["q"][:, t0:t0 + nt], out=lay["out"][:, t0:t0 + nt], t0=t0)
                calls.append(("hla", kw))
            calls.append(("write", dict(x=lay["h"], E_main=lay["E_main"], E_1=lay["E_1"],
                                        out0=lay["lat"], out1=lay["lat1"], r_k=c.r_k, d_h=c.d_h,
                                        pos0=self.i, rope_base=c.base)))
        return calls

    def run(self, events=None):
        L = self.L
        ei = 0
        for kind, kw in self.calls:
            if kind == "hla":
                ev = None
                if events is not None:
                    ev = events[ei]
                    ei += 1
                L.hla_decode_attn(workspace=self.ws, timing_events=ev, **kw)
            else:
                L.lla_write_latents(L.LLA_WRITE_HLA, workspace=self.ws, **kw)

    def n_read_calls(self):
        return sum(1 for k, _ in self.calls if k == "hla")

    def kernel_launches(self):
        n = 0
        n_lat = max(0, self.i - self.cfg.W)
        for kind, _ in self.calls:
            n += (3 + (n_lat > 0)) if kind == "hla" else 2
        return n

    # algorithmic bytes
    def split_bytes(self):
        """Latent bytes each read call streams (its latent-read kernel)."""
        c = self.cfg
        n_lat = max(0, self.i - c.W)
        out = []
        for kind, kw in self.calls:
            if kind == "hla":
                width = kw["lat"].shape[-1]
                out.append(c.B * n_lat * width * 2)
        return out

    def step_bytes(self):
        c = self.cfg
        n_lat = max(0, self.i - c.W)
        n_win = self.i - n_lat + 1
        total = 0
        for kind, kw in self.calls:
            if kind == "hla":
                nt = kw["q"].shape[1]
                total += c.B * n_lat * kw["lat"].shape[-1] * 2                       # latents
                total += c.B * nt * n_win * c.H * c.d_h * 2 * 2                       # window K and V
                total += (kw["A"].numel() + kw["Bm"].numel()) * 4                     # codec A, B
            else:
                total += (kw["E_main"].numel() + kw["E_1"].numel()) * 4               # writer codec
                total += kw["x"].numel() * 4                                          # new token h
                total += c.B * (kw["out0"].shape[-1] + kw["out1"].shape[-1]) * 2      # new rows
        return total

    def io_tensors(self):
        ins = [lay["q"] for lay in self.layers] + [lay["h"] for lay in self.layers]
        outs = [lay["out"] for lay in self.layers]
        return ins, outs


def make_step(cfg, dev, mode):
    if cfg.kind == "hla":
        return HlaStep(cfg, dev, mode)
    raise SystemExit(f"config {cfg.name}: kind {cfg.kind} has no bench step yet")


# ------------------------------------------------------ oracle timing --
def oracle_sample(cfg, seed=5):
    """Time the oracle on one (sequence, layer) slice of a decode step.

    Returns (seconds, threads): both absorbed reads of one sequence for one
    layer plus the writer for its new token, in fp64 numpy.
    """
    import numpy as np
    from oracle import hla
    c = cfg
    rng = np.random.default_rng(seed)
    n = c.N
    lat = rng.standard_normal((n, c.r_k + c.r_v)) * math.sqrt(c.d_h / c.r_k)
    lat1 = rng.standard_normal((n, 2 * c.r_1)) * math.sqrt(c.d_h / c.r_1)
    A = rng.standard_normal((c.T - 1, c.H, c.d_h, c.r_k)) / math.sqrt(c.d_h)
    A1 = rng.standard_normal((1, c.H, c.d_h, c.r_1)) / math.sqrt(c.d_h)
    Bm = rng.standard_normal((c.T - 1, c.H, c.r_v, c.d_h)) / math.sqrt(c.r_v)
    B1 = rng.standard_normal((1, c.H, c.r_1, c.d_h)) / math.sqrt(c.r_1)
    q = rng.standard_normal((c.T, c.H, c.d_h))
    wk = rng.standard_normal((c.T, c.W + 1, c.H, c.d_h))
    wv = rng.standard_normal((c.T, c.W + 1, c.H, c.d_h))
    h = rng.standard_normal((1, c.T, c.D))
    E = rng.standard_normal((c.T - 1, c.r_k + c.r_v, c.D)) / math.sqrt(c.D)
    E1 = rng.standard_normal((2 * c.r_1, c.D)) / math.sqrt(c.D)
    t = time.perf_counter()
    hla.decode(lat1, A1, B1, q[:1], wk, wv, 0, c.N, c.W, c.r_1, c.r_1, c.d_h, c.base)
    hla.decode(lat, A, Bm, q[1:], wk, wv, 1, c.N, c.W, c.r_k, c.r_v, c.d_h, c.base)
    hla.write(h, E, E1, c.N - 1, c.r_k, c.r_v, c.r_1, c.d_h, c.base)
    dt = time.perf_counter() - t
    return dt, _blas_threads()


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([d.get("num_threads", 1) for d in info] or [1])
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(cfg, budget_s=12.0):
    total, n, threads = 0.0, 0, 1
    while total < budget_s and n < 512:
        dt, threads = oracle_sample(cfg, seed=5 + n)
        total += dt
        n += 1
    tok_s = n / (cfg.L * total)   # n (sequence, layer) slices; a token needs L of them
    return {"value": tok_s, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} (sequence, layer) slices of the {cfg.name} step "
                      f"(both reads + writer, fp64 numpy), {total:.1f} s; tokens/s = slices / (L * time)"}


# ---------------------------------------------------------------- main --
def dist_init():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        return dist, dist.get_rank(), ws, int(os.environ.get("LOCAL_RANK", "0"))
    return None, 0, 1, 0


def run_reference(args, cfg):
    # Under torchrun only rank 0 runs the CPU oracle; the other ranks exit.
    if int(os.environ.get("RANK", "0")) != 0:
        return
    for w in range(args.warmup):
        oracle_sample(cfg, seed=100 + w)
    times, threads = [], 1
    for s in range(args.steps):
        dt, threads = oracle_sample(cfg, seed=200 + s)
        times.append(dt)
    total = sum(times)
    v = args.steps / (cfg.L * total)
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * cfg.L * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": cfg.name, "mode": args.mode,
                                        "sample": "one (sequence, layer) slice per step"},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"{args.steps} (sequence, layer) slices of {cfg.name}, {total:.1f} s"},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="ouro_hla_4k", choices=sorted(synth.CONFIGS))
    ap.add_argument("--mode", default="m1", choices=["m1", "m2"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    cfg = synth.CONFIGS[args.config]
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args, cfg)

    dist, rank, world, local = dist_init()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from looped_transformer_latent_b200 import build
    build.build()
    step = make_step(cfg, dev, args.mode)
    stream = torch.cuda.Stream(dev)
    nread = step.n_read_calls()
    evs = [(torch.cuda.Event(enable_timing=True, external=True),
            torch.cuda.Event(enable_timing=True, external=True)) for _ in range(nread)]
    with torch.cuda.stream(stream):
        for e0, e1 in evs:
            e0.record(stream)
            e1.record(stream)
        step.run()                      # eager warm-up (sets kernel attributes)
    torch.cuda.synchronize()
    _, outs = step.io_tensors()
    eager = [o.clone() for o in outs]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step.run(events=evs)
    torch.cuda.synchronize()
    for o in outs:
        o.fill_(float("nan"))
    graph.replay()
    torch.cuda.synchronize()
    for o, e in zip(outs, eager):       # the replayed step must reproduce the eager one
        if not torch.equal(o, e):
            raise SystemExit("graph replay output differs from the eager step")

    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        t1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = t0.elapsed_time(t1) / args.steps
    split_ms = [a.elapsed_time(b) for a, b in evs]       # last replay of the timed region
    if dist is not None:
        tt = torch.tensor([ms], device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ms = float(tt.item())
        dist.barrier()

    # end to end: pinned host inputs -> device, step, outputs -> host
    ins, outs = step.io_tensors()
    h_ins = [t.detach().cpu().pin_memory() for t in ins]
    h_outs = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
    h2d = sum(t.numel() * t.element_size() for t in h_ins)
    d2h = sum(t.numel() * t.element_size() for t in h_outs)
    with torch.cuda.stream(stream):
        for _ in range(3):
            for d, hsrc in zip(ins, h_ins):
                d.copy_(hsrc, non_blocking=True)
            graph.replay()
            for hdst, d in zip(h_outs, outs):
                hdst.copy_(d, non_blocking=True)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            for d, hsrc in zip(ins, h_ins):
                d.copy_(hsrc, non_blocking=True)
            graph.replay()
            for hdst, d in zip(h_outs, outs):
                hdst.copy_(d, non_blocking=True)
        e1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = e0.elapsed_time(e1) / args.steps
    if dist is not None:
        tt = torch.tensor([ms_e2e], device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ms_e2e = float(tt.item())

    hbm, tflops, src = peaks()
    sb = step.split_bytes()
    tot_split_ms = sum(split_ms)
    achieved = (sum(sb) / 1e9) / (tot_split_ms / 1e3) if tot_split_ms > 0 else 0.0
    step_bytes = step.step_bytes()
    tokens = cfg.B * world
    line = {
        "metric": METRIC,
        "value": tokens / (ms / 1e3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": cfg.name, "mode": args.mode, "batch_per_gpu": cfg.B, "context": cfg.N,
                   "layers": cfg.L, "loops": cfg.T, "heads": cfg.H, "d_h": cfg.d_h,
                   "r_k": cfg.r_k, "r_v": cfg.r_v, "r_1": cfg.r_1, "window": cfg.W,
                   "latent_dtype": cfg.lat_dtype, "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (per-step latents >> 126 MB)",
                   "timing": "CUDA graph replay, CUDA events on the replay stream"},
        "achieved_hbm_gbs": step_bytes / 1e9 / (ms / 1e3),
        "step_bytes": step_bytes,
        "step_roofline_frac": (step_bytes / 1e9 / (ms / 1e3)) / hbm,
        "e2e": {"value": tokens / (ms_e2e / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": step.kernel_launches() * args.steps,
        "clocks": clocks,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": None,
                     "kernel": "latent-read split kernel (absorbed read)",
                     "peak_source": src,
                     "per_launch_ms": tot_split_ms / max(1, len(split_ms)),
                     "launches_per_step": len(split_ms)},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg)
    if rank == 0:
        print(json.dumps(line))
    del graph
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
