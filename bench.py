"""Decode-step benchmark: tokens/s and achieved HBM bandwidth on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--mode m1|m2]
    python bench.py --impl reference ...      # the fp64 CPU oracle, bounded sample

One step = one decode token for every sequence of the batch through every
layer and loop of the hot path: per layer, the absorbed latent reads (loop-1
latent c^(1) and main latent c, eqs. 3-4, with the exact window) or the LLA
read, plus the latent writer (eq. 2) for the token.  In M1 the loop-1 and main
reads of a layer are independent and run on two streams.  The step is captured
once into a CUDA graph and replayed; timing is CUDA events on the replay stream.
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
class Step:
    """One decode step: every layer's latent reads plus the writer for the new
    token.  Subclasses fill self.calls with (kind, kwargs, tag) tuples; tag
    'main' marks the read calls whose latent-read kernel is the roofline's."""

    kind_launches = {"hla": 3, "lla": 2, "write": 2}
    overlap_writes = True   # False: writers in stream order (a read needs their row, or saturates HBM)

    def __init__(self, cfg, dev, mode):
        import looped_transformer_latent_b200 as L
        self.L = L
        self.cfg, self.dev, self.mode = cfg, dev, mode
        self.i = cfg.N - 1
        self.n_lat = max(0, self.i - cfg.W)
        self.n_win = self.i - self.n_lat + 1
        self.calls = []

    def _workspace(self):
        L = self.L
        nb, nbw = 0, 0
        for kind, kw, _ in self.calls:
            if kind == "hla":
                nb = max(nb, L.hla_decode_workspace_bytes(**kw))
            elif kind == "lla":
                nb = max(nb, L.lla_decode_workspace_bytes(**kw))
            else:
                mode = kw["mode"]
                nbw = max(nbw, L.lla_write_workspace_bytes(mode, **{k: v for k, v in kw.items() if k != "mode"}))
        self.ws = torch.empty(max(nb, nbw, 256), dtype=torch.uint8, device=self.dev)
        # The writer stores the new token's latent row, which no read of this
        # step uses (the next step's reads do): it runs on its own stream with
        # its own workspace, forked at its layer's start and joined at the end
        # of the step, so it overlaps the reads.
        self.wstream = torch.cuda.Stream(self.dev)
        self.ws_w = torch.empty(max(nbw, 256), dtype=torch.uint8, device=self.dev)
        self.wfork = [torch.cuda.Event() for _ in range(self.cfg.L)]
        self.wjoin = torch.cuda.Event()
        # the prefill ran on the constructing stream; the step may run on any
        # other, so setup ends with everything it issued complete
        torch.cuda.synchronize(self.dev)

    def layer_io(self):
        """(inputs, outputs) of each layer in order: every workload appends the
        same number of calls, inputs and outputs per layer."""
        n = self.cfg.L
        ci, co = len(self.ins) // n, len(self.outs) // n
        return [(self.ins[k * ci:(k + 1) * ci], self.outs[k * co:(k + 1) * co]) for k in range(n)]

    def run(self, events=None, hook=None):
        """Issue the step on the current stream.  hook(layer, "begin"/"end"),
        if given, runs on the current stream before a layer's first call and
        after its last one."""
        L = self.L
        main = torch.cuda.current_stream(self.dev)
        ei = 0
        per = len(self.calls) // self.cfg.L
        for idx, (kind, kw, _) in enumerate(self.calls):
            layer = idx // per
            if idx % per == 0:
                if hook is not None:
                    hook(layer, "begin")
                self.wfork[layer].record(main)
            if kind in ("hla", "lla"):
                ev = None
                if events is not None:
                    ev = events[ei]
                    ei += 1
                fn = L.hla_decode_attn if kind == "hla" else L.lla_decode_attn
                fn(workspace=self.ws, timing_events=ev, **kw)
            elif self.overlap_writes:
                self.write_async(layer, kw)
            else:
                L.lla_write_latents(kw["mode"], workspace=self.ws, **{k: v for k, v in kw.items() if k != "mode"})
            if hook is not None and idx % per == per - 1:
                hook(layer, "end")
        if self.overlap_writes:
            self.join_writers(main)

    def write_async(self, layer, kw):
        """The layer's writer on the writer stream, after everything issued on
        the step's stream before the layer began."""
        self.wstream.wait_event(self.wfork[layer])
        self.L.lla_write_latents(kw["mode"], workspace=self.ws_w, stream=self.wstream,
                                 **{k: v for k, v in kw.items() if k != "mode"})

    def join_writers(self, main):
        self.wjoin.record(self.wstream)
        main.wait_event(self.wjoin)

    def read_tags(self):
        return [tag for kind, _, tag in self.calls if kind in ("hla", "lla")]

    def kernel_launches(self):
        n = 0
        for kind, _, _ in self.calls:
            n += self.kind_launches["write" if kind.startswith("write") else kind]
            if kind in ("hla", "lla") and self.n_lat > 0:
                n += 1
        return n

    def latent_bytes(self, kind, kw):
        c = self.cfg
        if kind == "hla":
            lat = kw["lat"]
            return c.B * self.n_lat * lat.shape[-1] * lat.element_size()
        return c.B * c.H * self.n_lat * kw["cK"].shape[-1] * 2 * 2

    def read_latent_bytes(self):
        return [self.latent_bytes(kind, kw) for kind, kw, _ in self.calls if kind in ("hla", "lla")]

    def step_bytes(self):
        """Algorithmic bytes: latents + exact window + codecs read, writer inputs/outputs."""
        c = self.cfg
        total = 0
        for kind, kw, _ in self.calls:
            if kind in ("hla", "lla"):
                nt = kw["q"].shape[1]
                total += self.latent_bytes(kind, kw)
                total += c.B * nt * self.n_win * c.H * c.d_h * kw["win_k"].element_size() * 2
                mats = ("A", "Bm") if kind == "hla" else ("UK", "UV")
                total += sum(kw[m].numel() * 4 for m in mats)
            else:
                for k in ("E_main", "E_1", "E_K", "E_V", "x", "xv"):
                    if kw.get(k) is not None:
                        total += kw[k].numel() * 4
                for k in ("out0", "out1"):
                    o = kw.get(k)
                    if o is not None:
                        n_tok = kw["x"].shape[1]
                        rows = c.B * n_tok * (o.shape[1] if o.dim() == 4 else 1)
                        total += rows * o.shape[-1] * o.element_size()
        return total

    def io_tensors(self):
        return self.ins, self.outs


def _clone_layers(bufs, n):
    """Layer 0's buffer and n-1 independent copies (distinct memory)."""
    return [bufs] + [bufs.clone() for _ in range(n - 1)]


class HlaStep(Step):
    """HLA (Ouro-shaped): per layer the loop-1 read, the main read (loops 2..T
    together in M1, one call per loop in M2) and the writer."""

    def __init__(self, cfg, dev, mode, seed=1234):
        super().__init__(cfg, dev, mode)
        L = self.L
        c = cfg
        B, N, T, H, d_h, D = c.B, c.N, c.T, c.H, c.d_h, c.D
        self.codec_host = synth.hla_codec(c, seed)
        codec = {k: v.to(dev) for k, v in self.codec_host.items()}
        self.seed = seed
        g = torch.Generator(device=dev)
        g.manual_seed(seed + 7)
        lat0 = torch.empty(B, N, c.r_k + c.r_v, dtype=torch.bfloat16, device=dev)
        lat10 = torch.empty(B, N, 2 * c.r_1, dtype=torch.bfloat16, device=dev)
        # prefill: the writer fills layer 0 from synthetic hidden states; the
        # other layers get copies (the bytes every layer reads are its own)
        chunk = self.prefill_chunk = max(1, (1 << 28) // (N * T * D))
        for b0 in range(0, B, chunk):
            nb = min(chunk, B - b0)
            h = self._prefill_hidden_chunk(b0, nb)
            L.lla_write_latents(L.LLA_WRITE_HLA, x=h, E_main=codec["E_main"], E_1=codec["E_1"],
                                out0=lat0[b0:b0 + nb], out1=lat10[b0:b0 + nb], r_k=c.r_k, d_h=d_h,
                                pos0=0, rope_base=c.base)
            del h
        lats = _clone_layers(lat0, c.L)
        lat1s = _clone_layers(lat10, c.L)
        self.ins, self.outs, self.layers = [], [], []
        for layer in range(c.L):
            lay = {k: codec[k].clone() for k in ("E_main", "E_1", "A", "A_1", "Bm", "B_1")}
            self.layers.append(lay)
            lay["lat"], lay["lat1"] = lats[layer], lat1s[layer]
            Wcap = c.W + 1
            lay["wk"] = torch.randn(B, T, Wcap, H, d_h, generator=g, device=dev).to(torch.bfloat16)
            lay["wv"] = torch.randn(B, T, Wcap, H, d_h, generator=g, device=dev).to(torch.bfloat16)
            lay["q"] = torch.randn(B, T, H, d_h, generator=g, device=dev)
            lay["h"] = synth.hla_hidden(codec["P"], B, seed + 100 * layer + 1, D, device=dev).reshape(B, 1, T, D)
            lay["out"] = torch.empty(B, T, H, d_h, device=dev)
            self.ins += [lay["q"], lay["h"]]
            self.outs.append(lay["out"])
            common = dict(win_k=lay["wk"], win_v=lay["wv"], N=N, W=c.W, rope_base=c.base)
            groups = [(0, 1), (1, T - 1)] if mode == "m1" else [(t, 1) for t in range(T)]
            for t0, nt in groups:
                if t0 == 0:
                    kw = dict(lat=lay["lat1"], A=lay["A_1"], Bm=lay["B_1"], r_k=c.r_1)
                    tag = "loop1"
                else:
                    a = t0 - 1
                    kw = dict(lat=lay["lat"], A=lay["A"][a:a + nt], Bm=lay["Bm"][a:a + nt], r_k=c.r_k)
                    tag = "main"
                kw.update(common, q=lay["q"][:, t0:t0 + nt], out=lay["out"][:, t0:t0 + nt], t0=t0)
                self.calls.append(("hla", kw, tag))
            self.calls.append(("write", dict(mode=L.LLA_WRITE_HLA, x=lay["h"], E_main=lay["E_main"],
                                             E_1=lay["E_1"], out0=lay["lat"], out1=lay["lat1"], r_k=c.r_k,
                                             d_h=d_h, pos0=self.i, rope_base=c.base), None))
        self._workspace()
        # M1: a layer's loop-1 read and its main read are independent (every
        # loop's query exists), so the loop-1 read and the writer run on a second
        # stream with their own workspace; layers stay in order (fork and join
        # per layer)
        self.side = None
        if mode == "m1":
            self.side = torch.cuda.Stream(dev)
            self.ws_side = torch.empty_like(self.ws)
            self.fork = [torch.cuda.Event() for _ in range(c.L)]
            self.join = [torch.cuda.Event() for _ in range(c.L)]

    def _prefill_hidden_chunk(self, b0, nb):
        c = self.cfg
        return synth.hla_hidden(self.codec_host["P"], nb * (c.N - 1), self.seed + b0, c.D,
                                device=self.dev).reshape(nb, c.N - 1, c.T, c.D)

    def prefill_hidden(self, b):
        """Host copy of the hidden states [N-1, T, D] the prefill wrote for
        sequence b (regenerated from the same seeded generator)."""
        b0 = b // self.prefill_chunk * self.prefill_chunk
        nb = min(self.prefill_chunk, self.cfg.B - b0)
        return self._prefill_hidden_chunk(b0, nb)[b - b0].cpu()

    def run(self, events=None, hook=None):
        if self.side is None:
            return super().run(events, hook)
        L = self.L
        main = torch.cuda.current_stream(self.dev)
        ei = 0
        for layer in range(self.cfg.L):
            (k1, kw1, _), (k2, kw2, _), (_, kww, _) = self.calls[3 * layer:3 * layer + 3]
            assert k1 == "hla" and k2 == "hla"
            if hook is not None:
                hook(layer, "begin")
            self.fork[layer].record(main)
            self.wfork[layer].record(main)
            self.side.wait_event(self.fork[layer])
            L.hla_decode_attn(workspace=self.ws_side, stream=self.side,
                              timing_events=events[ei] if events is not None else None, **kw1)
            # the writer only touches the new token's row, which neither read uses
            self.write_async(layer, kww)
            self.join[layer].record(self.side)
            L.hla_decode_attn(workspace=self.ws, stream=main,
                              timing_events=events[ei + 1] if events is not None else None, **kw2)
            main.wait_event(self.join[layer])
            if hook is not None:
                hook(layer, "end")
            ei += 2
        self.join_writers(main)


class Lla2dStep(Step):
    """LLA-2D capacity regime: per layer one absorbed read of the folded latent
    (all 4 loops x 16 heads = 64 rows share it; LLA-D, no rotation, W = 0) and
    the folded writer.  The layers alternate between two latent buffers of
    B x N x (r_K + r_V) bf16 (7.25 GB each at batch 768): every read streams
    from HBM (each buffer is far larger than L2), 24 separate buffers would
    not fit in 180 GB next to everything else."""

    NBUF = 2

    def __init__(self, cfg, dev, mode, seed=4321):
        super().__init__(cfg, dev, mode)
        L = self.L
        c = cfg
        B, N, T, H, d_h = c.B, c.N, c.T, c.H, c.d_h
        self.codec_host = synth.lla_folded_codec(c, seed)
        codec = {k: v.to(dev) for k, v in self.codec_host.items()}
        self.seed = seed
        g = torch.Generator(device=dev)
        g.manual_seed(seed + 7)
        if c.lat_dtype == "fp8":   # byte rows: codes, then s^K, s^V and 8 zero bytes
            lat0 = torch.empty(B, N, c.r_k + c.r_v + 16, dtype=torch.uint8, device=dev)
        else:
            lat0 = torch.empty(B, N, c.r_k + c.r_v, dtype=torch.bfloat16, device=dev)
        chunk = self.prefill_chunk = max(1, (1 << 28) // (N * T * H * d_h * 2))
        for b0 in range(0, B, chunk):
            nb = min(chunk, B - b0)
            k, v = self._prefill_kv_chunk(b0, nb)
            L.lla_write_latents(L.LLA_WRITE_FOLDED, x=k, xv=v, E_K=codec["E_K"], E_V=codec["E_V"],
                                out0=lat0[b0:b0 + nb], pos0=0)
            del k, v
        # The bf16 read streams at close to full HBM bandwidth on every SM: a
        # writer running beside it slows it by more than the writer's own time
        # (measured 40.1 vs 38.7 ms per step), so the writers stay in stream
        # order there.  The fp8 read leaves bandwidth to spare.
        self.overlap_writes = c.lat_dtype == "fp8"
        lats = [lat0] + [lat0.clone() for _ in range(self.NBUF - 1)]
        self.ins, self.outs, self.layers = [], [], []
        for layer in range(c.L):
            lay = {"UK": codec["U_K"].clone(), "UVt": codec["U_V"].transpose(2, 3).contiguous(),
                   "EK": codec["E_K"].clone(), "EV": codec["E_V"].clone(), "lat": lats[layer % self.NBUF]}
            self.layers.append(lay)
            k_new, v_new = synth.lla_kv(codec["P"], B, d_h, seed + 1000 + layer, device=dev)
            lay["k"] = k_new.reshape(B, 1, T, H, d_h)
            lay["v"] = v_new.reshape(B, 1, T, H, d_h)
            ring = 1   # W = 0: the ring holds the current token only
            lay["wk"] = lay["k"].reshape(B, T, ring, H, d_h).to(torch.bfloat16)
            lay["wv"] = lay["v"].reshape(B, T, ring, H, d_h).to(torch.bfloat16)
            lay["q"] = torch.randn(B, T, H, d_h, generator=g, device=dev)
            lay["out"] = torch.empty(B, T, H, d_h, device=dev)
            self.ins += [lay["q"], lay["k"], lay["v"]]
            self.outs.append(lay["out"])
            self.calls.append(("hla", dict(lat=lay["lat"], A=lay["UK"], Bm=lay["UVt"], q=lay["q"],
                                           win_k=lay["wk"], win_v=lay["wv"], out=lay["out"], N=N, W=0,
                                           t0=0, rotate_query=False), "main"))
            self.calls.append(("write", dict(mode=L.LLA_WRITE_FOLDED, x=lay["k"], xv=lay["v"], E_K=lay["EK"],
                                             E_V=lay["EV"], out0=lay["lat"], pos0=self.i), None))
        self._workspace()


    def _prefill_kv_chunk(self, b0, nb):
        c = self.cfg
        k, v = synth.lla_kv(self.codec_host["P"], nb * (c.N - 1), c.d_h, self.seed + b0, device=self.dev)
        shape = (nb, c.N - 1, c.T, c.H, c.d_h)
        return k.reshape(shape), v.reshape(shape)

    def prefill_kv(self, b):
        """Host copies of the keys and values [N-1, T, H, d_h] the prefill
        wrote for sequence b (regenerated from the same seeded generator)."""
        b0 = b // self.prefill_chunk * self.prefill_chunk
        nb = min(self.prefill_chunk, self.cfg.B - b0)
        k, v = self._prefill_kv_chunk(b0, nb)
        return k[b - b0].cpu(), v[b - b0].cpu()


class LlaStep(Step):
    """LLA per-head reconstruct-on-read (Huginn-like): one layer, all T loops
    of every head read their head's latents in one call, plus the per-head
    writer.  With W = 0 the writer stores the new token's latent (read from the
    next step on).  With W > 0 (served semantics: an exact ring of the last W
    tokens and the current one) the writer is the streaming store of the token
    leaving the window, N - 2 - W, issued before the read, which needs it
    (prefill wrote it too; the writer's rows do not depend on how many tokens a
    call writes, so the store reproduces them bit for bit).  Elsewhere the
    writer's row is read only from the next step on, so writers run on their
    own stream, overlapping the reads."""

    def __init__(self, cfg, dev, mode, seed=777):
        super().__init__(cfg, dev, mode)
        L = self.L
        c = cfg
        B, N, T, H, d_h, r, W = c.B, c.N, c.T, c.H, c.d_h, c.r_k, c.W
        codec = {k: v.to(dev) for k, v in synth.lla_perhead_codec(c, seed).items()}
        g = torch.Generator(device=dev)
        g.manual_seed(seed + 7)
        Wc = W + 1
        cK = torch.empty(B, H, N, r, dtype=torch.bfloat16, device=dev)
        cV = torch.empty(B, H, N, r, dtype=torch.bfloat16, device=dev)
        ring_k = torch.zeros(B, T, Wc, H, d_h, dtype=torch.bfloat16, device=dev)
        ring_v = torch.zeros_like(ring_k)
        evict = N - 2 - W
        if W > 0:
            self.ek = torch.empty(B, 1, T, H, d_h, device=dev)
            self.ev = torch.empty(B, 1, T, H, d_h, device=dev)
        chunk = max(1, (1 << 28) // (N * T * H * d_h * 2))
        for b0 in range(0, B, chunk):
            nb = min(chunk, B - b0)
            k, v = synth.lla_kv(codec["P"], nb * (N - 1), d_h, seed + b0, device=dev)
            k = k.reshape(nb, N - 1, T, H, d_h)
            v = v.reshape(nb, N - 1, T, H, d_h)
            L.lla_write_latents(L.LLA_WRITE_PERHEAD, x=k, xv=v, E_K=codec["E_K"], E_V=codec["E_V"],
                                out0=cK[b0:b0 + nb], out1=cV[b0:b0 + nb], pos0=0)
            for j in range(max(0, N - 1 - W), N - 1):   # exact tokens of the window before the new one
                ring_k[b0:b0 + nb, :, j % Wc] = k[:, j].to(torch.bfloat16)
                ring_v[b0:b0 + nb, :, j % Wc] = v[:, j].to(torch.bfloat16)
            if W > 0:
                self.ek[b0:b0 + nb, 0] = k[:, evict]
                self.ev[b0:b0 + nb, 0] = v[:, evict]
            del k, v
        k_new, v_new = synth.lla_kv(codec["P"], B, d_h, seed + 99, device=dev)
        self.k = k_new.reshape(B, 1, T, H, d_h)
        self.v = v_new.reshape(B, 1, T, H, d_h)
        ring_k[:, :, (N - 1) % Wc] = self.k[:, 0].to(torch.bfloat16)
        ring_v[:, :, (N - 1) % Wc] = self.v[:, 0].to(torch.bfloat16)
        self.q = torch.randn(B, T, H, d_h, generator=g, device=dev)
        self.out = torch.empty(B, T, H, d_h, device=dev)
        self.ins, self.outs = [self.q, self.k, self.v], [self.out]
        read = ("lla", dict(cK=cK, cV=cV, UK=codec["U_K"], UV=codec["U_V"], q=self.q, win_k=ring_k,
                            win_v=ring_v, out=self.out, N=N, W=W, t0=0), "main")
        if W > 0:
            # served: the token leaving the window is stored first, then read
            # (it is among this step's latent tokens), in stream order
            self.ins += [self.ek, self.ev]
            self.overlap_writes = False
            self.calls.append(("write", dict(mode=L.LLA_WRITE_PERHEAD, x=self.ek, xv=self.ev, E_K=codec["E_K"],
                                             E_V=codec["E_V"], out0=cK, out1=cV, pos0=evict), None))
            self.calls.append(read)
        else:
            self.calls.append(read)
            self.calls.append(("write", dict(mode=L.LLA_WRITE_PERHEAD, x=self.k, xv=self.v, E_K=codec["E_K"],
                                             E_V=codec["E_V"], out0=cK, out1=cV, pos0=self.i), None))
        self._workspace()


def make_step(cfg, dev, mode):
    if cfg.kind == "hla":
        return HlaStep(cfg, dev, mode)
    if cfg.kind == "lla2d":
        return Lla2dStep(cfg, dev, mode)
    return LlaStep(cfg, dev, mode)


# ------------------------------------------------------ oracle timing --
def oracle_sample(cfg, seed=5):
    """Time the oracle on one slice of a decode step, fp64 numpy.

    HLA and LLA-2D: one (sequence, layer) slice -- its reads and the writer for
    its new token.  LLA reconstruct: one (sequence, head) slice of the single
    layer -- all T loops of that head.  Returns (seconds, threads, slices per
    decoded token)."""
    import numpy as np
    from oracle import hla, lla
    c = cfg
    rng = np.random.default_rng(seed)
    n = c.N
    if c.kind == "hla":
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
        per_token = c.L
    elif c.kind == "lla2d":
        lat = rng.standard_normal((n, c.r_k + c.r_v)) * math.sqrt(c.d_h / c.r_k)
        UK = rng.standard_normal((c.T, c.H, c.d_h, c.r_k)) / math.sqrt(c.r_k)
        UV = rng.standard_normal((c.T, c.H, c.d_h, c.r_v)) / math.sqrt(c.r_v)
        EK = rng.standard_normal((c.T, c.H, c.r_k, c.d_h)) / math.sqrt(c.d_h)
        EV = rng.standard_normal((c.T, c.H, c.r_v, c.d_h)) / math.sqrt(c.d_h)
        q = rng.standard_normal((c.T, c.H, c.d_h))
        k = rng.standard_normal((1, c.T, c.H, c.d_h))
        v = rng.standard_normal((1, c.T, c.H, c.d_h))
        if c.lat_dtype == "fp8":
            from oracle import quant
            rows = quant.row_bytes(*quant.quantize_rows(lat, c.r_k, c.r_v))
            t = time.perf_counter()
            lat = quant.from_row_bytes(rows, c.r_k, c.r_v)
            lla.decode_absorbed(lat, UK, UV, q, k[0][:, None], v[0][:, None], 0, c.N, 0, c.r_k, c.r_v)
            quant.quantize_rows(lla.write_folded(k, v, EK, EV), c.r_k, c.r_v)
        else:
            t = time.perf_counter()
            lla.decode_absorbed(lat, UK, UV, q, k[0][:, None], v[0][:, None], 0, c.N, 0, c.r_k, c.r_v)
            lla.write_folded(k, v, EK, EV)
        per_token = c.L
    else:
        cK = rng.standard_normal((1, n, c.r_k))
        cV = rng.standard_normal((1, n, c.r_k))
        UK = rng.standard_normal((c.T, 1, c.d_h, c.r_k)) / math.sqrt(c.r_k)
        UV = rng.standard_normal((c.T, 1, c.d_h, c.r_k)) / math.sqrt(c.r_k)
        q = rng.standard_normal((c.T, 1, c.d_h))
        wk = rng.standard_normal((c.T, 1, 1, c.d_h))
        wv = rng.standard_normal((c.T, 1, 1, c.d_h))
        t = time.perf_counter()
        lla.decode_reconstruct(cK, cV, UK, UV, q, wk, wv, 0, c.N, 0)
        per_token = c.H * c.L
    dt = time.perf_counter() - t
    return dt, _blas_threads(), per_token


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([d.get("num_threads", 1) for d in info] or [1])
    except Exception:
        return os.cpu_count() or 1


def _slice_name(cfg):
    return "(sequence, head) slices of the single layer" if cfg.kind == "lla" else "(sequence, layer) slices"


def cpu_baseline(cfg, budget_s=12.0, budget_1thread_s=6.0):
    """The oracle on the host cores: all BLAS threads for about budget_s, then
    one thread for about budget_1thread_s (value_1thread)."""
    total, n, threads, per_token = 0.0, 0, 1, 1
    while total < budget_s and n < 512:
        dt, threads, per_token = oracle_sample(cfg, seed=5 + n)
        total += dt
        n += 1
    tok_s = n / (per_token * total)   # a decoded token needs per_token slices
    out = {"value": tok_s, "unit": "tokens/s", "cores": threads, "kind": "oracle",
           "sample": f"{n} {_slice_name(cfg)} of the {cfg.name} step (fp64 numpy), {total:.1f} s; "
                     f"tokens/s = slices / ({per_token} slices per token x time)"}
    try:
        from threadpoolctl import threadpool_limits
    except ImportError:
        return out
    t1, n1 = 0.0, 0
    with threadpool_limits(limits=1):
        while t1 < budget_1thread_s and n1 < 64:
            dt, _, per_token = oracle_sample(cfg, seed=1005 + n1)
            t1 += dt
            n1 += 1
    out["value_1thread"] = n1 / (per_token * t1)
    out["sample_1thread"] = f"{n1} {_slice_name(cfg)} on one thread, {t1:.1f} s"
    return out


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
    times, threads, per_token = [], 1, 1
    for s in range(args.steps):
        dt, threads, per_token = oracle_sample(cfg, seed=200 + s)
        times.append(dt)
    total = sum(times)
    v = args.steps / (per_token * total)
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * per_token * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": cfg.name, "mode": args.mode,
                                        "sample": f"one of the {_slice_name(cfg)} per step"},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"{args.steps} {_slice_name(cfg)} of {cfg.name}, {total:.1f} s"},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


# DRAM traffic (read + write) per latent token of the tensor-core latent read,
# from ncu captures of dram__bytes_read.sum + dram__bytes_write.sum, keyed by
# the sha256 prefix of the kernel source it was taken on (comments and blank
# lines removed, so only code changes count) and the latent row width in
# bytes: a changed kernel, or a row width never captured, reports no traffic
# (null) until it is captured again.
TC_TRAFFIC_PER_TOKEN = {("b53d89033e936583", 2304): 2429.6}


def source_key(path):
    """sha256 prefix of a source file with comments and blank lines removed."""
    import hashlib
    import re
    try:
        src = open(path).read()
    except OSError:
        return None
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    src = "\n".join(ln.strip() for ln in src.splitlines() if ln.strip())
    return hashlib.sha256(src.encode()).hexdigest()[:16]


def tc_traffic_per_token(row_bytes):
    key = source_key(os.path.join(ROOT, "looped_transformer_latent_b200", "csrc", "decode_tc.cu"))
    return TC_TRAFFIC_PER_TOKEN.get((key, row_bytes))


_DRIVER = None


def memcpy_async(dst, src, stream):
    """One cuMemcpyAsync of a dense tensor on `stream` (unified addressing:
    either side may be pinned host memory); under stream capture it becomes a
    copy node of the graph, with no host-allocator bookkeeping."""
    global _DRIVER
    if _DRIVER is None:
        import ctypes
        lib = ctypes.CDLL("libcuda.so.1")
        lib.cuMemcpyAsync.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_size_t, ctypes.c_void_p]
        lib.cuMemcpyAsync.restype = ctypes.c_int
        _DRIVER = lib
    n = src.numel() * src.element_size()
    if not (dst.is_contiguous() and src.is_contiguous()) or dst.numel() * dst.element_size() != n:
        raise ValueError("memcpy_async needs two dense tensors of the same size")
    rc = _DRIVER.cuMemcpyAsync(dst.data_ptr(), src.data_ptr(), n, stream.cuda_stream)
    if rc != 0:
        raise RuntimeError(f"cuMemcpyAsync failed with CUresult {rc}")


def reduce_max(dist, value, device):
    """Max of a per-rank float over all ranks (the value itself on one rank)."""
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="ouro_lla2d_768", choices=sorted(synth.CONFIGS))
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
    tags = step.read_tags()
    nread = len(tags)
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
    ms = reduce_max(dist, ms, dev)
    if dist is not None:
        dist.barrier()

    # end to end: every step copies its inputs from pinned host memory, runs,
    # and copies its outputs back.  One graph holds all of it: layer l's
    # inputs go up on a copy stream ahead of its compute, its outputs come
    # down on another as soon as it finishes, so the copies overlap the
    # compute of neighbouring layers.
    layers = step.layer_io()
    h_layers = [([t.detach().cpu().pin_memory() for t in li],
                 [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in lo]) for li, lo in layers]
    h2d = sum(t.numel() * t.element_size() for hi, _ in h_layers for t in hi)
    d2h = sum(t.numel() * t.element_size() for _, ho in h_layers for t in ho)
    cin, cout = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in layers]
    ev_done = [torch.cuda.Event() for _ in layers]
    fork, fin = torch.cuda.Event(), torch.cuda.Event()

    def io_hook(layer, phase):
        cur = torch.cuda.current_stream(dev)
        if phase == "begin":
            cur.wait_event(ev_in[layer])
            return
        ev_done[layer].record(cur)
        cout.wait_event(ev_done[layer])
        for hdst, d in zip(h_layers[layer][1], layers[layer][1]):
            memcpy_async(hdst, d, cout)

    e2e_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(e2e_graph, stream=stream):
        fork.record(stream)
        cin.wait_event(fork)
        cout.wait_event(fork)
        for k, (li, _) in enumerate(layers):
            for d, hsrc in zip(li, h_layers[k][0]):
                memcpy_async(d, hsrc, cin)
            ev_in[k].record(cin)
        step.run(hook=io_hook)
        fin.record(cout)
        stream.wait_event(fin)
    torch.cuda.synchronize()
    e2e_graph.replay()
    torch.cuda.synchronize()
    h_all = [t for _, ho in h_layers for t in ho]
    for h, e in zip(h_all, eager):      # the copied-back outputs are the eager step's
        if not torch.equal(h, e.cpu()):
            raise SystemExit("end-to-end step output differs from the eager step")
    for _ in range(3):
        e2e_graph.replay()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            e2e_graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = e0.elapsed_time(e1) / args.steps
    ms_e2e = reduce_max(dist, ms_e2e, dev)

    hbm, tflops, src = peaks()
    lb = step.read_latent_bytes()
    main_ix = [k for k, t in enumerate(tags) if t == "main"]
    main_ms = [split_ms[k] for k in main_ix]
    main_bytes = [lb[k] for k in main_ix]
    mean_ms = sum(main_ms) / max(1, len(main_ms))
    achieved = (sum(main_bytes) / 1e9) / (sum(main_ms) / 1e3) if sum(main_ms) > 0 else 0.0
    overlapped = getattr(step, "side", None) is not None
    if overlapped:
        # the loop-1 and main reads of a layer run concurrently: their latent
        # bytes over the union of the two latent-read kernels' intervals
        spans, nbytes = [], 0
        for k in range(0, len(evs), 2):
            (s1, e1), (s2, e2) = evs[k], evs[k + 1]
            first = s1 if s1.elapsed_time(s2) >= 0 else s2
            spans.append(max(first.elapsed_time(e1), first.elapsed_time(e2)))
            nbytes += lb[k] + lb[k + 1]
        mean_ms = sum(spans) / max(1, len(spans))
        achieved = (nbytes / 1e9) / (sum(spans) / 1e3) if sum(spans) > 0 else 0.0
    all_gbs = (sum(lb) / 1e9) / (sum(split_ms) / 1e3) if sum(split_ms) > 0 else 0.0
    per_tok = (tc_traffic_per_token((cfg.r_k + cfg.r_v) * 2)
               if cfg.kind != "lla" and cfg.lat_dtype == "bf16" else None)
    traffic = None
    if per_tok is not None and main_ix:
        traffic = per_tok * cfg.B * step.n_lat
        if overlapped:   # both reads per span: loop-1 rows are half as wide (same kernel, same traffic ratio)
            traffic *= 1.0 + (2.0 * cfg.r_1) / (cfg.r_k + cfg.r_v)
    step_bytes = step.step_bytes()
    tokens = cfg.B * world
    srt = sorted(main_ms)
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
        "dtype": "fp8-e4m3 latents, bf16/f16 tensor-core operands" if cfg.lat_dtype == "fp8" else "bf16",
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
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm,
                     "unit": "GB/s", "frac": achieved / hbm, "traffic": traffic,
                     "kernel": ("tensor-core latent read (absorb_split_tc), loop-1 and main launches of each "
                                "layer running concurrently" if overlapped else
                                "tensor-core latent read of fp8 rows (absorb_split_fp8), main-latent launches"
                                if cfg.lat_dtype == "fp8" else
                                "tensor-core latent read (absorb_split_tc), main-latent launches"),
                     "peak_source": src, "per_launch_ms": mean_ms,
                     "per_launch_ms_min_med_max": [srt[0], srt[len(srt) // 2], srt[-1]] if srt else None,
                     "launches_per_step": 2 * len(main_ix) if overlapped else len(main_ix),
                     "algorithmic_bytes_per_launch": (sum(main_bytes) / max(1, len(main_bytes))),
                     "all_latent_reads_gbs": all_gbs,
                     "timing": ("CUDA events around each latent-read kernel in the captured step, read after the "
                                "last replay of the timed region; with the two reads of a layer concurrent, "
                                "achieved = both reads' latent bytes / the union of their kernel intervals "
                                "(per_launch_ms = that span)" if overlapped else
                                "CUDA events around each latent-read kernel in the captured step, "
                                "read after the last replay of the timed region")},
    }
    if cfg.kind == "lla":
        # reconstruct-on-read rebuilds k^ and v^ for every latent token, loop
        # and head on the tensor cores: 2*d_h*r flops each, plus 2*d_h for the
        # score and 2*d_h for the weighted sum (algorithmic count: one product
        # per term, rank and head dimension unpadded).  Peak: the measured dense
        # bf16 rate of this machine's B200s.
        flops = cfg.B * cfg.T * cfg.H * step.n_lat * (4.0 * cfg.d_h * cfg.r_k + 4.0 * cfg.d_h)
        tf = flops / 1e12 / (mean_ms / 1e3) if mean_ms > 0 else 0.0
        line["roofline"] = {"bound": "tensor", "achieved": tf, "peak": tflops, "unit": "TFLOP/s",
                            "frac": tf / tflops, "traffic": None,
                            "kernel": "LLA reconstruct-on-read (recon_group_tc)",
                            "peak_source": src + " (dense bf16)", "per_launch_ms": mean_ms,
                            "flops_per_launch": flops, "latent_gbs": achieved,
                            "launches_per_step": len(main_ix),
                            "fp32_alu_equivalent_frac": tf / (148 * 128 * 2 * ((clocks or {}).get("sm_max_mhz") or 1965.0) * 1e6 / 1e12)}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg)
    if rank == 0:
        print(json.dumps(line))
    del graph, e2e_graph
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
