"""Host-side logic of bench.py on CPU: the max-over-ranks timing reduction on
two gloo ranks, whole-job throughput, and the reference arm (the fp64 oracle)
being run by rank 0 only."""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank's "step time" differs; every rank must see the slowest
        got = bench.reduce_max(dist, 1.5 + rank, torch.device("cpu"))
        out_q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_reduce_max_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=600)   # spawned ranks import torch; slow on a loaded host
        assert p.exitcode == 0
    got = dict(q.get(timeout=60) for _ in range(2))
    assert got == {0: 2.5, 1: 2.5}


def test_reduce_max_single_process_is_identity():
    assert bench.reduce_max(None, 3.25, torch.device("cpu")) == 3.25


def _run_reference(env_extra, cfg="tiny_hla"):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--config", cfg, "--steps", "1", "--warmup", "3"],
                          capture_output=True, text=True, env=env, timeout=300)


def test_reference_arm_rank0_prints_one_line():
    r = _run_reference({"RANK": "0", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_silently():
    r = _run_reference({"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


@pytest.mark.parametrize("cfg", ["ouro_hla_4k", "ouro_lla2d_768", "huginn_lla_4k", "ouro_hla_16k"])
def test_traffic_table_keys_row_width(cfg):
    c = bench.synth.CONFIGS[cfg]
    v = bench.tc_traffic_per_token((c.r_k + c.r_v) * 2)
    assert v is None or v >= (c.r_k + c.r_v) * 2 * 0.9
