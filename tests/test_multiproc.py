"""Multi-process paths on CPU (gloo, world size 2). The layer does not shard:
N GPUs run N replicas and the benchmark reports the bytes of all replicas
over the slowest rank's time; the reference arm runs on rank 0 only."""
import argparse
import datetime
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    import bench
    t = bench.dist_max(1.5 + rank, torch.device("cpu"), ws)
    b = bench.dist_sum(10.0 * (rank + 1), torch.device("cpu"), ws)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, t, b))


def test_replica_reductions_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, b in out:
        assert t == 2.5          # slowest rank's time
        assert b == 30.0         # bytes of both replicas


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.run_reference(argparse.Namespace(steps=1, warmup=3, gpus=2))
    assert capsys.readouterr().out == ""


def test_reference_arm_loads_only_the_oracle():
    # rank 0 of the reference arm on a small layer: one JSON line with the workload's config, and no
    # product module or library in the process
    import json
    import subprocess
    code = (
        "import sys, argparse, dataclasses, json; sys.path.insert(0, %r)\n"
        "import bench\n"
        "from synth import workloads as wl\n"
        "bench.MAIN_SPEC = dataclasses.replace(wl.DECODE_D2K256, E=16, hidden=512, inter=256, name='small')\n"
        "bench.MAIN_T = 4\n"
        "bench.run_reference(argparse.Namespace(steps=2, warmup=3, gpus=1))\n"
        "assert 'vector_quantized_moe_b200' not in sys.modules\n"
        "maps = open('/proc/self/maps').read()\n"
        "assert 'libvqmoe' not in maps and 'libvqoracle' in maps\n" % ROOT)
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["config"]["workload"] == "small" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"

