"""The multi-rank path of bench.py on the CPU: the timing maximum over two gloo ranks, and the
reference arm under WORLD_SIZE=2 (rank 0 alone runs and prints; rank 1 exits without work).
Replicas only: the decode path itself has no collective."""
import importlib.util
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        b = _bench()
        # rank r reports (r + 1, 10 - r, 0.5 r): the maximum takes each entry's largest
        got = b.max_over_ranks([rank + 1.0, 10.0 - rank, 0.5 * rank], dist, torch.device("cpu"))
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(2, _free_port(), out), nprocs=2, join=True,
                       start_method="spawn")
    assert out[0] == [2.0, 10.0, 0.5]
    assert out[1] == [2.0, 10.0, 0.5]


def test_max_over_ranks_single_process():
    import torch
    assert _bench().max_over_ranks([3, 1.5], None, torch.device("cpu")) == [3.0, 1.5]


def _reference(rank):
    env = dict(os.environ, WORLD_SIZE="2", RANK=str(rank), LOCAL_RANK=str(rank),
               MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--config", "tiny", "--steps", "1", "--warmup", "3"],
                          env=env, capture_output=True, text=True, timeout=300)


def test_reference_arm_runs_on_rank0_only():
    r1 = _reference(1)
    assert r1.returncode == 0, r1.stderr[-2000:]
    assert r1.stdout.strip() == ""
    r0 = _reference(0)
    assert r0.returncode == 0, r0.stderr[-2000:]
    lines = [l for l in r0.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["config"]["workload"] == "tiny"
    assert d["cpu_baseline"]["kind"] == "oracle"
