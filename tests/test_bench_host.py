"""Host-side logic of bench.py: the max-over-ranks timing with two gloo ranks on CPU,
the JSON config and the peak-table fallback (no GPU needed)."""
import json
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    r, local, ws = bench.dist_init("gloo")
    t = bench.max_over_ranks(10.0 + 5 * rank)  # rank 1 is the slow one
    bench.barrier()
    q.put((r, ws, t))
    torch.distributed.destroy_process_group()


def test_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out == [(0, 2, 15.0), (1, 2, 15.0)]


def test_single_process_is_identity():
    assert bench.max_over_ranks(3.5) == 3.5


def test_config_and_peaks():
    c = bench.config_dict()
    assert c["M"] == 8192 and c["N"] == 14336 and c["K"] == 4096 and c["hadamard"] == 16
    assert "workload" in c and "l2" in c
    json.dumps(c)
    peaks, src = bench.load_peaks()
    assert src in ("measured", "fallback") and peaks["hbm_gbs"] > 1000


def test_reference_arm_other_ranks_exit_without_work(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        steps, warmup = 1, 0
    assert bench.reference_arm(A()) == 0


def _run_bench(args, env_extra=None, timeout=180):
    import subprocess
    import sys
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR",
                                                            "MASTER_PORT", "LOCAL_WORLD_SIZE")}
    env.update(env_extra or {})
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "bench.py")
    return subprocess.run([sys.executable, path, *args], capture_output=True, text=True, timeout=timeout, env=env)


def test_gpus_flag_self_launches_two_gloo_ranks():
    # --gpus 2 without a launcher: bench.py re-runs itself under torch.distributed.run with two
    # ranks; the launch check joins them over gloo and rank 0 reports the world size
    r = _run_bench(["--gpus", "2", "--launch-check"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]
    assert lines == [{"launch_check": True, "n_gpus": 2, "max_rank": 1.0}]


def test_gpus_flag_disagreeing_with_world_size_fails():
    r = _run_bench(["--gpus", "2", "--launch-check"], {"WORLD_SIZE": "1", "RANK": "0", "LOCAL_RANK": "0"})
    assert r.returncode != 0 and "WORLD_SIZE" in r.stderr
