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
