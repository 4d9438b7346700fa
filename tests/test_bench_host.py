"""Host-side logic of bench.py's multi-process launch, on CPU with gloo:
rank / world discovery, the barrier, the max over ranks that makes a
multi-GPU timing, and the reference arm leaving all work to rank 0."""

import os
import socket
import sys

import pytest

from conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, values, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), LOCAL_RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch
    import bench
    w, r, local = bench.dist_setup("gloo")
    try:
        bench.barrier(w)
        got = bench.max_over_ranks(w, values[r])
        bench.barrier(w)
        out.put((r, w, local, got))
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.parametrize("values", [(1.5, 7.25), (9.0, -3.0)])
def test_max_over_ranks_world_size_two(values):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, values, out)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[:3] for r in results] == [(0, 2, 0), (1, 2, 1)]
    assert all(r[3] == max(values) for r in results)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")

    class Args:
        gpus, steps, warmup = 2, 3, 3

    assert bench.run_reference(Args()) == 0
    assert capsys.readouterr().out == ""


def test_single_process_needs_no_group(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_setup("gloo") == (1, 0, 0)
    assert bench.max_over_ranks(1, 4.0) == 4.0
