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


def test_bench_byte_counts_match_the_oracle_and_the_library():
    """The bytes bench.py divides by (its GB/s) are the format's algorithmic
    bytes as the oracle defines them, and the decode step's total is the sum
    over its 224 projections; the library's image for INT4 adds only padding
    and a header on top of them."""
    sys.path.insert(0, ROOT)
    import bench
    import workloads
    import bit_weight_only_pack_b200 as lbq
    from oracle import int4, lut3
    for K, N, g, mode in [(4096, 4096, 32, "sym"), (4096, 14336, 32, "asym"), (8192, 28672, 128, "sym"),
                          (14336, 4096, 64, "asym")]:
        assert bench.int4_bytes(K, N, g, mode) == int4.algorithmic_bytes(K, N, g, mode)
        assert lbq.lbq_packed_size(K, N, g, 0 if mode == "sym" else 1) >= bench.int4_bytes(K, N, g, mode)
    assert bench.lut3_bytes(4096, 14336) == lut3.algorithmic_bytes(4096, 14336)
    step = 32 * sum(int4.algorithmic_bytes(K, N, 32, "asym") for _, K, N in workloads.LLAMA3_8B_PROJ)
    assert step == 4143972352


def test_profile_summaries_name_commands_that_exist():
    """Every summary under profiles/ gives the command that made it, and that
    command runs committed files only: bench.py with a profile case it defines
    or with flags its parser accepts."""
    import glob
    import re
    sys.path.insert(0, ROOT)
    import bench
    files = sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md")))
    assert files
    for path in files:
        text = open(path).read()
        cmds = re.findall(r"python bench\.py[^\n`]*", text)
        assert cmds, f"{os.path.basename(path)} gives no command"
        for cmd in cmds:
            m = re.search(r"--profile (\S+)", cmd)
            if m:
                assert m.group(1) in bench.PROFILE_CASES, (path, m.group(1))
            for flag in re.findall(r"(--[a-z-]+)", cmd):
                assert flag in ("--profile", "--steps", "--warmup", "--no-secondary", "--no-cpu-baseline",
                                "--gpus", "--impl", "--quick", "--ungrouped", "--no-pdl", "--layers"), (path, flag)


def test_profile_commands_stay_within_the_capture_rules():
    """Every ncu command under profiles/ either records launch times only
    (gpu__time_duration.sum) or captures one kernel (-k) for at most three
    launches (-c); none collects more over a whole run."""
    import glob
    import re
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        text = open(path).read().replace("\\\n", " ")
        for cmd in re.findall(r"^\s*ncu [^\n`]*", text, flags=re.M):
            assert "--clock-control none" in cmd, (path, cmd)
            m = re.search(r"--metrics (\S+)", cmd)
            times_only = m is not None and m.group(1) == "gpu__time_duration.sum" and "--set" not in cmd \
                and "--section" not in cmd
            if times_only:
                continue
            assert re.search(r"-k (regex:)?\S+", cmd), (path, cmd)
            c = re.search(r"-c (\d+)", cmd)
            assert c and int(c.group(1)) <= 3, (path, cmd)


def test_step_traffic_records_are_consistent():
    """The decode step's traffic figure is reported only when every launch
    shape has a record taken with the current kernel sources and planner, and
    every record names a committed summary."""
    sys.path.insert(0, ROOT)
    import bench
    assert set(bench.STEP_TRAFFIC) == {"c2qkv", "c2o", "c2gateup", "c2down"}
    for name, (nbytes, sources, summary) in bench.STEP_TRAFFIC.items():
        assert name in bench.PROFILE_CASES
        assert os.path.exists(os.path.join(ROOT, summary)) or nbytes is None, summary
        if nbytes is not None:
            assert set(sources) == set(bench.STEP_SOURCES)
    now = bench.current_hashes()
    assert all(v is not None for v in now.values())
    complete = all(r[0] is not None and r[1] == now for r in bench.STEP_TRAFFIC.values())
    assert (bench.traffic_from_profiles() is not None) == complete


def test_profile_cases_are_the_shapes_they_name():
    """Every profile case is a shape the library takes (K a multiple of 64 and
    at most 65536, N positive, M in 1 .. 8192), and the decode step's cases
    have the step's shapes (K = 4096, or 14336 for down)."""
    sys.path.insert(0, ROOT)
    import bench
    for name, case in bench.PROFILE_CASES.items():
        K, N, group, mode, xdt, M = case[:6]
        assert K % 64 == 0 and 64 <= K <= 65536, (name, K)
        Ns = N if isinstance(N, tuple) else (N,)
        assert all(0 <= n <= 1 << 20 for n in Ns), (name, N)
        assert 1 <= M <= 8192, (name, M)
    step = {"c2qkv": (4096, (4096, 1024, 1024)), "c2o": (4096, 4096), "c2gateup": (4096, (14336, 14336)),
            "c2down": (14336, 4096)}
    for name, (K, N) in step.items():
        assert tuple(bench.PROFILE_CASES[name][:2]) == (K, N), name
    # the step's traffic records: mean bytes per launch within 1% of the algorithmic bytes
    mean = sum(r[0] for r in bench.STEP_TRAFFIC.values()) / len(bench.STEP_TRAFFIC)
    assert abs(mean / 32374784 - 1.0) < 0.01
