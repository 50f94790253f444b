"""Host-side checks of the benchmark harness: the replica (N > 1) timing
reduction over a real process group (gloo, world size 2, on CPU), the
throughput formula, and the reference arm's rank handling."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    # each rank measured a different time; the job's time is the slowest
    t = bench.max_over_ranks(10.0 + 5.0 * rank, dist, torch.device("cpu"))
    v = bench.job_throughput(1000, world, t)
    out.put((rank, t, v))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 2000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, v in res:
        assert t == 15.0                       # max over ranks, seen by every rank
        assert v == pytest.approx(2 * 1000 / 0.015)


def test_single_process_reduction_is_identity():
    assert bench.max_over_ranks(3.5, None, torch.device("cpu")) == 3.5
    assert bench.job_throughput(100, 1, 1000.0) == pytest.approx(100.0)


def test_reference_arm_nonzero_rank_exits_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "2", "--warmup", "1"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_prints_one_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "3", "--warmup", "1"], env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["metric"] == bench.METRIC


def test_source_hash_ignores_comments_only():
    """The ncu traffic record stays valid across comment edits and is retired
    by any change to the code itself."""
    import bench
    src = 'int f(int a) { // add one\n  return a + 1; /* done */ }\nconst char* s = "// kept";\n'
    assert bench.code_only(src) == bench.code_only(src.replace("add one", "increment"))
    assert bench.code_only(src) != bench.code_only(src.replace("a + 1", "a + 2"))
    assert "// kept" in bench.code_only(src)
    assert "add one" not in bench.code_only(src) and "done" not in bench.code_only(src)


def test_graph_plan_runs_exactly_the_requested_cycles():
    for steps in (0, 1, 5, 14, 15, 16, 20, 29, 30, 31, 59, 60, 61, 75, 20000):
        plan = bench.graph_plan(steps, 15)
        assert sum(c * r for c, r in plan) == steps
        assert len(plan) <= 2 and all(c >= 1 and r >= 1 for c, r in plan)
    assert bench.graph_plan(20, 15) == [(20, 1)]
    assert bench.graph_plan(61, 15) == [(15, 4), (1, 1)]


def test_e2e_counts_follow_steps_with_a_floor():
    assert bench.e2e_counts(20, 5) == (bench.E2E_MIN_CYCLES, bench.E2E_MIN_WARMUP)
    assert bench.e2e_counts(200, 40) == (200, 40)


def test_parse_cpulist():
    """The sysfs cpulist format of a PCI device's local CPUs."""
    assert bench.parse_cpulist("0-3,8,10-11\n") == {0, 1, 2, 3, 8, 10, 11}
    assert bench.parse_cpulist("5") == {5}
    assert bench.parse_cpulist("\n") == set()


def test_pci_locality_reads_sysfs_and_intersects(tmp_path):
    """The e2e leg's host-buffer placement: the GPU's NUMA node and its CPUs
    among those this process may use; nothing when sysfs does not say."""
    (tmp_path / "numa_node").write_text("1\n")
    (tmp_path / "local_cpulist").write_text("8-15,24\n")
    assert bench.pci_locality(str(tmp_path), {0, 8, 9, 24, 30}) == (1, {8, 9, 24})
    assert bench.pci_locality(str(tmp_path / "missing"), {0, 1}) == (None, set())
    (tmp_path / "numa_node").write_text("-1\n")
    assert bench.pci_locality(str(tmp_path), range(32))[0] == -1
