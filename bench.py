#!/usr/bin/env python
"""Benchmark: block-hybrid attention, active-block tokens/s per layer on B200.

Workload (default): the long-prefix regime of a 16B dLLM attention layer --
batch 64, 16 query / 4 KV heads, head dim 128, active block B = 32, a
committed prefix of 32768 tokens folded into the fp32 prefix state by the
GPU prefill.  One timed step is one block of the decoding loop: 8 denoising
steps (bha_hybrid_step) followed by the block commit (bha_state_commit);
tokens per step = batch x B x 8 active-block tokens.  Inputs are resident in
HBM; 14+ disjoint input sets rotate so the working set exceeds 4 x L2.  The
timed loop replays CUDA graphs of the library's launches.

Printed: one JSON line (rank 0) with the metric, the roofline of the
dominant kernel, the CPU-oracle baseline, the end-to-end number through the
C ABI with host buffers, the exact-prefix-softmax comparison on identical
shapes and the SM clocks sampled during the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
"""
import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "hybrid-attn active-block tokens/s per layer at 1 B200; % of HBM roofline"
DATA = ("synthetic: seeded Gaussian bf16 Q/K/V, N(0, std 1/sqrt(128)); prefix state from "
        "the GPU prefill of a seeded 32768-token prompt (stands in for trained-model "
        "activations; timing does not depend on values)")
N_, HQ, HKV, B_, D_, P_ = 64, 16, 4, 32, 128, 32768
DENOISE = 8
UNIT_BYTES_STEP = (HQ // HKV) * B_ * D_ * 2 * 2 + 2 * B_ * D_ * 2 + D_ * D_ * 4  # Q+Y, K+V, S
UNIT_BYTES_COMMIT = 2 * B_ * D_ * 2 + 2 * D_ * D_ * 4                           # K+V, S r+w
UNIT_BYTES_FUSED = UNIT_BYTES_STEP + D_ * D_ * 4                                # + S write
UNIT_BYTES_SHARED = UNIT_BYTES_STEP + D_ * 4                                     # + z read
WORKLOAD = ("long-prefix: batch 64, 16q/4kv heads, d=128, active block B=32, prefix 32768 "
            "in fp32 state; step = one block: 8 hybrid denoising steps, the last fused with "
            "the block commit")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline")
    ap.add_argument("--no-compare", action="store_true", help="skip the exact-path comparison")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the secondary workloads in the benchmark line")
    ap.add_argument("--only", choices=["step", "step_shared", "step_commit", "commit", "prefill",
                                       "prefix", "paged", "reuse"],
                    help="launch just this kernel warmup + steps times (small case for ncu)")
    ap.add_argument("--prefix", type=int, default=8192,
                    help="prompt / cache length used by --only prefill|prefix")
    ap.add_argument("--batch", type=int, default=None,
                    help="batch used by --only step|step_commit|commit (default 64)")
    ap.add_argument("--workload", default="long-prefix",
                    choices=["long-prefix", "single-step", "generation-loop", "stack",
                             "feature-maps", "ragged", "reuse"],
                    help="long-prefix is the benchmark line; the others are the secondary "
                         "workloads (one JSON line each)")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def code_only(text):
    """C/C++ source without its comments, whitespace runs collapsed: what the
    compiler sees, so that editing a comment does not retire a capture."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def source_sha256(src_file):
    """sha256 over the code (comments aside) of a kernel's source file and of
    the device helpers it includes."""
    h = hashlib.sha256()
    for name in (src_file, "bha_ptx.cuh"):
        with open(os.path.join(ROOT, "block_hybrid_linear_b200", "csrc", name)) as f:
            h.update(code_only(f.read()).encode())
    return h.hexdigest()


def traffic_record(kernel, src_file):
    """dram bytes per launch from the committed ncu summary, if the kernel's
    source is unchanged since the capture (else None)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel)
    if not rec or rec.get("source_sha256") != source_sha256(src_file):
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.out = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.QUERY,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def max_over_ranks(value, dist, device):
    """Largest `value` across the process group (the job's time is the
    slowest rank's); `dist` is torch.distributed or None for one process."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def graph_plan(steps, cycles_per_graph):
    """CUDA-graph replays that run exactly `steps` block cycles: a list of
    (cycles in the graph, replays).  Up to 4 rotation periods run as one
    graph of exactly `steps` cycles; beyond that, replays of the graph of one
    period and one graph of the remainder (every graph boundary costs a
    launch gap, so there are at most two graphs)."""
    steps = max(0, int(steps))
    if steps == 0:
        return []
    if steps <= 4 * cycles_per_graph:
        return [(steps, 1)]
    plan = [(cycles_per_graph, steps // cycles_per_graph)]
    if steps % cycles_per_graph:
        plan.append((steps % cycles_per_graph, 1))
    return plan


E2E_MIN_CYCLES, E2E_MIN_WARMUP = 50, 10


def e2e_counts(steps, warmup):
    """Timed and warm-up block cycles of the end-to-end leg: --steps and
    --warmup, floored at 50 and 10 (30 timed cycles after 3 warm-up cycles
    under-measured the copies: 5.4e6 tokens/s where 50 after 3 gave 8.5e6)."""
    return max(E2E_MIN_CYCLES, int(steps)), max(E2E_MIN_WARMUP, int(warmup))


def parse_cpulist(text):
    """CPU numbers of a sysfs cpulist ("0-3,8,10-11" -> {0, 1, 2, 3, 8, 10, 11})."""
    cpus = set()
    for part in text.strip().split(","):
        if not part:
            continue
        lo, _, hi = part.partition("-")
        cpus.update(range(int(lo), int(hi or lo) + 1))
    return cpus


def pci_locality(path, allowed):
    """(NUMA node, CPUs of that node among `allowed`) of the PCI device whose
    sysfs folder is `path`; (None, set()) when the platform does not say."""
    try:
        with open(os.path.join(path, "numa_node")) as f:
            node = int(f.read())
        with open(os.path.join(path, "local_cpulist")) as f:
            cpus = parse_cpulist(f.read())
    except (OSError, ValueError):
        return None, set()
    return node, cpus & set(allowed)


def gpu_host_locality(dev):
    """pci_locality of the GPU's PCI device, for the CPUs this process may use."""
    import torch
    p = torch.cuda.get_device_properties(dev)
    path = "/sys/bus/pci/devices/%04x:%02x:%02x.0" % (p.pci_domain_id, p.pci_bus_id,
                                                       p.pci_device_id)
    return pci_locality(path, os.sched_getaffinity(0))


def job_throughput(tokens_per_rank, world, time_ms):
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * world / (time_ms / 1e3)


# ---------------------------------------------------------------- reference

def run_reference(args, rank, world):
    """The CPU oracle as the reference arm: the same metric on bounded samples
    of the same workload, on the host cores.  A step's sample shrinks (whole
    requests -> query heads x denoising steps) so that K + W steps stay
    within about two minutes."""
    if rank != 0:
        return
    import oracle
    from block_hybrid_linear_b200 import inputs
    cores = len(os.sched_getaffinity(0))
    oracle.set_threads(cores)
    std = 1.0 / math.sqrt(D_)
    nmax = 16
    _, Qv = inputs.normal_bf16_np(4000, inputs.TID_Q, (nmax, HQ, B_, D_), std)
    _, Kv = inputs.normal_bf16_np(4000, inputs.TID_K, (nmax, HKV, B_, D_), std)
    _, Vv = inputs.normal_bf16_np(4000, inputs.TID_V, (nmax, HKV, B_, D_), std)
    Sv, zv = inputs.synthetic_state_np(4000, nmax, HKV, D_, P_, std)
    G = HQ // HKV

    def full_cycle(nreq):
        for _ in range(DENOISE):
            oracle.hybrid_step(Qv[:nreq], Kv[:nreq], Vv[:nreq], Sv[:nreq], zv[:nreq])
        oracle.state_commit(Sv[:nreq], zv[:nreq], Kv[:nreq], Vv[:nreq])

    def head_steps(hs, ns):
        # hs query heads of request 0 (sharing KV head 0 while hs <= G), ns steps
        hkv = 1 if hs <= G else hs // G
        for _ in range(ns):
            oracle.hybrid_step(Qv[:1, :hs], Kv[:1, :hkv], Vv[:1, :hkv], Sv[:1, :hkv],
                               zv[:1, :hkv])

    budget = min(1.0, 120.0 / max(1, args.steps + args.warmup))
    t0 = time.perf_counter()
    full_cycle(1)
    t_req = time.perf_counter() - t0
    if t_req <= budget:
        nreq = int(min(nmax, max(1, budget // max(t_req, 1e-9))))
        work = lambda: full_cycle(nreq)
        tokens_per_step = nreq * B_ * DENOISE
        sample = ("%d of 64 requests (16 query / 4 KV heads each) through one block cycle "
                  "per step: 8 oracle hybrid steps + 1 oracle commit, fp64" % nreq)
    else:
        t0 = time.perf_counter()
        head_steps(1, 1)
        t_hs = max(time.perf_counter() - t0, 1e-9)
        k = int(max(1, min(HQ * DENOISE, budget // t_hs)))
        ns = min(DENOISE, k)
        hs = max(1, min(G, k // ns))
        work = lambda: head_steps(hs, ns)
        tokens_per_step = hs / HQ * B_ * ns
        sample = ("%d of 16 query heads of one request x %d of 8 denoising steps per step "
                  "(oracle hybrid step, fp64; counted as %.3g active tokens)"
                  % (hs, ns, tokens_per_step))
    for _ in range(args.warmup):
        work()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        work()
    dt = time.perf_counter() - t0
    value = tokens_per_step * args.steps / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": DATA,
        "config": {"workload": WORKLOAD, "sample": sample},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline_native():
    """The oracle on this host's cores, on bounded samples (about 20 s in all):
    the block cycle on all cores (the reported value) and on one thread, and,
    per batch row (one request: 4 KV heads, 16 query heads), the 32768-token
    prefill and the exact path over a 32768-token cache on all cores."""
    import oracle
    from block_hybrid_linear_b200 import inputs
    cores = len(os.sched_getaffinity(0))
    std = 1.0 / math.sqrt(D_)
    nreq = 16
    Qb, Qv = inputs.normal_bf16_np(4000, inputs.TID_Q, (nreq, HQ, B_, D_), std)
    Kb, Kv = inputs.normal_bf16_np(4000, inputs.TID_K, (nreq, HKV, B_, D_), std)
    Vb, Vv = inputs.normal_bf16_np(4000, inputs.TID_V, (nreq, HKV, B_, D_), std)
    Sv, zv = inputs.synthetic_state_np(4000, nreq, HKV, D_, P_, std)

    def cycles_for(nr, seconds, max_cycles):
        t0 = time.perf_counter()
        cycles = 0
        while True:
            for _ in range(DENOISE):
                oracle.hybrid_step(Qv[:nr], Kv[:nr], Vv[:nr], Sv[:nr], zv[:nr])
            oracle.state_commit(Sv[:nr], zv[:nr], Kv[:nr], Vv[:nr])
            cycles += 1
            if time.perf_counter() - t0 > seconds or cycles >= max_cycles:
                break
        return cycles, time.perf_counter() - t0

    oracle.set_threads(cores)
    cycles, dt = cycles_for(nreq, 8.0, 50)
    out = {"value": nreq * B_ * DENOISE * cycles / dt, "unit": "tokens/s", "cores": cores,
           "kind": "oracle",
           "sample": "%d of 64 requests x %d block cycles (8 steps + commit), fp64 oracle, "
                     "%.1f s on %d threads" % (nreq, cycles, dt, cores)}
    oracle.set_threads(1)
    c1, dt1 = cycles_for(1, 4.0, 50)
    out["single_thread"] = {"value": B_ * DENOISE * c1 / dt1, "unit": "tokens/s", "cores": 1,
                            "sample": "1 of 64 requests x %d block cycles, %.1f s" % (c1, dt1)}
    # per row: one request of the long-prefix workload
    oracle.set_threads(cores)
    _, Kp = inputs.normal_bf16_np(4001, inputs.TID_KP, (1, HKV, P_, D_), std)
    _, Vp = inputs.normal_bf16_np(4001, inputs.TID_VP, (1, HKV, P_, D_), std)
    t0 = time.perf_counter()
    oracle.state_prefill(Kp, Vp)
    out["per_row_prefill_32k_s"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.prefix_softmax(Qv[:1], Kp, Vp, P_, Kv[:1], Vv[:1])
    out["per_row_exact_32k_s"] = time.perf_counter() - t0
    out["per_row_note"] = ("per-row: one request (4 KV heads, 16 query heads x 32 active "
                           "tokens) with a 32768-token prompt / cache, fp64 oracle on %d "
                           "threads; per_row_exact_32k_s is one denoising step of the exact "
                           "path" % cores)
    return out


# ---------------------------------------------------------------- native

def same_bytes_copy(nbytes, R, stream, dev, peak):
    """Per-launch time of ``dst.copy_(src)`` moving ``nbytes`` (read + write)
    over R rotating buffer pairs, 4 R launches per graph replay."""
    import torch
    n = nbytes // 4
    src = [torch.ones(n, dtype=torch.bfloat16, device=dev) for _ in range(R)]
    dst = [torch.empty_like(x) for x in src]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for k in range(4 * R):
            dst[k % R].copy_(src[k % R])
    for _ in range(3):
        g.replay()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(10):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / (10 * 4 * R)
    gbs = 4 * n / (us / 1e6) / 1e9
    del g
    return {"launch_us": us, "achieved_gbs": gbs, "frac_of_peak": gbs / peak}


def run_native(args, rank, world, local):
    import torch
    import block_hybrid_linear_b200 as bha
    from block_hybrid_linear_b200 import build, inputs

    build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist
    std = 1.0 / math.sqrt(D_)
    seed = 4000 + 17 * rank
    props = torch.cuda.get_device_properties(dev)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20))

    def barrier():
        if pg is not None:
            pg.barrier()

    # ---- prompt -> prefix state (prefill), timed as a side line
    Kp = inputs.normal_bf16_torch(seed, inputs.TID_KP, (N_, HKV, P_, D_), std, dev)
    Vp = inputs.normal_bf16_torch(seed, inputs.TID_VP, (N_, HKV, P_, D_), std, dev)
    S0 = torch.empty(N_, HKV, D_, D_, device=dev)
    z0 = torch.empty(N_, HKV, D_, device=dev)
    need = bha.bha_state_prefill_workspace_size(N_, HKV, P_, D_)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    bha.bha_state_prefill(Kp, Vp, S0, z0, workspace=ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 5
    e0.record()
    for _ in range(reps):
        bha.bha_state_prefill(Kp, Vp, S0, z0, workspace=ws)
    e1.record()
    torch.cuda.synchronize()
    prefill_ms = e0.elapsed_time(e1) / reps
    prefill_bytes = N_ * HKV * (2 * P_ * D_ * 2 + D_ * D_ * 4)

    # ---- rotating input sets (disjoint memory, > 4 x L2 in total)
    set_bytes = N_ * HKV * UNIT_BYTES_STEP
    R = max(4, math.ceil(4 * l2 / set_bytes))
    sets = []
    for r in range(R):
        sets.append(dict(
            Q=inputs.normal_bf16_torch(seed + r, inputs.TID_Q, (N_, HQ, B_, D_), std, dev),
            K=inputs.normal_bf16_torch(seed + r, inputs.TID_K, (N_, HKV, B_, D_), std, dev),
            V=inputs.normal_bf16_torch(seed + r, inputs.TID_V, (N_, HKV, B_, D_), std, dev),
            S=S0.clone(), z=z0.clone(),
            Y=torch.empty(N_, HQ, B_, D_, dtype=torch.bfloat16, device=dev)))
    torch.cuda.synchronize()

    stream = torch.cuda.Stream(device=dev)

    def cycle(c):
        # one block: 8 denoising steps on 8 different sets; the last one also
        # commits the block (the fused step + commit kernel)
        for s in range(DENOISE - 1):
            st = sets[(c * DENOISE + s) % R]
            bha.bha_hybrid_step(st["Q"], st["K"], st["V"], st["S"], st["Y"], z=st["z"],
                                stream=stream)
        st = sets[(c * DENOISE + DENOISE - 1) % R]
        bha.bha_hybrid_step_commit(st["Q"], st["K"], st["V"], st["S"], st["Y"], z=st["z"],
                                   stream=stream)

    # graphs of whole block cycles (every set is touched in each role, rotation
    # period R), so that exactly --steps cycles are timed (graph_plan)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for c in range(2):
            cycle(c)
        st = sets[0]   # (each kernel variant runs once before any capture)
        bha.bha_hybrid_step(st["Q"], st["K"], st["V"], st["S"], st["Y"], z=st["z"],
                            flags=bha.BHA_FLAG_SHARED_DENOM, stream=stream)
    stream.synchronize()
    g_cycles = R
    steps, warmup = max(1, args.steps), max(0, args.warmup)
    graphs = {}
    for ncyc, _ in graph_plan(steps, g_cycles) + graph_plan(warmup, g_cycles):
        if ncyc not in graphs:
            g1 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g1, stream=stream):
                for c in range(ncyc):
                    cycle(c)
            graphs[ncyc] = g1
    # kernel-only graphs for the per-launch durations of the kernels
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step, stream=stream):
        for k in range(4 * R):
            st = sets[k % R]
            bha.bha_hybrid_step(st["Q"], st["K"], st["V"], st["S"], st["Y"], z=st["z"],
                                stream=stream)
    g_commit = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_commit, stream=stream):
        for k in range(2 * R):
            st = sets[k % R]
            bha.bha_hybrid_step_commit(st["Q"], st["K"], st["V"], st["S"], st["Y"], z=st["z"],
                                       stream=stream)
    g_shared = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_shared, stream=stream):
        for k in range(4 * R):
            st = sets[k % R]
            bha.bha_hybrid_step(st["Q"], st["K"], st["V"], st["S"], st["Y"], z=st["z"],
                                flags=bha.BHA_FLAG_SHARED_DENOM, stream=stream)
    torch.cuda.synchronize()

    torch.cuda.set_stream(stream)   # graph replays launch on the current stream

    def run_cycles(k):
        for ncyc, reps in graph_plan(k, g_cycles):
            for _ in range(reps):
                graphs[ncyc].replay()
    # The timing events: when the K cycles are one graph, they are recorded by
    # the graph itself (event-record nodes before the first and after the
    # last kernel), so that the host's graph submission, which precedes the
    # first kernel on an idle stream, is not counted as device time of the K
    # steps (measured: 2.9 us per cycle at K = 20).
    ev0 = torch.cuda.Event(enable_timing=True, external=True)
    ev1 = torch.cuda.Event(enable_timing=True, external=True)
    timed_graph = None
    if len(graph_plan(steps, g_cycles)) == 1:
        timed_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(timed_graph, stream=stream):
            ev0.record(stream)
            for c in range(steps):
                cycle(c)
            ev1.record(stream)
    # every graph is launched once before the warm-up: the first launch of an
    # instantiated graph uploads it to the device (measured: a timed region
    # holding a graph's first launch ran 0.082 ms per cycle against 0.066)
    for g_ in list(graphs.values()) + [g_step, g_commit, g_shared] + (
            [timed_graph] if timed_graph is not None else []):
        g_.replay()
    torch.cuda.synchronize()
    run_cycles(warmup)
    torch.cuda.synchronize()
    assert bha.bha_device_error(True) == 0

    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    if timed_graph is not None:
        timed_graph.replay()
    else:
        ev0.record(stream)
        run_cycles(steps)
        ev1.record(stream)
    # per-kernel durations, measured in the same run on the launching stream:
    # every replay of a kernel-only graph (60 or 30 back-to-back launches) timed
    # on its own, at least 5 replays; the mean over replays is the roofline's
    # launch time, the spread over replays is reported beside it
    kreps = max(5, math.ceil(steps / (4 * g_cycles)))

    def time_replays(g):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(kreps)]
        for a_, b_ in evs:
            a_.record(stream)
            g.replay()
            b_.record(stream)
        return evs
    ev_step, ev_commit, ev_shared = (time_replays(g_step), time_replays(g_commit),
                                     time_replays(g_shared))
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    t_ms = ev0.elapsed_time(ev1)

    def per_launch(evs, launches):
        return [a_.elapsed_time(b_) / launches for a_, b_ in evs]
    step_ms_all = per_launch(ev_step, 4 * R)
    commit_ms_all = per_launch(ev_commit, 2 * R)
    shared_ms_all = per_launch(ev_shared, 4 * R)
    step_launch_ms = sum(step_ms_all) / len(step_ms_all)
    commit_launch_ms = sum(commit_ms_all) / len(commit_ms_all)
    shared_launch_ms = sum(shared_ms_all) / len(shared_ms_all)

    def spread_us(v):
        q = sorted(x * 1e3 for x in v)
        pick = lambda f: q[min(len(q) - 1, int(round(f * (len(q) - 1))))]
        return {"p10": pick(0.1), "p50": pick(0.5), "p90": pick(0.9), "replays": len(q)}
    assert bha.bha_device_error(True) == 0
    t_ms = max_over_ranks(t_ms, pg, dev)
    value = job_throughput(steps * N_ * B_ * DENOISE, world, t_ms)

    peak, peak_kind = measured_peaks()
    step_bytes = N_ * HKV * UNIT_BYTES_STEP
    achieved = step_bytes / (step_launch_ms / 1e3) / 1e9
    fused_bytes = N_ * HKV * UNIT_BYTES_FUSED
    shared_bytes = N_ * HKV * UNIT_BYTES_SHARED
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": steps, "warmup": warmup, "ms_per_step": t_ms / steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": DATA,
        "config": {"workload": WORKLOAD, "batch": N_, "heads_q": HQ, "heads_kv": HKV,
                   "head_dim": D_, "block": B_, "prefix": P_, "denoise_steps": DENOISE,
                   "l2": "rotating %d disjoint input sets, %.0f MB > 4 x L2 (%.0f MB)"
                         % (R, R * set_bytes / 1e6, l2 / 1e6),
                   "parallelism": "replicas x%d (no collective)" % world},
        "roofline": {"bound": "hbm", "kernel": "k_step_bf16", "achieved": achieved,
                     "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_kind": peak_kind,
                     "traffic": traffic_record("k_step_bf16", "k_step.cu"),
                     "algorithmic_bytes_per_launch": step_bytes,
                     "launch_us": step_launch_ms * 1e3,
                     "launch_us_spread": spread_us(step_ms_all),
                     "shared_denom": {
                         "kernel": "k_step_bf16 (shared denominator)",
                         "launch_us": shared_launch_ms * 1e3,
                         "launch_us_spread": spread_us(shared_ms_all),
                         "algorithmic_bytes_per_launch": shared_bytes,
                         "achieved": shared_bytes / (shared_launch_ms / 1e3) / 1e9,
                         "frac": shared_bytes / (shared_launch_ms / 1e3) / 1e9 / peak,
                         "traffic": traffic_record("k_step_bf16_shared", "k_step.cu")}},
        "hbm_roofline_frac": achieved / peak,
        "step_commit": {"kernel": "k_step_bf16 (fused commit)",
                        "launch_us": commit_launch_ms * 1e3,
                        "launch_us_spread": spread_us(commit_ms_all),
                        "achieved_gbs": fused_bytes / (commit_launch_ms / 1e3) / 1e9,
                        "frac_of_peak": fused_bytes / (commit_launch_ms / 1e3) / 1e9 / peak,
                        "algorithmic_bytes_per_launch": fused_bytes,
                        "traffic": traffic_record("k_step_bf16_fused_commit", "k_step.cu")},
        "prefill": {"ms": prefill_ms, "tokens": N_ * P_,
                    "achieved_gbs": prefill_bytes / (prefill_ms / 1e3) / 1e9},
        "gpu_launches": steps * DENOISE,
        "timed_graphs": {"plan": [{"cycles": c, "replays": r}
                                  for c, r in graph_plan(steps, g_cycles)],
                         "events": "inside the graph" if timed_graph is not None
                                   else "on the stream around the replays",
                         "note": "CUDA graphs of whole block cycles, each launched once "
                                 "(uploaded) before the warm-up"},
        "clocks": clk,
    }

    # ---- calibration: the peak's own method (a torch copy, half the bytes read
    # and half written) at the step's bytes per launch, back to back in a graph
    # over rotating buffers like the step, right after it: what a plain stream
    # of this size reaches on this GPU at these clocks
    if not args.no_compare:
        line["roofline"]["same_bytes_copy"] = same_bytes_copy(step_bytes, R, stream, dev, peak)

    # ---- exact prefix softmax on identical shapes (the comparison path)
    if not args.no_compare:
        del graphs, g_step, g_commit, g_shared, timed_graph
        cap = P_ + B_
        Kc = torch.empty(N_, HKV, cap, D_, dtype=torch.bfloat16, device=dev)
        Vc = torch.empty_like(Kc)
        Kc[:, :, :P_].copy_(Kp)
        Vc[:, :, :P_].copy_(Vp)
        st = sets[0]
        Kc[:, :, P_:].copy_(st["K"])
        Vc[:, :, P_:].copy_(st["V"])
        del Kp, Vp
        need = bha.bha_prefix_softmax_workspace_size(N_, HQ, HKV, B_, D_, P_)
        wsp = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
        Yx = torch.empty_like(st["Y"])
        for _ in range(2):
            bha.bha_prefix_softmax(st["Q"], Kc, Vc, P_, st["K"], st["V"], Yx, workspace=wsp)
        torch.cuda.synchronize()
        n_rep = 10
        e0.record()
        for _ in range(n_rep):
            bha.bha_prefix_softmax(st["Q"], Kc, Vc, P_, st["K"], st["V"], Yx, workspace=wsp)
        e1.record()
        torch.cuda.synchronize()
        px_ms = e0.elapsed_time(e1) / n_rep
        px_bytes = N_ * HKV * (2 * (P_ + B_) * D_ * 2) + 2 * N_ * HQ * B_ * D_ * 2
        comp = {"prefix_softmax": {"ms": px_ms, "tokens_per_s": N_ * B_ / (px_ms / 1e3),
                                   "achieved_gbs": px_bytes / (px_ms / 1e3) / 1e9,
                                   "frac_of_peak": px_bytes / (px_ms / 1e3) / 1e9 / peak}}
        # library attention on the same shapes, as a sanity line for the exact path
        try:
            import torch.nn.functional as F
            q = st["Q"]
            for _ in range(2):
                F.scaled_dot_product_attention(q, Kc, Vc, enable_gqa=True)
            torch.cuda.synchronize()
            e0.record()
            for _ in range(n_rep):
                F.scaled_dot_product_attention(q, Kc, Vc, enable_gqa=True)
            e1.record()
            torch.cuda.synchronize()
            sd_ms = e0.elapsed_time(e1) / n_rep
            comp["torch_sdpa"] = {"ms": sd_ms, "tokens_per_s": N_ * B_ / (sd_ms / 1e3)}
        except Exception as exc:  # pragma: no cover
            comp["torch_sdpa"] = {"error": str(exc)[:200]}
        hybrid_step_ms = step_launch_ms
        comp["hybrid_step_over_exact_speedup"] = px_ms / hybrid_step_ms
        line["comparison"] = comp
        del Kc, Vc

    # ---- end to end through the C ABI with host buffers: every denoising
    # step copies its Q, K, V in from pinned host memory and its Y out.  The
    # copies in (one stream) and out (another) run on PCIe's two directions
    # while the kernels run on a third, with two device buffer sets so step
    # s + 1's inputs land while step s computes.  A step's Q, K, V sit back to
    # back in one pinned host buffer and go in as one copy.
    if not args.no_e2e:
        st = sets[0]
        nq, nk = st["Q"].numel(), st["K"].numel()
        # the pinned buffers on the GPU's own NUMA node: allocated and first
        # written by this thread while it runs on that node's CPUs (copies
        # from a far node's memory cross the socket link on every step)
        numa_node, local_cpus = gpu_host_locality(dev)
        old_cpus = os.sched_getaffinity(0)
        if local_cpus:
            os.sched_setaffinity(0, local_cpus)
        try:
            hQKV = torch.cat([st[k].reshape(-1).cpu() for k in ("Q", "K", "V")]).pin_memory()
            hY = torch.empty(st["Y"].shape, dtype=torch.bfloat16).pin_memory()
            hY.zero_()
        finally:
            os.sched_setaffinity(0, old_cpus)
        hQ = hQKV[:nq].view(st["Q"].shape)
        hK = hQKV[nq:nq + nk].view(st["K"].shape)
        hV = hQKV[nq + nk:].view(st["V"].shape)
        dbuf = []
        for _ in range(2):
            flat = torch.empty_like(hQKV, device=dev)
            dbuf.append({"QKV": flat, "Q": flat[:nq].view(st["Q"].shape),
                         "K": flat[nq:nq + nk].view(st["K"].shape),
                         "V": flat[nq + nk:].view(st["V"].shape),
                         "Y": torch.empty_like(st["Y"])})
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of buffer b landed
        ev_comp = [torch.cuda.Event() for _ in range(2)]   # step on buffer b done
        ev_out = [torch.cuda.Event() for _ in range(2)]    # Y of buffer b copied out
        for b in range(2):
            for e in (ev_comp[b], ev_out[b]):
                e.record(stream)
        n_e2e, warm_e2e = e2e_counts(args.steps, args.warmup)

        def e2e_cycle():
            for s in range(DENOISE):
                b = s % 2
                d = dbuf[b]
                with torch.cuda.stream(s_in):
                    s_in.wait_event(ev_comp[b])            # buffer b's last step has read it
                    d["QKV"].copy_(hQKV, non_blocking=True)
                    ev_in[b].record(s_in)
                stream.wait_event(ev_in[b])
                stream.wait_event(ev_out[b])               # buffer b's last Y is out
                call = bha.bha_hybrid_step_commit if s == DENOISE - 1 else bha.bha_hybrid_step
                call(d["Q"], d["K"], d["V"], st["S"], d["Y"], z=st["z"], stream=stream)
                ev_comp[b].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_comp[b])
                    hY.copy_(d["Y"], non_blocking=True)
                    ev_out[b].record(s_out)

        for _ in range(warm_e2e):
            e2e_cycle()
        torch.cuda.synchronize()
        barrier()
        t0 = time.perf_counter()
        ev0.record(s_in)
        for _ in range(n_e2e):
            e2e_cycle()
        ev1.record(s_out)
        torch.cuda.synchronize()
        wall = time.perf_counter() - t0
        e2e_ms = max(ev0.elapsed_time(ev1), wall * 1e3)
        e2e_ms = max_over_ranks(e2e_ms, pg, dev)
        h2d = DENOISE * (hQ.numel() + hK.numel() + hV.numel()) * 2
        d2h = DENOISE * hY.numel() * 2
        # the link alone: one copy each way of the same buffers, after the loop
        link = {}
        for name, dst, src, nbytes in (("h2d_gbs", dbuf[0]["QKV"], hQKV, hQKV.numel() * 2),
                                       ("d2h_gbs", hY, dbuf[0]["Y"], hY.numel() * 2)):
            e0l, e1l = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0l.record(stream)
            with torch.cuda.stream(stream):
                for _ in range(5):
                    dst.copy_(src, non_blocking=True)
            e1l.record(stream)
            torch.cuda.synchronize()
            link[name] = 5 * nbytes / (e0l.elapsed_time(e1l) / 1e3) / 1e9
        line["e2e"] = {"value": job_throughput(n_e2e * N_ * B_ * DENOISE, world, e2e_ms),
                       "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                       "d2h_bytes_per_step": d2h, "steps": n_e2e, "warmup": warm_e2e,
                       "host_numa_node": numa_node, "host_buffers_local": bool(local_cpus),
                       "link_alone": link,
                       "note": "block cycles: --steps and --warmup, at least %d and %d"
                               % (E2E_MIN_CYCLES, E2E_MIN_WARMUP)}
        line["gpu_launches_e2e"] = n_e2e * DENOISE

    # every rank has finished its collective steps; rank 0 alone goes on
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return
    # ---- secondary workloads on this GPU, from a clean device: the single
    # step (batch 8), the generation loop against the exact path, the exact
    # path with reuse for stable tokens, and the 20-layer stack's largest
    # batch before out-of-memory
    if not args.no_secondary:
        # drop every device buffer of the benchmark line
        sets = S0 = z0 = ws = st = dbuf = Kp = Vp = Kc = Vc = Yx = wsp = None
        graphs = g_step = g_commit = g_shared = timed_graph = None
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        line["secondary"] = {
            "single_step_batch8": measure_single_step(dev),
            "generation_loop": measure_generation_loop(dev),
            "reuse": measure_reuse(dev),
            "stack_memory": stack_oom(dev),
        }
    if not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline_native()
    print(json.dumps(line), flush=True)


def run_only(args):
    """One kernel on the long-prefix shapes (prompt / cache length --prefix),
    warmup + steps plain launches, for profiler captures."""
    import torch
    import block_hybrid_linear_b200 as bha
    from block_hybrid_linear_b200 import build, inputs
    build.build()
    dev = torch.device("cuda", 0)
    std = 1.0 / math.sqrt(D_)
    P = args.prefix
    nb = (args.batch if args.batch and args.only in ("step", "step_shared", "step_commit", "commit")
          else N_)
    Q = inputs.normal_bf16_torch(1, inputs.TID_Q, (nb, HQ, B_, D_), std, dev)
    K = inputs.normal_bf16_torch(1, inputs.TID_K, (nb, HKV, B_, D_), std, dev)
    V = inputs.normal_bf16_torch(1, inputs.TID_V, (nb, HKV, B_, D_), std, dev)
    Y = torch.empty_like(Q)
    S = torch.randn(nb, HKV, D_, D_, device=dev)
    z = torch.rand(nb, HKV, D_, device=dev)
    if args.only in ("prefill", "prefix", "reuse"):
        Kp = inputs.normal_bf16_torch(1, inputs.TID_KP, (nb, HKV, P, D_), std, dev)
        Vp = inputs.normal_bf16_torch(1, inputs.TID_VP, (nb, HKV, P, D_), std, dev)
    if args.only == "prefill":
        need = bha.bha_state_prefill_workspace_size(nb, HKV, P, D_)
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
        fn = lambda: bha.bha_state_prefill(Kp, Vp, S, z, workspace=ws)
    elif args.only == "prefix":
        need = bha.bha_prefix_softmax_workspace_size(nb, HQ, HKV, B_, D_, P)
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
        fn = lambda: bha.bha_prefix_softmax(Q, Kp, Vp, P, K, V, Y, workspace=ws)
    elif args.only == "reuse":
        # a selecting step (k = 8 of 32 tokens) of the exact path with reuse; the
        # cache comes from one dense step first
        k = 8
        Q1 = inputs.normal_bf16_torch(2, inputs.TID_Q, (nb, HQ, B_, D_), std, dev)
        O = torch.empty(nb, HQ, B_, D_, device=dev)
        L = torch.empty(nb, HQ, B_, device=dev)
        need = bha.bha_prefix_softmax_reuse_workspace_size(nb, HQ, HKV, B_, D_, P, k)
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
        bha.bha_prefix_softmax_reuse(Q, None, Kp, Vp, P, K, V, Y, O, L, k, workspace=ws)
        fn = lambda: bha.bha_prefix_softmax_reuse(Q1, Q, Kp, Vp, P, K, V, Y, O, L, k,
                                                  workspace=ws)
    elif args.only == "paged":
        # the ragged workload's paged exact path (batch 64, lengths in [1, 16384])
        _, max_pages, Kpool, Vpool, tab, plen, Q, K, V = _ragged_paged_batch(nb, dev)
        Y = torch.empty_like(Q)
        need = bha.bha_prefix_softmax_paged_workspace_size(nb, HQ, HKV, B_, D_, max_pages,
                                                           RAGGED_PAGE)
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
        fn = lambda: bha.bha_prefix_softmax_paged(Q, Kpool, Vpool, tab, plen, K, V, Y,
                                                  workspace=ws)
    elif args.only == "commit":
        fn = lambda: bha.bha_state_commit(K, V, S, z)
    elif args.only == "step_shared":
        fn = lambda: bha.bha_hybrid_step(Q, K, V, S, Y, z=z, flags=bha.BHA_FLAG_SHARED_DENOM)
    elif args.only == "step_commit":
        fn = lambda: bha.bha_hybrid_step_commit(Q, K, V, S, Y, z=z)
    else:
        fn = lambda: bha.bha_hybrid_step(Q, K, V, S, Y, z=z)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    assert bha.bha_device_error(True) == 0
    print(json.dumps({"only": args.only, "prefix": P, "launches": args.steps,
                      "avg_ms": e0.elapsed_time(e1) / max(1, args.steps)}), flush=True)


def _graph(fn, stream):
    import torch
    with torch.cuda.stream(stream):
        fn()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def _time_graph(g, stream, reps):
    import torch
    torch.cuda.set_stream(stream)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def measure_single_step(dev):
    """Batch 8, 16q/4kv, B=32, prefix 4096 in the state: one denoising step
    (launch-latency bound at this size), beside the exact path and a plain
    copy of the same bytes."""
    import torch
    import block_hybrid_linear_b200 as bha
    from block_hybrid_linear_b200 import inputs
    n, P = 8, 4096
    std = 1.0 / math.sqrt(D_)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    Kp = inputs.normal_bf16_torch(2000, inputs.TID_KP, (n, HKV, P + B_, D_), std, dev)
    Vp = inputs.normal_bf16_torch(2000, inputs.TID_VP, (n, HKV, P + B_, D_), std, dev)
    S0 = torch.empty(n, HKV, D_, D_, device=dev)
    z0 = torch.empty(n, HKV, D_, device=dev)
    need = bha.bha_state_prefill_workspace_size(n, HKV, P, D_)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    bha.bha_state_prefill(Kp[:, :, :P].contiguous(), Vp[:, :, :P].contiguous(), S0, z0,
                          workspace=ws)
    R = max(4, math.ceil(4 * l2 / (n * HKV * UNIT_BYTES_STEP)))
    sets = [dict(Q=inputs.normal_bf16_torch(r, inputs.TID_Q, (n, HQ, B_, D_), std, dev),
                 K=inputs.normal_bf16_torch(r, inputs.TID_K, (n, HKV, B_, D_), std, dev),
                 V=inputs.normal_bf16_torch(r, inputs.TID_V, (n, HKV, B_, D_), std, dev),
                 S=S0.clone(), z=z0.clone(),
                 Y=torch.empty(n, HQ, B_, D_, dtype=torch.bfloat16, device=dev))
            for r in range(R)]
    stream = torch.cuda.Stream(device=dev)

    def steps(flags=0, commit=False):
        call = bha.bha_hybrid_step_commit if commit else bha.bha_hybrid_step
        for st in sets:
            call(st["Q"], st["K"], st["V"], st["S"], st["Y"], z=st["z"], flags=flags,
                 stream=stream)
    g = _graph(steps, stream)
    step_us = _time_graph(g, stream, 50) * 1e3 / R
    g = _graph(lambda: steps(flags=bha.BHA_FLAG_SHARED_DENOM), stream)
    shared_us = _time_graph(g, stream, 50) * 1e3 / R
    g = _graph(lambda: steps(commit=True), stream)
    commit_us = _time_graph(g, stream, 50) * 1e3 / R
    del g
    needp = bha.bha_prefix_softmax_workspace_size(n, HQ, HKV, B_, D_, P)
    wsp = torch.empty(max(needp, 16), dtype=torch.uint8, device=dev)
    st = sets[0]

    def exact():
        bha.bha_prefix_softmax(st["Q"], Kp, Vp, P, st["K"], st["V"], st["Y"], workspace=wsp,
                               stream=stream)
    gx = _graph(exact, stream)
    exact_us = _time_graph(gx, stream, 50) * 1e3
    del gx
    bytes_step = n * HKV * UNIT_BYTES_STEP
    peak, _ = measured_peaks()
    torch.cuda.synchronize()
    assert bha.bha_device_error(True) == 0
    return {
        "workload": "single-step: batch 8, 16q/4kv, d=128, B=32, prefix 4096 in the state",
        "hybrid_step": {"launch_us": step_us, "tokens_per_s": n * B_ / (step_us / 1e6),
                        "achieved_gbs": bytes_step / (step_us / 1e6) / 1e9,
                        "frac_of_peak": bytes_step / (step_us / 1e6) / 1e9 / peak,
                        "algorithmic_bytes": bytes_step},
        "hybrid_step_shared_denom_us": shared_us,
        "hybrid_step_commit_us": commit_us,
        "prefix_softmax": {"launch_us": exact_us, "tokens_per_s": n * B_ / (exact_us / 1e6)},
        "same_bytes_copy": same_bytes_copy(bytes_step, R, stream, dev, peak),
        "note": "4.7 MB per step: bound by per-CTA latency, not by HBM"}


def run_single_step(args):
    import torch
    from block_hybrid_linear_b200 import build
    build.build()
    out = measure_single_step(torch.device("cuda", 0))
    out["metric"], out["unit"] = METRIC, "tokens/s"
    print(json.dumps(out), flush=True)


def run_feature_maps(args):
    """The long-prefix shapes (batch 64, 16q/4kv, d=128, B=32) under each
    feature map (ReLU, elu + 1, ReLU after a per-KV-head projection W_g):
    per-launch times of the step, the last step fused with the commit, the
    commit, and a 32768-token prefill, as kernel-only CUDA graphs over
    rotating input sets 4x the size of L2."""
    import torch
    import block_hybrid_linear_b200 as bha
    from block_hybrid_linear_b200 import build, inputs
    build.build()
    dev = torch.device("cuda", 0)
    n, P = N_, 32768
    std = 1.0 / math.sqrt(D_)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    R = max(4, math.ceil(4 * l2 / (n * HKV * UNIT_BYTES_STEP)))
    W = inputs.normal_bf16_torch(4000, 90, (HKV, D_, D_), 1.0 / math.sqrt(D_), dev)  # N(0, 1/d)
    sets = [dict(Q=inputs.normal_bf16_torch(r, inputs.TID_Q, (n, HQ, B_, D_), std, dev),
                 K=inputs.normal_bf16_torch(r, inputs.TID_K, (n, HKV, B_, D_), std, dev),
                 V=inputs.normal_bf16_torch(r, inputs.TID_V, (n, HKV, B_, D_), std, dev),
                 S=torch.randn(n, HKV, D_, D_, device=dev), z=torch.rand(n, HKV, D_, device=dev),
                 Y=torch.empty(n, HQ, B_, D_, dtype=torch.bfloat16, device=dev))
            for r in range(R)]
    Kp = inputs.normal_bf16_torch(4000, inputs.TID_KP, (n, HKV, P, D_), std, dev)
    Vp = inputs.normal_bf16_torch(4000, inputs.TID_VP, (n, HKV, P, D_), std, dev)
    need = bha.bha_state_prefill_workspace_size(n, HKV, P, D_)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    Sp = torch.empty(n, HKV, D_, D_, device=dev)
    zp = torch.empty(n, HKV, D_, device=dev)
    stream = torch.cuda.Stream(device=dev)
    peak, _ = measured_peaks()
    units = n * HKV
    prefill_bytes = units * (2 * P * D_ * 2 + D_ * D_ * 4 + D_ * 4)
    out = {}
    for name, f in (("relu", bha.BHA_FMAP_RELU), ("elu1", bha.BHA_FMAP_ELU1),
                    ("relu_proj", bha.BHA_FMAP_RELU_PROJ)):
        Wf = W if f == bha.BHA_FMAP_RELU_PROJ else None
        wbytes = 0 if Wf is None else HKV * D_ * D_ * 2

        def per_launch(call, reps=50):
            g = _graph(lambda: [call(st) for st in sets], stream)
            return _time_graph(g, stream, reps) * 1e3 / R

        res = {}
        for op, call, ubytes in (
                ("step", lambda st: bha.bha_hybrid_step_fm(
                    st["Q"], st["K"], st["V"], st["S"], st["Y"], z=st["z"], fmap=f, W=Wf,
                    stream=stream), UNIT_BYTES_STEP),
                ("step_commit", lambda st: bha.bha_hybrid_step_commit_fm(
                    st["Q"], st["K"], st["V"], st["S"], st["Y"], z=st["z"], fmap=f, W=Wf,
                    stream=stream), UNIT_BYTES_FUSED),
                ("commit", lambda st: bha.bha_state_commit_fm(
                    st["K"], st["V"], st["S"], st["z"], fmap=f, W=Wf, stream=stream),
                 UNIT_BYTES_COMMIT)):
            us = per_launch(call)
            nbytes = units * ubytes + wbytes
            res[op] = {"launch_us": round(us, 3), "algorithmic_bytes": nbytes,
                       "achieved_gbs": round(nbytes / (us / 1e6) / 1e9, 1),
                       "frac_of_peak": round(nbytes / (us / 1e6) / 1e9 / peak, 4)}
        gp = _graph(lambda: bha.bha_state_prefill_fm(Kp, Vp, Sp, zp, fmap=f, W=Wf, workspace=ws,
                                                     stream=stream), stream)
        us = _time_graph(gp, stream, 5) * 1e3
        nbytes = prefill_bytes + wbytes
        res["prefill_32768"] = {"launch_us": round(us, 1), "algorithmic_bytes": nbytes,
                                "achieved_gbs": round(nbytes / (us / 1e6) / 1e9, 1),
                                "frac_of_peak": round(nbytes / (us / 1e6) / 1e9 / peak, 4)}
        out[name] = res
    torch.cuda.synchronize()
    assert bha.bha_device_error(True) == 0
    print(json.dumps({
        "workload": "feature-maps: batch 64, 16q/4kv, d=128, B=32; prefill of 32768 tokens",
        "rotating_sets": R, "peak_gbs": peak, "maps": out}), flush=True)


RAGGED_PAGE, RAGGED_LMAX = 128, 16384


def _ragged_paged_batch(n, dev):
    """The ragged workload's batch: prefix lengths drawn uniformly from
    [1, 16384] (seeded), each request's cache in its own pages of 128 tokens
    of one pool in a seeded random order, and the active block's Q, K, V."""
    import numpy as np
    import torch
    from block_hybrid_linear_b200 import inputs
    ps = RAGGED_PAGE
    std = 1.0 / math.sqrt(D_)
    lengths = np.random.default_rng(6000).integers(1, RAGGED_LMAX + 1, size=8192)
    P_lens = lengths[:n]
    pages = (P_lens + ps - 1) // ps
    num_pages, max_pages = int(pages.sum()), int(pages.max())
    order = np.random.default_rng(6001).permutation(num_pages)
    table = np.full((n, max_pages), -1, dtype=np.int32)
    k = 0
    for i in range(n):
        table[i, :pages[i]] = order[k:k + pages[i]]
        k += pages[i]
    Kpool = inputs.normal_bf16_torch(6000, inputs.TID_KC, (num_pages, HKV, ps, D_), std, dev)
    Vpool = inputs.normal_bf16_torch(6000, inputs.TID_VC, (num_pages, HKV, ps, D_), std, dev)
    tab = torch.from_numpy(table).to(dev)
    plen = torch.from_numpy(P_lens.astype(np.int32)).to(dev)
    Q = inputs.normal_bf16_torch(6000, inputs.TID_Q, (n, HQ, B_, D_), std, dev)
    K = inputs.normal_bf16_torch(6000, inputs.TID_K, (n, HKV, B_, D_), std, dev)
    V = inputs.normal_bf16_torch(6000, inputs.TID_V, (n, HKV, B_, D_), std, dev)
    return P_lens, max_pages, Kpool, Vpool, tab, plen, Q, K, V


def run_ragged(args):
    """Batch 64, 16q/4kv, d=128, B=32 with per-request prefix lengths drawn
    uniformly from [1, 16384] (mean about 8192, seeded): the exact path over a
    paged KV cache (pages of 128 tokens) against the same path padded to the
    longest cache, the hybrid step, the ragged prefill of the same prompts, and
    the 20-layer stack (6 hybrid + 14 exact layers) memory per request and
    largest batch before out-of-memory with paged and with padded caches."""
    import numpy as np
    import torch
    import block_hybrid_linear_b200 as bha
    from block_hybrid_linear_b200 import build, inputs
    build.build()
    dev = torch.device("cuda", 0)
    n, ps, Lmax, layers, hyb = N_, RAGGED_PAGE, RAGGED_LMAX, 20, 6
    std = 1.0 / math.sqrt(D_)
    P_lens, max_pages, Kpool, Vpool, tab, plen, Q, K, V = _ragged_paged_batch(n, dev)
    # the stack's memory per request over the first 8192 draws of the same lengths
    lengths = np.random.default_rng(6000).integers(1, Lmax + 1, size=8192)
    Y = torch.empty_like(Q)
    S = torch.randn(n, HKV, D_, D_, device=dev)
    stream = torch.cuda.Stream(device=dev)
    peak, _ = measured_peaks()
    units = n * HKV
    # exact path, paged, each request over its own cache
    need = bha.bha_prefix_softmax_paged_workspace_size(n, HQ, HKV, B_, D_, max_pages, ps)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    g = _graph(lambda: bha.bha_prefix_softmax_paged(Q, Kpool, Vpool, tab, plen, K, V, Y,
                                                    workspace=ws, stream=stream), stream)
    paged_ms = _time_graph(g, stream, 20)
    paged_bytes = int(HKV * (P_lens.sum() + n * B_) * D_ * 4 + units * 65536)
    del g
    # the same path over caches padded to the longest one
    Pmax = int(P_lens.max())
    Kc = inputs.normal_bf16_torch(6002, inputs.TID_KC, (n, HKV, Pmax, D_), std, dev)
    Vc = inputs.normal_bf16_torch(6002, inputs.TID_VC, (n, HKV, Pmax, D_), std, dev)
    needc = bha.bha_prefix_softmax_workspace_size(n, HQ, HKV, B_, D_, Pmax)
    wsc = torch.empty(max(needc, 16), dtype=torch.uint8, device=dev)
    g = _graph(lambda: bha.bha_prefix_softmax(Q, Kc, Vc, Pmax, K, V, Y, workspace=wsc,
                                              stream=stream), stream)
    padded_ms = _time_graph(g, stream, 20)
    del g
    g = _graph(lambda: bha.bha_hybrid_step(Q, K, V, S, Y, stream=stream), stream)
    step_us = _time_graph(g, stream, 200) * 1e3
    del g
    # ragged prefill of the same prompt lengths from the padded buffers
    needp = bha.bha_state_prefill_workspace_size(n, HKV, Pmax, D_)
    wsp = torch.empty(max(needp, 16), dtype=torch.uint8, device=dev)
    z = torch.empty(n, HKV, D_, device=dev)
    g = _graph(lambda: bha.bha_state_prefill_ragged(Kc, Vc, plen, S, z, workspace=wsp,
                                                    stream=stream), stream)
    prefill_ms = _time_graph(g, stream, 10)
    prefill_bytes = int(HKV * P_lens.sum() * D_ * 4 + units * (D_ * D_ + D_) * 4)
    del g, Kc, Vc, Kpool, Vpool, wsc, ws, wsp
    torch.cuda.synchronize()
    assert bha.bha_device_error(True) == 0
    torch.cuda.empty_cache()
    # memory of the 20-layer stack per request, and the largest batch that fits
    kv_tok = HKV * D_ * 2 * 2                     # K and V bytes per cached token, one layer
    st_req = HKV * (D_ * D_ + D_) * 4
    pg_all = ((lengths + ps - 1) // ps) * ps
    hybrid_paged = hyb * st_req + (layers - hyb) * kv_tok * pg_all
    exact_paged = layers * kv_tok * pg_all
    exact_padded = np.full_like(lengths, layers * kv_tok * Lmax)

    def fits(nbytes):
        try:
            buf = torch.empty(int(nbytes), dtype=torch.uint8, device=dev)
            del buf
            return True
        except torch.OutOfMemoryError:
            return False
        finally:
            torch.cuda.empty_cache()

    def max_batch(per_req):
        cum = np.cumsum(per_req.astype(np.float64))
        lo, hi = 0, len(cum)
        while hi - lo > 1:
            mid = (lo + hi) // 2
            lo, hi = (mid, hi) if fits(cum[mid - 1]) else (lo, mid)
        return lo
    print(json.dumps({
        "workload": "ragged: batch 64, 16q/4kv, d=128, B=32, prefix lengths uniform in "
                    "[1, 16384] (seeded), paged KV cache with 128-token pages",
        "metric": METRIC, "unit": "tokens/s",
        "prefix_tokens": {"sum": int(P_lens.sum()), "max": Pmax, "mean": float(P_lens.mean())},
        "exact_paged": {"ms": paged_ms, "tokens_per_s": n * B_ / (paged_ms / 1e3),
                        "algorithmic_bytes": paged_bytes,
                        "achieved_gbs": paged_bytes / (paged_ms / 1e3) / 1e9,
                        "frac_of_peak": paged_bytes / (paged_ms / 1e3) / 1e9 / peak},
        "exact_padded_to_longest": {"ms": padded_ms, "tokens_per_s": n * B_ / (padded_ms / 1e3)},
        "hybrid_step": {"us": step_us, "tokens_per_s": n * B_ / (step_us / 1e6)},
        "ragged_prefill": {"ms": prefill_ms, "algorithmic_bytes": prefill_bytes,
                           "achieved_gbs": prefill_bytes / (prefill_ms / 1e3) / 1e9,
                           "frac_of_peak": prefill_bytes / (prefill_ms / 1e3) / 1e9 / peak},
        "stack_bytes_per_request_mean": {"hybrid_paged": float(hybrid_paged.mean()),
                                         "all_exact_paged": float(exact_paged.mean()),
                                         "all_exact_padded_16384": float(exact_padded.mean())},
        "stack_max_batch_before_oom": {"hybrid_paged": max_batch(hybrid_paged),
                                       "all_exact_paged": max_batch(exact_paged),
                                       "all_exact_padded_16384": max_batch(exact_padded)}}),
          flush=True)


def measure_generation_loop(dev):
    """Batch 32, prompt 1024 -> state, 32 blocks x 8 denoising steps (the
    last step of each block fused with its commit), against exact attention
    over the growing KV cache (appending each finished block).  Whole loops
    replayed as CUDA graphs."""
    import torch
    import block_hybrid_linear_b200 as bha
    from block_hybrid_linear_b200 import inputs
    n, T, nblk, nst = 32, 1024, 32, DENOISE
    std = 1.0 / math.sqrt(D_)
    cap = T + nblk * B_
    Kc = inputs.normal_bf16_torch(3000, inputs.TID_KP, (n, HKV, cap, D_), std, dev)
    Vc = inputs.normal_bf16_torch(3000, inputs.TID_VP, (n, HKV, cap, D_), std, dev)
    Kp, Vp = Kc[:, :, :T].contiguous(), Vc[:, :, :T].contiguous()
    Qs = inputs.normal_bf16_torch(3000, inputs.TID_Q, (nblk, nst, n, HQ, B_, D_), std, dev)
    Ks = inputs.normal_bf16_torch(3000, inputs.TID_K, (nblk, nst, n, HKV, B_, D_), std, dev)
    Vs = inputs.normal_bf16_torch(3000, inputs.TID_V, (nblk, nst, n, HKV, B_, D_), std, dev)
    S = torch.empty(n, HKV, D_, D_, device=dev)
    z = torch.empty(n, HKV, D_, device=dev)
    Y = torch.empty(n, HQ, B_, D_, dtype=torch.bfloat16, device=dev)
    need = bha.bha_state_prefill_workspace_size(n, HKV, T, D_)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    needp = max(bha.bha_prefix_softmax_workspace_size(n, HQ, HKV, B_, D_, T + blk * B_)
                for blk in range(nblk))
    wsp = torch.empty(max(needp, 16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def hybrid_loop():
        bha.bha_state_prefill(Kp, Vp, S, z, workspace=ws, stream=stream)
        for blk in range(nblk):
            for st in range(nst - 1):
                bha.bha_hybrid_step(Qs[blk, st], Ks[blk, st], Vs[blk, st], S, Y, z=z,
                                    stream=stream)
            bha.bha_hybrid_step_commit(Qs[blk, nst - 1], Ks[blk, nst - 1], Vs[blk, nst - 1], S,
                                       Y, z=z, stream=stream)

    def exact_loop():
        for blk in range(nblk):
            P = T + blk * B_
            for st in range(nst):
                bha.bha_prefix_softmax(Qs[blk, st], Kc, Vc, P, Ks[blk, st], Vs[blk, st], Y,
                                       workspace=wsp, stream=stream)
            with torch.cuda.stream(stream):   # append the finished block to the cache
                Kc[:, :, P:P + B_].copy_(Ks[blk, nst - 1])
                Vc[:, :, P:P + B_].copy_(Vs[blk, nst - 1])

    gh = _graph(hybrid_loop, stream)
    gx = _graph(exact_loop, stream)
    h_ms = _time_graph(gh, stream, 5)
    x_ms = _time_graph(gx, stream, 5)
    del gh, gx
    torch.cuda.synchronize()
    assert bha.bha_device_error(True) == 0
    tokens = n * B_ * nblk * nst
    return {
        "workload": "generation-loop: batch 32, 16q/4kv, d=128, prompt 1024 prefilled, "
                    "32 blocks x 8 denoising steps, B=32",
        "hybrid": {"loop_ms": h_ms, "tokens_per_s": tokens / (h_ms / 1e3),
                   "launches": 2 + nblk * nst},
        "exact_prefix_softmax": {"loop_ms": x_ms, "tokens_per_s": tokens / (x_ms / 1e3)},
        "speedup": x_ms / h_ms}


def measure_reuse(dev, ks=(8, 4, 16)):
    """The exact path with reuse for stable tokens at the long-prefix shape
    (batch 64, 16q/4kv, d=128, B=32, a 32768-token cache): one block of 8
    denoising steps -- the first dense, the other 7 selecting the k tokens
    whose queries changed most -- against 8 steps of the exact path, as CUDA
    graphs.  Queries drift from step to step with a per-token weight (a few
    tokens change much, most little); timing does not depend on the values."""
    import torch
    import block_hybrid_linear_b200 as bha
    from block_hybrid_linear_b200 import inputs
    n, P = N_, P_
    std = 1.0 / math.sqrt(D_)
    Kc = inputs.normal_bf16_torch(4400, inputs.TID_KC, (n, HKV, P, D_), std, dev)
    Vc = inputs.normal_bf16_torch(4400, inputs.TID_VC, (n, HKV, P, D_), std, dev)
    g = torch.Generator(device=dev)
    g.manual_seed(4401)
    q = torch.randn(n, HQ, B_, D_, generator=g, device=dev) * std
    Qs = [q.to(torch.bfloat16)]
    for _ in range(1, DENOISE):
        w = torch.empty(n, 1, B_, 1, device=dev).exponential_(generator=g) ** 2
        q = q + 0.3 * w * torch.randn(q.shape, generator=g, device=dev) * std
        Qs.append(q.to(torch.bfloat16))
    Ks = [inputs.normal_bf16_torch(4402 + t, inputs.TID_K, (n, HKV, B_, D_), std, dev)
          for t in range(DENOISE)]
    Vs = [inputs.normal_bf16_torch(4402 + t, inputs.TID_V, (n, HKV, B_, D_), std, dev)
          for t in range(DENOISE)]
    Y = torch.empty(n, HQ, B_, D_, dtype=torch.bfloat16, device=dev)
    O = torch.empty(n, HQ, B_, D_, device=dev)
    L = torch.empty(n, HQ, B_, device=dev)
    need = max(bha.bha_prefix_softmax_reuse_workspace_size(n, HQ, HKV, B_, D_, P, k)
               for k in ks)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    needx = bha.bha_prefix_softmax_workspace_size(n, HQ, HKV, B_, D_, P)
    wsx = torch.empty(max(needx, 16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    peak, _ = measured_peaks()
    kv_bytes = n * HKV * P * D_ * 2 * 2

    def exact_block():
        for t in range(DENOISE):
            bha.bha_prefix_softmax(Qs[t], Kc, Vc, P, Ks[t], Vs[t], Y, workspace=wsx,
                                   stream=stream)
    gx = _graph(exact_block, stream)
    x_ms = _time_graph(gx, stream, 5)
    del gx
    out = {"workload": "reuse: batch 64, 16q/4kv, d=128, B=32, cache 32768; one block of 8 "
                       "denoising steps (the first dense)",
           "kv_cache_bytes_per_step": kv_bytes,
           "exact_block_ms": x_ms, "exact_step_ms": x_ms / DENOISE}
    for k in ks:
        def reuse_block():
            for t in range(DENOISE):
                bha.bha_prefix_softmax_reuse(Qs[t], None if t == 0 else Qs[t - 1], Kc, Vc, P,
                                             Ks[t], Vs[t], Y, O, L, k, workspace=ws,
                                             stream=stream)

        def reuse_steps():   # the selecting steps alone
            for t in range(1, DENOISE):
                bha.bha_prefix_softmax_reuse(Qs[t], Qs[t - 1], Kc, Vc, P, Ks[t], Vs[t], Y, O,
                                             L, k, workspace=ws, stream=stream)
        gr = _graph(reuse_block, stream)
        r_ms = _time_graph(gr, stream, 5)
        del gr
        gs = _graph(reuse_steps, stream)
        s_ms = _time_graph(gs, stream, 5) / (DENOISE - 1)
        del gs
        out["k%d" % k] = {"block_ms": r_ms, "speedup_vs_exact": x_ms / r_ms,
                          "selecting_step_ms": s_ms,
                          "selecting_step_kv_gbs": kv_bytes / (s_ms / 1e3) / 1e9,
                          "selecting_step_frac_of_peak": kv_bytes / (s_ms / 1e3) / 1e9 / peak,
                          "tokens_per_s": n * B_ * DENOISE / (r_ms / 1e3)}
    torch.cuda.synchronize()
    assert bha.bha_device_error(True) == 0
    out["note"] = ("a dense prefix pass over the active tokens still reads the whole cache "
                   "(kv_cache_bytes_per_step) whenever a KV head has one: reuse saves the "
                   "stable tokens' prefix arithmetic, not cache traffic")
    return out


def run_reuse(args):
    import torch
    from block_hybrid_linear_b200 import build
    build.build()
    out = measure_reuse(torch.device("cuda", 0))
    out["metric"], out["unit"] = METRIC, "tokens/s"
    print(json.dumps(out), flush=True)


def run_generation_loop(args):
    import torch
    from block_hybrid_linear_b200 import build
    build.build()
    out = measure_generation_loop(torch.device("cuda", 0))
    out["metric"], out["unit"] = METRIC, "tokens/s"
    print(json.dumps(out), flush=True)


def run_stack(args):
    """20-layer attention stack (6 hybrid + 14 exact layers), prefix 8192:
    one denoising step through the stack per batch size, the all-exact stack
    beside it, device bytes per request, and the largest batch whose state
    fits (searched by allocation, out-of-memory caught)."""
    import torch
    import block_hybrid_linear_b200 as bha
    from block_hybrid_linear_b200 import build, inputs
    build.build()
    dev = torch.device("cuda", 0)
    P, layers, hyb = 8192, 20, 6
    std = 1.0 / math.sqrt(D_)
    stream = torch.cuda.Stream(device=dev)
    rows = []
    batches = [1, 2, 4, 8, 16, 32, 64, 128, 256]
    nmax = batches[-1]
    # one KV cache per exact layer and one state per hybrid layer, allocated
    # once at the largest batch (distinct memory per layer); smaller batches
    # use the leading requests
    caches = [(inputs.normal_bf16_torch(5000 + l, inputs.TID_KC, (nmax, HKV, P, D_), std, dev),
               inputs.normal_bf16_torch(5000 + l, inputs.TID_VC, (nmax, HKV, P, D_), std, dev))
              for l in range(layers)]
    states = [torch.randn(nmax, HKV, D_, D_, device=dev) for _ in range(hyb)]
    Qa = inputs.normal_bf16_torch(5000, inputs.TID_Q, (nmax, HQ, B_, D_), std, dev)
    Ka = inputs.normal_bf16_torch(5000, inputs.TID_K, (nmax, HKV, B_, D_), std, dev)
    Va = inputs.normal_bf16_torch(5000, inputs.TID_V, (nmax, HKV, B_, D_), std, dev)
    Ya = torch.empty_like(Qa)
    for n in batches:
        Q, K, V, Y = Qa[:n], Ka[:n], Va[:n], Ya[:n]
        needp = bha.bha_prefix_softmax_workspace_size(n, HQ, HKV, B_, D_, P)
        wsp = torch.empty(max(needp, 16), dtype=torch.uint8, device=dev)

        def hybrid_stack():
            for l in range(layers):
                if l < hyb:
                    bha.bha_hybrid_step(Q, K, V, states[l][:n], Y, stream=stream)
                else:
                    bha.bha_prefix_softmax(Q, caches[l][0][:n], caches[l][1][:n], P, K, V, Y,
                                           workspace=wsp, stream=stream)

        def exact_stack():
            for l in range(layers):
                bha.bha_prefix_softmax(Q, caches[l][0][:n], caches[l][1][:n], P, K, V, Y,
                                       workspace=wsp, stream=stream)
        gh, gx = _graph(hybrid_stack, stream), _graph(exact_stack, stream)
        th = _time_graph(gh, stream, 10)
        tx = _time_graph(gx, stream, 10)
        rows.append({"batch": n, "hybrid_ms": th, "hybrid_tokens_per_s": n * B_ / (th / 1e3),
                     "exact_ms": tx, "exact_tokens_per_s": n * B_ / (tx / 1e3),
                     "speedup": tx / th})
        del gh, gx, wsp
    del caches, states, Qa, Ka, Va, Ya
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    out = {"workload": "stack: 20 attention layers (6 hybrid + 14 exact), 16q/4kv, d=128, "
                       "B=32, prefix 8192; one denoising step through the stack",
           "metric": METRIC, "unit": "tokens/s", "sweep": rows}
    out.update(stack_oom(dev))
    print(json.dumps(out), flush=True)


def stack_oom(dev):
    """The 20-layer stack (6 hybrid + 14 exact layers) at prefix 8192 with
    contiguous caches: device bytes per request and the largest batch whose
    per-request state fits in the free device memory (doubling, then
    bisection, by allocation with out-of-memory caught)."""
    import torch
    P, layers, hyb = 8192, 20, 6
    kv_req = HKV * P * D_ * 2 * 2             # one exact layer, per request
    st_req = HKV * (D_ * D_ + D_) * 4         # one hybrid layer, per request
    hybrid_req = hyb * st_req + (layers - hyb) * kv_req
    exact_req = layers * kv_req
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    def fits(per_req, n):
        try:
            buf = torch.empty(int(per_req) * n, dtype=torch.uint8, device=dev)
            del buf
            return True
        except torch.OutOfMemoryError:
            return False
        finally:
            torch.cuda.empty_cache()

    def max_batch(per_req):
        lo, hi = 0, 1
        while hi <= 4096 and fits(per_req, hi):   # doubling until allocation fails
            lo, hi = hi, hi * 2
        while hi - lo > 1:                        # then bisect
            mid = (lo + hi) // 2
            lo, hi = (mid, hi) if fits(per_req, mid) else (lo, mid)
        return lo
    free, total = torch.cuda.mem_get_info(dev)
    return {"layout": "contiguous KV caches of 8192 tokens per exact layer, an fp32 S and z "
                      "per hybrid layer",
            "bytes_per_request": {"hybrid_layer_state": st_req, "exact_layer_kv": kv_req,
                                  "hybrid_stack": hybrid_req, "all_exact_stack": exact_req},
            "max_batch_before_oom": {"hybrid_stack": max_batch(hybrid_req),
                                     "all_exact_stack": max_batch(exact_req),
                                     "device_free_bytes": free, "device_total_bytes": total}}


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.only:
        run_only(args)
        return
    if args.workload != "long-prefix":
        if rank == 0:
            {"single-step": run_single_step, "generation-loop": run_generation_loop,
             "stack": run_stack, "feature-maps": run_feature_maps,
             "ragged": run_ragged, "reuse": run_reuse}[args.workload](args)
        return
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    run_native(args, rank, world, local)


if __name__ == "__main__":
    main()
