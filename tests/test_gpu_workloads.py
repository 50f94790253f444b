"""GPU parity on the full workloads, through the C ABI, against the fp64 oracle.

* worked example (L=10, B=4, d=16, fp32): the decoding loop end to end;
* single step (batch 8, 16q/4kv, d=128, B=32, prefix 4096): prefill and step,
  all units;
* generation loop (batch 32, prompt 1024, B=32): the first blocks of the loop,
  prefill -> steps -> commit chained on each side, all units;
* long prefix (batch 64, prefix 32768): the step and the commit on all 256
  units; the 32k prefill and the exact prefix softmax on sampled units (the
  oracle's cost per unit is ~1 s there), in the launch configuration the
  benchmark times;
* stack (prefix 8192) at its largest swept batch, 256: one exact and one
  hybrid layer on sampled units; and the longest prompt, 131072 tokens.
Plus the timeout self-test of the bounded waits.
"""
import math

import numpy as np
import pytest

import oracle
import block_hybrid_linear_b200 as bha
from block_hybrid_linear_b200 import inputs

from gpu_util import (TOL_BF16_ABS, TOL_BF16_REL, TOL_F32_REL, TOL_STATE_REL, bf16_case, dev_f32,
                      host, log_parity, max_abs, rel_l2)

pytestmark = pytest.mark.gpu

STD = 1.0 / math.sqrt(128)


@pytest.fixture(scope="module", autouse=True)
def _setup():
    import torch
    from block_hybrid_linear_b200 import build
    build.build()
    oracle.set_threads(max(1, oracle.max_threads()))
    assert bha.bha_device_error(True) == 0
    yield
    torch.cuda.synchronize()
    assert bha.bha_device_error(True) == 0


def check_bf16(name, got, ref, **kw):
    e_rel, e_abs = rel_l2(got, ref), max_abs(got, ref)
    log_parity(name, rel_l2=e_rel, max_abs=e_abs, **kw)
    assert e_rel <= TOL_BF16_REL and e_abs <= TOL_BF16_ABS, (name, e_rel, e_abs)


def check_rel(name, got, ref, tol, **kw):
    e = rel_l2(got, ref)
    log_parity(name, rel_l2=e, **kw)
    assert e <= tol, (name, e)


def test_worked_example_decoding_loop_fp32():
    """Worked example: L=10 in blocks 4,4,2 (partition from the library), fp32
    N(0,1), phi=ReLU; block 1 softmax only, block 2 uses S_1, block 3 S_1+S_2."""
    import torch
    cfg = inputs.WORKLOADS["worked-example"]
    L, B, d = cfg["L"], cfg["B"], cfg["d"]
    bounds = bha.bha_block_partition(L, B)
    assert bounds == oracle.block_partition(L, B) == [0, 4, 8, 10]
    q = inputs.normal_f32_np(cfg["seed"], inputs.TID_Q, (1, 1, L, d))
    k = inputs.normal_f32_np(cfg["seed"], inputs.TID_K, (1, 1, L, d))
    v = inputs.normal_f32_np(cfg["seed"], inputs.TID_V, (1, 1, L, d))
    blocks = list(zip(bounds[:-1], bounds[1:]))
    ref_out, ref_S, ref_z = oracle.generate([[q[:, :, a:b]] for a, b in blocks],
                                            [[k[:, :, a:b]] for a, b in blocks],
                                            [[v[:, :, a:b]] for a, b in blocks])
    S = torch.zeros(1, 1, d, d, device="cuda")
    z = torch.zeros(1, 1, d, device="cuda")
    for bi, (a, b) in enumerate(blocks):
        Qb, Kb, Vb = (dev_f32(x[:, :, a:b]) for x in (q, k, v))
        Y = torch.empty(1, 1, b - a, d, device="cuda")
        bha.bha_hybrid_step(Qb, Kb, Vb, S, Y, z=z)
        torch.cuda.synchronize()
        check_rel("worked_example_block%d" % (bi + 1), host(Y), ref_out[bi][0], TOL_F32_REL)
        bha.bha_state_commit(Kb, Vb, S, z)
    torch.cuda.synchronize()
    check_rel("worked_example_S", host(S), ref_S, TOL_F32_REL)
    check_rel("worked_example_z", host(z), ref_z, TOL_F32_REL)


def test_single_step_config_all_units():
    """Batch 8, 16q/4kv, B=32, prefix 4096 folded into S by the prefill."""
    import torch
    cfg = inputs.WORKLOADS["single-step"]
    n, hq, hkv, b, P, seed = cfg["n"], cfg["hq"], cfg["hkv"], cfg["b"], cfg["P"], cfg["seed"]
    Kp, Kpv = bf16_case((seed, inputs.TID_KP), (n, hkv, P, 128), STD)
    Vp, Vpv = bf16_case((seed, inputs.TID_VP), (n, hkv, P, 128), STD)
    S = torch.empty(n, hkv, 128, 128, device="cuda")
    z = torch.empty(n, hkv, 128, device="cuda")
    need = bha.bha_state_prefill_workspace_size(n, hkv, P, 128)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    bha.bha_state_prefill(Kp, Vp, S, z, workspace=ws)
    torch.cuda.synchronize()
    rS, rz = oracle.state_prefill(Kpv, Vpv)
    check_rel("config2_prefill_S", host(S), rS, TOL_STATE_REL)
    check_rel("config2_prefill_z", host(z), rz, TOL_STATE_REL)
    # the step gets the oracle's state, so no oracle input comes from the GPU
    Q, Qv = bf16_case((seed, inputs.TID_Q), (n, hq, b, 128), STD)
    K, Kv = bf16_case((seed, inputs.TID_K), (n, hkv, b, 128), STD)
    V, Vv = bf16_case((seed, inputs.TID_V), (n, hkv, b, 128), STD)
    Y = torch.empty(n, hq, b, 128, dtype=torch.bfloat16, device="cuda")
    for shared in (False, True):
        bha.bha_hybrid_step(Q, K, V, dev_f32(rS), Y, z=dev_f32(rz),
                            flags=bha.BHA_FLAG_SHARED_DENOM if shared else 0)
        torch.cuda.synchronize()
        check_bf16("config2_step", host(Y), oracle.hybrid_step(Qv, Kv, Vv, rS, rz, shared=shared),
                   shared=shared)


def test_generation_loop_first_blocks():
    """Batch 32, prompt 1024 -> S, then 3 blocks x 2 denoising steps with a
    commit per block, chained on the GPU and in the oracle independently."""
    import torch
    cfg = inputs.WORKLOADS["generation-loop"]
    n, hq, hkv, b, T, seed = cfg["n"], cfg["hq"], cfg["hkv"], cfg["b"], cfg["prompt"], cfg["seed"]
    nblk, nstep = 3, 2
    Kp, Kpv = bf16_case((seed, inputs.TID_KP), (n, hkv, T, 128), STD)
    Vp, Vpv = bf16_case((seed, inputs.TID_VP), (n, hkv, T, 128), STD)
    Qs, Ks, Vs = [], [], []
    for blk in range(nblk):
        Qs.append([bf16_case((seed, inputs.step_tid(inputs.TID_Q, blk, s)), (n, hq, b, 128), STD)
                   for s in range(nstep)])
        Ks.append([bf16_case((seed, inputs.step_tid(inputs.TID_K, blk, s)), (n, hkv, b, 128), STD)
                   for s in range(nstep)])
        Vs.append([bf16_case((seed, inputs.step_tid(inputs.TID_V, blk, s)), (n, hkv, b, 128), STD)
                   for s in range(nstep)])
    ref_out, ref_S, ref_z = oracle.generate(
        [[x[1] for x in r] for r in Qs], [[x[1] for x in r] for r in Ks],
        [[x[1] for x in r] for r in Vs], Kpv, Vpv)
    S = torch.empty(n, hkv, 128, 128, device="cuda")
    z = torch.empty(n, hkv, 128, device="cuda")
    need = bha.bha_state_prefill_workspace_size(n, hkv, T, 128)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    bha.bha_state_prefill(Kp, Vp, S, z, workspace=ws)
    Y = torch.empty(n, hq, b, 128, dtype=torch.bfloat16, device="cuda")
    for blk in range(nblk):
        for s in range(nstep):
            bha.bha_hybrid_step(Qs[blk][s][0], Ks[blk][s][0], Vs[blk][s][0], S, Y, z=z)
            torch.cuda.synchronize()
            check_bf16("config3_step", host(Y), ref_out[blk][s], blk=blk, step=s)
        bha.bha_state_commit(Ks[blk][-1][0], Vs[blk][-1][0], S, z)
    torch.cuda.synchronize()
    check_rel("config3_final_S", host(S), ref_S, TOL_STATE_REL)
    check_rel("config3_final_z", host(z), ref_z, TOL_STATE_REL)


def _timed_loop_case(seed, nblk, nstep, T):
    """Inputs of the benchmark's block cycle at its shape (batch 64, 16q/4kv,
    d = 128, B = 32): a T-token prompt and Q, K, V for every (block, step),
    seeded per row; the oracle's prefix state of the prompt, built piecewise
    (16 requests at a time) to bound host memory."""
    cfg = inputs.WORKLOADS["long-prefix"]
    n, hq, hkv, b = cfg["n"], cfg["hq"], cfg["hkv"], cfg["b"]
    Kp, Kpv = bf16_case((seed, inputs.TID_KP), (n, hkv, T, 128), STD)
    Vp, Vpv = bf16_case((seed, inputs.TID_VP), (n, hkv, T, 128), STD)
    S0 = np.empty((n, hkv, 128, 128))
    z0 = np.empty((n, hkv, 128))
    for r0 in range(0, n, 16):
        S0[r0:r0 + 16], z0[r0:r0 + 16] = oracle.state_prefill(Kpv[r0:r0 + 16], Vpv[r0:r0 + 16])
    del Kpv, Vpv
    steps = {}
    for name, tid, h in (("Q", inputs.TID_Q, hq), ("K", inputs.TID_K, hkv),
                         ("V", inputs.TID_V, hkv)):
        steps[name] = [[bf16_case((seed, inputs.step_tid(tid, blk, s)), (n, h, b, 128), STD)
                        for s in range(nstep)] for blk in range(nblk)]
    return (n, hq, hkv, b), Kp, Vp, S0, z0, steps


def _run_timed_loop(shared, seed):
    """The benchmark's decoding loop on the GPU: a prefill-built state, then
    4 blocks x 8 denoising steps -- 7 x bha_hybrid_step and the last step
    through bha_hybrid_step_commit -- captured in one CUDA graph on one stream
    and replayed once, with no host synchronisation inside the loop (every
    step writes its own output buffer).  Every step's output and the final
    state are compared with the oracle's decoding loop from the oracle's own
    prefill of the same prompt."""
    import torch
    nblk, nstep, T = 4, 8, 4096
    (n, hq, hkv, b), Kp, Vp, S0v, z0v, st = _timed_loop_case(seed, nblk, nstep, T)
    flags = bha.BHA_FLAG_SHARED_DENOM if shared else 0
    ref_out, ref_S, ref_z = oracle.generate(
        [[x[1] for x in r] for r in st["Q"]], [[x[1] for x in r] for r in st["K"]],
        [[x[1] for x in r] for r in st["V"]], shared=shared, S0=S0v, z0=z0v)
    S = torch.empty(n, hkv, 128, 128, device="cuda")
    z = torch.empty(n, hkv, 128, device="cuda")
    need = bha.bha_state_prefill_workspace_size(n, hkv, T, 128)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    Ys = [[torch.empty(n, hq, b, 128, dtype=torch.bfloat16, device="cuda")
           for _ in range(nstep)] for _ in range(nblk)]
    stream = torch.cuda.Stream()

    def loop(S_, z_):
        for blk in range(nblk):
            for s in range(nstep):
                call = bha.bha_hybrid_step_commit if s == nstep - 1 else bha.bha_hybrid_step
                call(st["Q"][blk][s][0], st["K"][blk][s][0], st["V"][blk][s][0], S_,
                     Ys[blk][s], z=z_, flags=flags, stream=stream)

    # warm-up (kernel attributes are set on first use) on a throw-away state
    with torch.cuda.stream(stream):
        loop(torch.zeros_like(S), torch.zeros_like(z))
    stream.synchronize()
    bha.bha_state_prefill(Kp, Vp, S, z, workspace=ws, stream=stream)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        loop(S, z)
    for Yrow in Ys:
        for Y in Yrow:
            Y.fill_(float("nan"))
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize()
    assert bha.bha_device_error(True) == 0
    tag = "timed_loop_shared" if shared else "timed_loop"
    for blk in range(nblk):
        for s in range(nstep):
            check_bf16(tag, host(Ys[blk][s]), ref_out[blk][s], blk=blk, step=s)
    check_rel(tag + "_final_S", host(S), ref_S, TOL_STATE_REL)
    check_rel(tag + "_final_z", host(z), ref_z, TOL_STATE_REL)
    del g


def test_generation_loop_fused_timed_shape():
    """The exact launch sequence the benchmark times (batch 64, 16q/4kv, B=32;
    each block's last step fused with its commit, one CUDA graph, no host sync):
    every output of 4 blocks x 8 steps and the final S, z against the oracle.
    Block 2 reads the state block 1's fused commit left (worked example: block
    2 uses S_1, block 3 uses S_1 + S_2)."""
    _run_timed_loop(False, 4100)


def test_generation_loop_shared_denominator_timed_shape():
    """The same loop with the shared denominator (the last step of each block
    runs as a step kernel then a commit kernel, the fused kernel being
    default-mode only)."""
    _run_timed_loop(True, 4200)


def test_long_prefix_step_and_commit_all_units():
    """Batch 64, 16q/4kv, B=32, a 32k-token prefix state (drawn with a 32k
    prefill's statistics): the step and the commit on all 256 units."""
    import torch
    cfg = inputs.WORKLOADS["long-prefix"]
    n, hq, hkv, b, P, seed = cfg["n"], cfg["hq"], cfg["hkv"], cfg["b"], cfg["P"], cfg["seed"]
    Q, Qv = bf16_case((seed, inputs.TID_Q), (n, hq, b, 128), STD)
    K, Kv = bf16_case((seed, inputs.TID_K), (n, hkv, b, 128), STD)
    V, Vv = bf16_case((seed, inputs.TID_V), (n, hkv, b, 128), STD)
    Sv, zv = inputs.synthetic_state_np(seed, n, hkv, 128, P, STD)
    S, z = dev_f32(Sv), dev_f32(zv)
    Y = torch.empty(n, hq, b, 128, dtype=torch.bfloat16, device="cuda")
    bha.bha_hybrid_step(Q, K, V, S, Y, z=z)
    torch.cuda.synchronize()
    check_bf16("config4_step", host(Y), oracle.hybrid_step(Qv, Kv, Vv, Sv, zv))
    bha.bha_state_commit(K, V, S, z)
    torch.cuda.synchronize()
    rS, rz = oracle.state_commit(Sv, zv, Kv, Vv)
    check_rel("config4_commit_S", host(S), rS, TOL_STATE_REL)
    check_rel("config4_commit_z", host(z), rz, TOL_STATE_REL)


def test_long_prefix_prefill_and_exact_path_sampled():
    """Batch 64 x 4 KV heads x 32768 prompt tokens drawn on the device: the
    prefill (8 chunks per unit) and the exact prefix softmax over the same
    32k cache, checked on units {first, middle, last} against the oracle."""
    import torch
    cfg = inputs.WORKLOADS["long-prefix"]
    n, hq, hkv, b, P, seed = cfg["n"], cfg["hq"], cfg["hkv"], cfg["b"], cfg["P"], cfg["seed"]
    Kp = inputs.normal_bf16_torch(seed, inputs.TID_KP, (n, hkv, P, 128), STD, "cuda")
    Vp = inputs.normal_bf16_torch(seed, inputs.TID_VP, (n, hkv, P, 128), STD, "cuda")
    S = torch.empty(n, hkv, 128, 128, device="cuda")
    z = torch.empty(n, hkv, 128, device="cuda")
    need = bha.bha_state_prefill_workspace_size(n, hkv, P, 128)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    bha.bha_state_prefill(Kp, Vp, S, z, workspace=ws)
    Q = inputs.normal_bf16_torch(seed, inputs.TID_Q, (n, hq, b, 128), STD, "cuda")
    K = inputs.normal_bf16_torch(seed, inputs.TID_K, (n, hkv, b, 128), STD, "cuda")
    V = inputs.normal_bf16_torch(seed, inputs.TID_V, (n, hkv, b, 128), STD, "cuda")
    Y = torch.empty(n, hq, b, 128, dtype=torch.bfloat16, device="cuda")
    needp = bha.bha_prefix_softmax_workspace_size(n, hq, hkv, b, 128, P)
    wsp = torch.empty(needp, dtype=torch.uint8, device="cuda")
    bha.bha_prefix_softmax(Q, Kp, Vp, P, K, V, Y, workspace=wsp)
    torch.cuda.synchronize()
    G = hq // hkv
    for u in (0, (n * hkv) // 2 + 1, n * hkv - 1):
        ni, g = divmod(u, hkv)
        kp = host(Kp[ni:ni + 1, g:g + 1])
        vp = host(Vp[ni:ni + 1, g:g + 1])
        rS, rz = oracle.state_prefill(kp, vp)
        check_rel("config4_prefill_S", host(S[ni:ni + 1, g:g + 1]), rS, TOL_STATE_REL, unit=u)
        check_rel("config4_prefill_z", host(z[ni:ni + 1, g:g + 1]), rz, TOL_STATE_REL, unit=u)
        qh = host(Q[ni:ni + 1, g * G:(g + 1) * G])
        ref = oracle.prefix_softmax(qh, kp, vp, P, host(K[ni:ni + 1, g:g + 1]),
                                    host(V[ni:ni + 1, g:g + 1]))
        check_bf16("config4_prefix", host(Y[ni:ni + 1, g * G:(g + 1) * G]), ref, unit=u)


def test_stack_config_exact_and_hybrid_layers_largest_batch_sampled():
    """The stack workload at its largest swept batch (256 requests, prefix
    8192): one exact layer (the contiguous exact path) and one hybrid layer
    (prefill of the same prefix, then a step), checked on units {first,
    middle, last} against the oracle."""
    import torch
    n, hq, hkv, b, P, seed = 256, 16, 4, 32, 8192, 5000
    Kc = inputs.normal_bf16_torch(seed, inputs.TID_KC, (n, hkv, P, 128), STD, "cuda")
    Vc = inputs.normal_bf16_torch(seed, inputs.TID_VC, (n, hkv, P, 128), STD, "cuda")
    Q = inputs.normal_bf16_torch(seed, inputs.TID_Q, (n, hq, b, 128), STD, "cuda")
    K = inputs.normal_bf16_torch(seed, inputs.TID_K, (n, hkv, b, 128), STD, "cuda")
    V = inputs.normal_bf16_torch(seed, inputs.TID_V, (n, hkv, b, 128), STD, "cuda")
    Yx = torch.empty(n, hq, b, 128, dtype=torch.bfloat16, device="cuda")
    Yh = torch.empty_like(Yx)
    needp = bha.bha_prefix_softmax_workspace_size(n, hq, hkv, b, 128, P)
    wsp = torch.empty(max(needp, 16), dtype=torch.uint8, device="cuda")
    bha.bha_prefix_softmax(Q, Kc, Vc, P, K, V, Yx, workspace=wsp)
    S = torch.empty(n, hkv, 128, 128, device="cuda")
    need = bha.bha_state_prefill_workspace_size(n, hkv, P, 128)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    bha.bha_state_prefill(Kc, Vc, S, None, workspace=ws)
    bha.bha_hybrid_step(Q, K, V, S, Yh)
    torch.cuda.synchronize()
    G = hq // hkv
    for u in (0, (n * hkv) // 2 + 3, n * hkv - 1):
        ni, g = divmod(u, hkv)
        kc, vc = host(Kc[ni:ni + 1, g:g + 1]), host(Vc[ni:ni + 1, g:g + 1])
        qh = host(Q[ni:ni + 1, g * G:(g + 1) * G])
        kh, vh = host(K[ni:ni + 1, g:g + 1]), host(V[ni:ni + 1, g:g + 1])
        check_bf16("config5_exact", host(Yx[ni:ni + 1, g * G:(g + 1) * G]),
                   oracle.prefix_softmax(qh, kc, vc, P, kh, vh), unit=u)
        rS, _ = oracle.state_prefill(kc, vc, with_z=False)
        check_rel("config5_prefill_S", host(S[ni:ni + 1, g:g + 1]), rS, TOL_STATE_REL, unit=u)
        check_bf16("config5_hybrid", host(Yh[ni:ni + 1, g * G:(g + 1) * G]),
                   oracle.hybrid_step(qh, kh, vh, rS), unit=u)


def test_prefill_longest_prompt_sampled():
    """A 131072-token prompt (32 chunks per unit, reduced in order) for one
    request: every KV head against the oracle."""
    import torch
    n, hkv, T = 1, 4, 131072
    Kp = inputs.normal_bf16_torch(7000, inputs.TID_KP, (n, hkv, T, 128), STD, "cuda")
    Vp = inputs.normal_bf16_torch(7000, inputs.TID_VP, (n, hkv, T, 128), STD, "cuda")
    S = torch.empty(n, hkv, 128, 128, device="cuda")
    z = torch.empty(n, hkv, 128, device="cuda")
    need = bha.bha_state_prefill_workspace_size(n, hkv, T, 128)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    bha.bha_state_prefill(Kp, Vp, S, z, workspace=ws)
    torch.cuda.synchronize()
    rS, rz = oracle.state_prefill(host(Kp), host(Vp))
    check_rel("prefill_131072_S", host(S), rS, TOL_STATE_REL, ws=need)
    check_rel("prefill_131072_z", host(z), rz, TOL_STATE_REL)


def test_bounded_wait_timeout_is_reported_and_context_survives():
    import torch
    assert bha.bha_device_error(True) == 0
    bha.bha_selftest_timeout()
    assert bha.bha_device_error(True) == bha.BHA_ERR_TIMEOUT
    assert bha.bha_device_error(True) == 0
    # the context is still usable: a normal step runs and checks out
    Q, Qv = bf16_case((3, 0), (1, 4, 32, 128), STD)
    K, Kv = bf16_case((3, 1), (1, 1, 32, 128), STD)
    V, Vv = bf16_case((3, 2), (1, 1, 32, 128), STD)
    Sv, zv = inputs.synthetic_state_np(3, 1, 1, 128, 1024, STD)
    Y = torch.empty(1, 4, 32, 128, dtype=torch.bfloat16, device="cuda")
    bha.bha_hybrid_step(Q, K, V, dev_f32(Sv), Y)
    torch.cuda.synchronize()
    check_bf16("after_timeout_step", host(Y), oracle.hybrid_step(Qv, Kv, Vv, Sv))
