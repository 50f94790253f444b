"""GPU parity of the exact path with reuse for stable tokens
(bha_prefix_softmax_reuse), through the C ABI, against the fp64 oracle.

The method is the LoSA page's (gist.science explainer of arXiv 2604.12056,
"3. 方法论 LoSA" and "技术细节") with a dense prefix pass over the active
tokens.  Each case runs the denoising steps of one block: the first dense,
the later ones selecting the k tokens whose queries changed most.  Compared
per step: the outputs (bf16 tolerances), the active lists (integers,
bit-exact: both sides score in fp64 with the same sum order), and the reuse
cache (the prefix outputs in the bf16 output tolerance, the log-normalisers
to 1e-4 absolute).  Query changes are heterogeneous, as the page describes
(a few tokens change much, most little): Q_t = Q_{t-1} + noise scaled by a
per-token weight drawn from an exponential distribution.
"""
import math

import numpy as np
import pytest

import oracle
import block_hybrid_linear_b200 as bha
from block_hybrid_linear_b200 import inputs

from gpu_util import (TOL_BF16_ABS, TOL_BF16_REL, bf16_case, dev_bf16, dev_f32, host,
                      log_parity, max_abs, rel_l2)

pytestmark = pytest.mark.gpu

STD = 1.0 / math.sqrt(128)
TOL_LSE_ABS = 1e-4


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


def step_queries(seed, n, hq, b, steps):
    """bf16 queries of consecutive denoising steps with token-dependent change."""
    _, q = inputs.normal_bf16_np(seed, inputs.TID_Q, (n, hq, b, 128), STD)
    rng = np.random.default_rng(seed + 17)
    out = [q]
    for t in range(1, steps):
        w = rng.exponential(1.0, size=(n, 1, b, 1)).astype(np.float32) ** 2
        noise = inputs.normal_f32_np(seed + t, inputs.TID_Q, (n, hq, b, 128), STD)
        nxt = out[-1] + (0.3 * w * noise).astype(np.float32)
        out.append(inputs.bf16_bits_to_f32(inputs.f32_to_bf16_bits(nxt)))
    return [(dev_bf16(inputs.f32_to_bf16_bits(x)), x) for x in out]


def check_out(name, got, ref, **kw):
    e_rel, e_abs = rel_l2(got, ref), max_abs(got, ref)
    log_parity(name, rel_l2=e_rel, max_abs=e_abs, **kw)
    assert e_rel <= TOL_BF16_REL and e_abs <= TOL_BF16_ABS, (name, e_rel, e_abs, kw)


def check_cache(name, O, L, rO, rL, **kw):
    fin = np.isfinite(rL)
    assert np.array_equal(np.isfinite(L), fin), (name, "normaliser -inf pattern", kw)
    e_o = rel_l2(O, rO) if np.any(rO) else float(np.max(np.abs(O)))
    e_l = float(np.max(np.abs(L[fin] - rL[fin]))) if fin.any() else 0.0
    log_parity(name, O_rel_l2=e_o, L_max_abs=e_l, **kw)
    assert e_o <= TOL_BF16_REL and e_l <= TOL_LSE_ABS, (name, e_o, e_l, kw)


def run_block(seed, n, hq, hkv, b, P, k, steps=3, cap_extra=5):
    """One block of `steps` denoising steps on the GPU and in the oracle."""
    import torch
    cap = P + cap_extra
    Kc, Kcv = bf16_case((seed, inputs.TID_KC), (n, hkv, cap, 128), STD)
    Vc, Vcv = bf16_case((seed, inputs.TID_VC), (n, hkv, cap, 128), STD)
    Qs = step_queries(seed, n, hq, b, steps)
    Ks = [bf16_case((seed, inputs.step_tid(inputs.TID_K, 0, t)), (n, hkv, b, 128), STD)
          for t in range(steps)]
    Vs = [bf16_case((seed, inputs.step_tid(inputs.TID_V, 0, t)), (n, hkv, b, 128), STD)
          for t in range(steps)]
    need = bha.bha_prefix_softmax_reuse_workspace_size(n, hq, hkv, b, 128, P, k)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    O = torch.full((n, hq, b, 128), float("nan"), device="cuda")
    L = torch.full((n, hq, b), float("nan"), device="cuda")
    act = torch.full((n, max(k, 1)), -1, dtype=torch.int32, device="cuda")
    Y = torch.empty(n, hq, b, 128, dtype=torch.bfloat16, device="cuda")
    # the oracle's block loop, step by step (its own cache carried along)
    rO = rL = None
    acts = []
    for t in range(steps):
        Y.fill_(float("nan"))
        bha.bha_prefix_softmax_reuse(Qs[t][0], None if t == 0 else Qs[t - 1][0], Kc, Vc, P,
                                     Ks[t][0], Vs[t][0], Y, O, L, k, active=act,
                                     workspace=ws)
        torch.cuda.synchronize()
        rY, rO, rL, ract = oracle.losa_step(Qs[t][1], None if t == 0 else Qs[t - 1][1], Kcv,
                                            Vcv, P, Ks[t][1], Vs[t][1], rO, rL, k)
        acts.append(ract)
        tag = dict(n=n, hq=hq, hkv=hkv, b=b, P=P, k=k, step=t)
        check_out("reuse_y", host(Y), rY, **tag)
        if t > 0 and 0 < k < b:
            got = act.cpu().numpy()[:, :k]
            assert np.array_equal(got, acts[t]), ("active", tag, got, acts[t])
        check_cache("reuse_cache", host(O), host(L), rO, rL, **tag)
    return acts


# (n, hq, hkv, b, P, k)
CASES = [
    (2, 16, 4, 32, 1000, 8),    # the model's heads, several cache tiles, a ragged tail
    (2, 16, 4, 32, 1000, 1),
    (2, 16, 4, 32, 1000, 31),
    (2, 16, 4, 32, 0, 8),       # no cache: the block alone
    (2, 16, 4, 32, 64, 0),      # k = 0: every token stable after the first step
    (1, 8, 2, 17, 300, 5),      # ragged block (BPAD 32)
    (2, 8, 2, 10, 129, 3),      # BPAD 16
    (1, 4, 1, 1, 77, 1),        # one active token
    (1, 16, 4, 64, 500, 20),    # two query tiles per KV head (BPAD 64)
    (1, 8, 1, 33, 200, 7),      # G b = 264 rows: three query tiles, a ragged third
    (40, 16, 4, 32, 150, 8),    # 160 units: whole-unit block pass (no column halves)
]


@pytest.mark.parametrize("n,hq,hkv,b,P,k", CASES)
def test_reuse_block_loop(n, hq, hkv, b, P, k):
    run_block(1000 + n * 7 + b + k, n, hq, hkv, b, P, k)


def test_reuse_all_active_equals_exact_path():
    """k = b: every step is the exact path (bha_prefix_softmax on the GPU and
    the oracle agree with it within the bf16 tolerances)."""
    import torch
    n, hq, hkv, b, P = 2, 16, 4, 32, 700
    Kc, _ = bf16_case((61, inputs.TID_KC), (n, hkv, P, 128), STD)
    Vc, _ = bf16_case((61, inputs.TID_VC), (n, hkv, P, 128), STD)
    Qs = step_queries(61, n, hq, b, 2)
    K, _ = bf16_case((61, inputs.TID_K), (n, hkv, b, 128), STD)
    V, _ = bf16_case((61, inputs.TID_V), (n, hkv, b, 128), STD)
    need = bha.bha_prefix_softmax_reuse_workspace_size(n, hq, hkv, b, 128, P, b)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    O = torch.empty(n, hq, b, 128, device="cuda")
    L = torch.empty(n, hq, b, device="cuda")
    Y = torch.empty(n, hq, b, 128, dtype=torch.bfloat16, device="cuda")
    Yx = torch.empty_like(Y)
    needx = bha.bha_prefix_softmax_workspace_size(n, hq, hkv, b, 128, P)
    wsx = torch.empty(max(needx, 16), dtype=torch.uint8, device="cuda")
    for t in range(2):
        bha.bha_prefix_softmax_reuse(Qs[t][0], None if t == 0 else Qs[t - 1][0], Kc, Vc, P, K,
                                     V, Y, O, L, b, workspace=ws)
        bha.bha_prefix_softmax(Qs[t][0], Kc, Vc, P, K, V, Yx, workspace=wsx)
        torch.cuda.synchronize()
        check_out("reuse_all_active_vs_exact", host(Y), host(Yx), step=t)


def test_reuse_long_prefix_sampled():
    """The long-prefix shape (batch 64, 16q/4kv, B = 32, a 32768-token cache,
    k = 8): three denoising steps in the launch configuration the benchmark
    times; every request's active list against the oracle (bit-exact), and
    the outputs and cache of requests {0, 31, 63} against the oracle's block
    loop over their own caches."""
    import torch
    n, hq, hkv, b, P, k, steps = 64, 16, 4, 32, 32768, 8, 3
    seed = 4300
    Kc = inputs.normal_bf16_torch(seed, inputs.TID_KC, (n, hkv, P, 128), STD, "cuda")
    Vc = inputs.normal_bf16_torch(seed, inputs.TID_VC, (n, hkv, P, 128), STD, "cuda")
    Qs = step_queries(seed, n, hq, b, steps)
    Ks = [inputs.normal_bf16_torch(seed + t, inputs.TID_K, (n, hkv, b, 128), STD, "cuda")
          for t in range(steps)]
    Vs = [inputs.normal_bf16_torch(seed + t, inputs.TID_V, (n, hkv, b, 128), STD, "cuda")
          for t in range(steps)]
    need = bha.bha_prefix_softmax_reuse_workspace_size(n, hq, hkv, b, 128, P, k)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    O = torch.empty(n, hq, b, 128, device="cuda")
    L = torch.empty(n, hq, b, device="cuda")
    act = torch.empty(n, k, dtype=torch.int32, device="cuda")
    Ys = [torch.empty(n, hq, b, 128, dtype=torch.bfloat16, device="cuda") for _ in range(steps)]
    caches = []
    for t in range(steps):
        bha.bha_prefix_softmax_reuse(Qs[t][0], None if t == 0 else Qs[t - 1][0], Kc, Vc, P,
                                     Ks[t], Vs[t], Ys[t], O, L, k, active=act, workspace=ws)
        torch.cuda.synchronize()
        if t > 0:
            ract, _ = oracle.losa_select(Qs[t][1], Qs[t - 1][1], k)
            assert np.array_equal(act.cpu().numpy(), ract), ("active", t)
        caches.append((host(O), host(L)))
    for ni in (0, 31, 63):
        sl = slice(ni, ni + 1)
        outs, _, rO, rL = oracle.losa_block([q[1][sl] for q in Qs], [host(x[sl]) for x in Ks],
                                            [host(x[sl]) for x in Vs], host(Kc[sl]),
                                            host(Vc[sl]), P, k)
        for t in range(steps):
            check_out("reuse_long_prefix_y", host(Ys[t][sl]), outs[t], request=ni, step=t)
        check_cache("reuse_long_prefix_cache", caches[-1][0][sl], caches[-1][1][sl], rO, rL,
                    request=ni, step=steps - 1)


def test_reuse_selection_ties_go_to_the_lower_index():
    """Tokens whose queries changed identically tie exactly (both sides score
    in fp64, in the same order); the lower token index wins."""
    import torch
    n, hq, hkv, b, P, k = 2, 16, 4, 32, 64, 3
    Qs = step_queries(71, n, hq, b, 2)
    q0, q1 = Qs[0][1].copy(), Qs[1][1].copy()
    # tokens 5, 9 and 20 get the same (largest) change; token 2 a smaller one
    delta = 30.0 * inputs.normal_f32_np(72, 0, (n, hq, 1, 128), STD)
    for i in (5, 9, 20):
        q0[:, :, i] = q0[:, :, 0]
        q1[:, :, i] = inputs.bf16_bits_to_f32(inputs.f32_to_bf16_bits(q0[:, :, 0] + delta[:, :, 0]))
    ract, score = oracle.losa_select(q1, q0, k)
    assert score[0, 5] == score[0, 9] == score[0, 20]
    Kc, _ = bf16_case((73, inputs.TID_KC), (n, hkv, P, 128), STD)
    Vc, _ = bf16_case((73, inputs.TID_VC), (n, hkv, P, 128), STD)
    K, _ = bf16_case((73, inputs.TID_K), (n, hkv, b, 128), STD)
    V, _ = bf16_case((73, inputs.TID_V), (n, hkv, b, 128), STD)
    need = bha.bha_prefix_softmax_reuse_workspace_size(n, hq, hkv, b, 128, P, k)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    O = torch.empty(n, hq, b, 128, device="cuda")
    L = torch.empty(n, hq, b, device="cuda")
    Y = torch.empty(n, hq, b, 128, dtype=torch.bfloat16, device="cuda")
    act = torch.empty(n, k, dtype=torch.int32, device="cuda")
    Q0 = dev_bf16(inputs.f32_to_bf16_bits(q0))
    Q1 = dev_bf16(inputs.f32_to_bf16_bits(q1))
    bha.bha_prefix_softmax_reuse(Q0, None, Kc, Vc, P, K, V, Y, O, L, k, workspace=ws)
    bha.bha_prefix_softmax_reuse(Q1, Q0, Kc, Vc, P, K, V, Y, O, L, k, active=act, workspace=ws)
    torch.cuda.synchronize()
    assert np.array_equal(act.cpu().numpy(), ract)
    assert list(ract[0]) == [5, 9, 20]


F32_CASES = [  # (n, hq, hkv, b, d, P, k)
    (1, 1, 1, 4, 16, 6, 2),      # the worked example's head size
    (2, 4, 2, 13, 64, 37, 5),    # GQA, ragged block
    (1, 8, 2, 32, 128, 300, 8),  # the model's head dim, several key chunks
    (2, 4, 1, 5, 16, 0, 2),      # no cache
]


@pytest.mark.parametrize("n,hq,hkv,b,d,P,k", F32_CASES)
def test_reuse_f32_block_loop(n, hq, hkv, b, d, P, k):
    """fp32 reference mode: three denoising steps against the oracle at 1e-4
    relative L2 (outputs and cache), the active lists bit-exact."""
    import torch
    from gpu_util import TOL_F32_REL
    seed = 1500 + d + b + k
    rng = np.random.default_rng(seed)
    Kc = inputs.normal_f32_np(seed, inputs.TID_KC, (n, hkv, P + 3, d), 1.0)
    Vc = inputs.normal_f32_np(seed, inputs.TID_VC, (n, hkv, P + 3, d), 1.0)
    q = inputs.normal_f32_np(seed, inputs.TID_Q, (n, hq, b, d), 1.0)
    Qs = [q]
    for t in range(1, 3):
        w = rng.exponential(1.0, size=(n, 1, b, 1)).astype(np.float32) ** 2
        Qs.append((Qs[-1] + 0.3 * w * inputs.normal_f32_np(seed + t, 0, (n, hq, b, d), 1.0))
                  .astype(np.float32))
    Ks = [inputs.normal_f32_np(seed + 10 + t, inputs.TID_K, (n, hkv, b, d), 1.0) for t in range(3)]
    Vs = [inputs.normal_f32_np(seed + 10 + t, inputs.TID_V, (n, hkv, b, d), 1.0) for t in range(3)]
    O = torch.full((n, hq, b, d), float("nan"), device="cuda")
    L = torch.full((n, hq, b), float("nan"), device="cuda")
    Y = torch.empty(n, hq, b, d, device="cuda")
    act = torch.full((n, max(k, 1)), -1, dtype=torch.int32, device="cuda")
    rO = rL = None
    dKc, dVc = dev_f32(Kc), dev_f32(Vc)
    for t in range(3):
        bha.bha_prefix_softmax_reuse(dev_f32(Qs[t]), None if t == 0 else dev_f32(Qs[t - 1]), dKc,
                                     dVc, P, dev_f32(Ks[t]), dev_f32(Vs[t]), Y, O, L, k,
                                     active=act)
        torch.cuda.synchronize()
        rY, rO, rL, ract = oracle.losa_step(Qs[t], None if t == 0 else Qs[t - 1], Kc, Vc, P,
                                            Ks[t], Vs[t], rO, rL, k)
        e = rel_l2(host(Y), rY)
        log_parity("reuse_f32_y", rel_l2=e, step=t, d=d, b=b, k=k)
        assert e <= TOL_F32_REL, (t, e)
        assert rel_l2(host(O), rO) <= TOL_F32_REL or not np.any(rO)
        fin = np.isfinite(rL)
        assert np.array_equal(np.isfinite(host(L)), fin)
        if fin.any():
            assert float(np.max(np.abs(host(L)[fin] - rL[fin]))) <= 1e-4
        if t > 0 and 0 < k < b:
            assert np.array_equal(act.cpu().numpy()[:, :k], ract)
