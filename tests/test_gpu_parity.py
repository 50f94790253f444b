"""GPU parity: every CUDA kernel, called through the C ABI, against the fp64
CPU oracle on the same seeded inputs.

Small cases span several tiles and ragged tails (b not a multiple of 16,
G*b above 128 rows, prompts and caches not a multiple of the token tile);
the full-size workloads are checked on all units where the oracle is quick
and on sampled units otherwise.  Outputs sit between canaries and are
NaN-filled before each launch.
"""
import math

import numpy as np
import pytest

import oracle
from block_hybrid_linear_b200 import inputs
import block_hybrid_linear_b200 as bha

from gpu_util import (TOL_BF16_ABS, TOL_BF16_REL, TOL_F32_REL, TOL_STATE_REL, Guarded,
                      bf16_case, dev_f32, host, log_parity, max_abs, rel_l2)

pytestmark = pytest.mark.gpu

STD = 1.0 / math.sqrt(128)


@pytest.fixture(scope="module", autouse=True)
def _setup():
    import torch
    from block_hybrid_linear_b200 import build
    build.build()
    oracle.set_threads(max(1, min(16, oracle.max_threads())))
    torch.cuda.synchronize()
    assert bha.bha_device_error(True) == 0
    yield
    assert bha.bha_device_error(True) == 0


def check_bf16(name, got, ref, **kw):
    e_rel, e_abs = rel_l2(got, ref), max_abs(got, ref)
    log_parity(name, rel_l2=e_rel, max_abs=e_abs, **kw)
    assert e_rel <= TOL_BF16_REL and e_abs <= TOL_BF16_ABS, (name, e_rel, e_abs)


def check_rel(name, got, ref, tol, **kw):
    e_rel = rel_l2(got, ref)
    log_parity(name, rel_l2=e_rel, max_abs=max_abs(got, ref), **kw)
    assert e_rel <= tol, (name, e_rel)


# ------------------------------------------------------------ hybrid step

STEP_CASES = [  # (n, hq, hkv, b)
    (2, 16, 4, 32),    # the model's shape: G*b = 128 rows, one M tile
    (3, 4, 4, 32),     # G = 1: 32 rows in a 128-row tile
    (2, 8, 2, 17),     # ragged b, BPAD 32
    (2, 8, 2, 10),     # ragged b, BPAD 16
    (1, 4, 1, 1),      # a single active token
    (2, 8, 1, 33),     # BPAD 64, G*b = 264 rows: three M tiles, ragged tail
    (1, 16, 4, 64),    # b = 64, G*b = 256 rows: two M tiles
    (2, 2, 1, 16),
    # The cases above are grids of at most one CTA per SM, which run as column
    # halves (two CTAs per unit); these exceed the SM count and run whole units.
    (37, 16, 4, 32),   # 148 unit rows: the largest grid still split (296 CTAs)
    (38, 16, 4, 32),   # 152 unit rows: whole units, BPAD 32
    (40, 8, 4, 10),    # whole units, BPAD 16
    (75, 4, 1, 33),    # 75 units x two M tiles = 150 unit rows: whole units, BPAD 64
]


@pytest.mark.parametrize("shared", [False, True], ids=["default", "shared"])
@pytest.mark.parametrize("case", STEP_CASES, ids=lambda c: "n%d_hq%d_hkv%d_b%d" % c)
def test_step_bf16(case, shared):
    import torch
    n, hq, hkv, b = case
    seed = 100 + b
    Q, Qv = bf16_case((seed, 0), (n, hq, b, 128), STD)
    K, Kv = bf16_case((seed, 1), (n, hkv, b, 128), STD)
    V, Vv = bf16_case((seed, 2), (n, hkv, b, 128), STD)
    Sv, zv = inputs.synthetic_state_np(seed, n, hkv, 128, 4096, STD)
    S, z = dev_f32(Sv), dev_f32(zv)
    Y = Guarded((n, hq, b, 128), torch.bfloat16)
    bha.bha_hybrid_step(Q, K, V, S, Y.t, z=z,
                        flags=bha.BHA_FLAG_SHARED_DENOM if shared else 0)
    torch.cuda.synchronize()
    assert Y.intact() and Y.no_nan()
    ref = oracle.hybrid_step(Qv, Kv, Vv, Sv, zv, shared=shared)
    check_bf16("step_bf16", host(Y.t), ref, case=case, shared=shared)


def test_step_bf16_scale_and_zero_state():
    """Explicit scale, and S = 0 (block 1 of the worked example: softmax only)."""
    import torch
    n, hq, hkv, b = 2, 16, 4, 32
    Q, Qv = bf16_case((7, 0), (n, hq, b, 128), 1.0)
    K, Kv = bf16_case((7, 1), (n, hkv, b, 128), 1.0)
    V, Vv = bf16_case((7, 2), (n, hkv, b, 128), 1.0)
    S = torch.zeros(n, hkv, 128, 128, device="cuda")
    Y = torch.empty(n, hq, b, 128, dtype=torch.bfloat16, device="cuda")
    bha.bha_hybrid_step(Q, K, V, S, Y, scale=0.05)
    torch.cuda.synchronize()
    ref = oracle.hybrid_step(Qv, Kv, Vv, np.zeros((n, hkv, 128, 128)), scale=0.05)
    check_bf16("step_bf16_scale", host(Y), ref)


@pytest.mark.parametrize("n", [2, 64], ids=["halves", "whole_units"])
def test_step_bf16_is_deterministic(n):
    """The MMA order is fixed in every path (column halves issue the state
    products and P V in a set order, not in the order their operands land),
    so repeated calls on the same inputs give the same bits; scale 4 makes
    some rows of the shared-denominator tile take the rescaled order."""
    import torch
    hq, hkv, b = 16, 4, 32
    Q, _ = bf16_case((9, 0), (n, hq, b, 128), 1.0)
    K, _ = bf16_case((9, 1), (n, hkv, b, 128), 1.0)
    V, _ = bf16_case((9, 2), (n, hkv, b, 128), 1.0)
    Sv, zv = inputs.synthetic_state_np(9, n, hkv, 128, 4096, STD)
    S, z = dev_f32(Sv), dev_f32(zv)
    for flags, scale in ((0, 0.0), (bha.BHA_FLAG_SHARED_DENOM, 0.0),
                         (bha.BHA_FLAG_SHARED_DENOM, 4.0)):
        outs = []
        for _ in range(3):
            Y = torch.empty(n, hq, b, 128, dtype=torch.bfloat16, device="cuda")
            bha.bha_hybrid_step(Q, K, V, S, Y, z=z, scale=scale, flags=flags)
            outs.append(Y)
        torch.cuda.synchronize()
        assert all(torch.equal(outs[0], o) for o in outs[1:]), (n, flags, scale)


@pytest.mark.parametrize("scale", [1.0, 4.0])
def test_step_bf16_shared_large_scores(scale):
    """Shared denominator with unit-variance inputs: row maxima of the scaled
    scores reach about 30 (scale 1: the factor goes into P) and above 64
    (scale 4: some rows put e^{-max} into phi(q) instead)."""
    import torch
    n, hq, hkv, b = 2, 16, 4, 32
    Q, Qv = bf16_case((8, 0), (n, hq, b, 128), 1.0)
    K, Kv = bf16_case((8, 1), (n, hkv, b, 128), 1.0)
    V, Vv = bf16_case((8, 2), (n, hkv, b, 128), 1.0)
    Sv, zv = inputs.synthetic_state_np(8, n, hkv, 128, 4096, STD)
    Y = Guarded((n, hq, b, 128), torch.bfloat16)
    bha.bha_hybrid_step(Q, K, V, dev_f32(Sv), Y.t, z=dev_f32(zv), scale=scale,
                        flags=bha.BHA_FLAG_SHARED_DENOM)
    torch.cuda.synchronize()
    assert Y.intact() and Y.no_nan()
    ref = oracle.hybrid_step(Qv, Kv, Vv, Sv, zv, scale=scale, shared=True)
    check_bf16("step_bf16_shared_large", host(Y.t), ref, scale=scale)


@pytest.mark.parametrize("d", [16, 64, 128])
@pytest.mark.parametrize("shared", [False, True], ids=["default", "shared"])
def test_step_f32(d, shared):
    import torch
    n, hq, hkv, b = 2, 4, 2, 13
    Qv = inputs.normal_f32_np(31, 0, (n, hq, b, d), 1.0)
    Kv = inputs.normal_f32_np(31, 1, (n, hkv, b, d), 1.0)
    Vv = inputs.normal_f32_np(31, 2, (n, hkv, b, d), 1.0)
    Sv = inputs.normal_f32_np(31, 3, (n, hkv, d, d), 1.0)
    zv = np.abs(inputs.normal_f32_np(31, 4, (n, hkv, d), 10.0))
    Y = Guarded((n, hq, b, d), torch.float32)
    bha.bha_hybrid_step(dev_f32(Qv), dev_f32(Kv), dev_f32(Vv), dev_f32(Sv), Y.t, z=dev_f32(zv),
                        flags=bha.BHA_FLAG_SHARED_DENOM if shared else 0)
    torch.cuda.synchronize()
    assert Y.intact() and Y.no_nan()
    ref = oracle.hybrid_step(Qv, Kv, Vv, Sv, zv, shared=shared)
    check_rel("step_f32", host(Y.t), ref, TOL_F32_REL, d=d, shared=shared)


# ------------------------------------------------------------ commit

@pytest.mark.parametrize("b", [1, 10, 16, 32, 33, 64])
@pytest.mark.parametrize("with_z", [False, True])
def test_commit_bf16(b, with_z):
    import torch
    n, hkv = 3, 4
    K, Kv = bf16_case((200 + b, 1), (n, hkv, b, 128), STD)
    V, Vv = bf16_case((200 + b, 2), (n, hkv, b, 128), STD)
    Sv, zv = inputs.synthetic_state_np(200 + b, n, hkv, 128, 1024, STD)
    S, z = dev_f32(Sv), dev_f32(zv) if with_z else None
    bha.bha_state_commit(K, V, S, z)
    torch.cuda.synchronize()
    rS, rz = oracle.state_commit(Sv, zv, Kv, Vv)
    check_rel("commit_bf16_S", host(S), rS, TOL_STATE_REL, b=b)
    if with_z:
        check_rel("commit_bf16_z", host(z), rz, TOL_STATE_REL, b=b)


@pytest.mark.parametrize("d", [16, 128])
def test_commit_f32(d):
    import torch
    n, hkv, b = 2, 2, 9
    Kv = inputs.normal_f32_np(41, 1, (n, hkv, b, d), 1.0)
    Vv = inputs.normal_f32_np(41, 2, (n, hkv, b, d), 1.0)
    Sv = inputs.normal_f32_np(41, 3, (n, hkv, d, d), 1.0)
    zv = inputs.normal_f32_np(41, 4, (n, hkv, d), 1.0)
    S, z = dev_f32(Sv), dev_f32(zv)
    bha.bha_state_commit(dev_f32(Kv), dev_f32(Vv), S, z)
    torch.cuda.synchronize()
    rS, rz = oracle.state_commit(Sv, zv, Kv, Vv)
    check_rel("commit_f32_S", host(S), rS, TOL_F32_REL, d=d)
    check_rel("commit_f32_z", host(z), rz, TOL_F32_REL, d=d)


# ------------------------------------------------------------ prefill

@pytest.mark.parametrize("T", [0, 1, 63, 64, 65, 1000, 4113])
def test_prefill_bf16(T):
    import torch
    n, hkv = 2, 2
    K, Kv = bf16_case((300 + T, 3), (n, hkv, T, 128), STD)
    V, Vv = bf16_case((300 + T, 4), (n, hkv, T, 128), STD)
    S = Guarded((n, hkv, 128, 128), torch.float32)
    z = Guarded((n, hkv, 128), torch.float32)
    need = bha.bha_state_prefill_workspace_size(n, hkv, T, 128)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda") if need else None
    bha.bha_state_prefill(K, V, S.t, z.t, workspace=ws)
    torch.cuda.synchronize()
    assert S.intact() and S.no_nan() and z.intact() and z.no_nan()
    rS, rz = oracle.state_prefill(Kv, Vv)
    if T == 0:
        assert np.all(host(S.t) == 0) and np.all(host(z.t) == 0)
        return
    check_rel("prefill_bf16_S", host(S.t), rS, TOL_STATE_REL, T=T, ws=need)
    check_rel("prefill_bf16_z", host(z.t), rz, TOL_STATE_REL, T=T)


def test_prefill_is_deterministic():
    import torch
    n, hkv, T = 2, 2, 5000
    K, _ = bf16_case((55, 3), (n, hkv, T, 128), STD)
    V, _ = bf16_case((55, 4), (n, hkv, T, 128), STD)
    need = bha.bha_state_prefill_workspace_size(n, hkv, T, 128)
    assert need > 0   # several chunks reduced in a fixed order
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(2):
        S = torch.empty(n, hkv, 128, 128, device="cuda")
        bha.bha_state_prefill(K, V, S, None, workspace=ws)
        outs.append(S)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])


def test_prefill_f32():
    import torch
    n, hkv, T, d = 2, 2, 300, 16
    Kv = inputs.normal_f32_np(61, 3, (n, hkv, T, d), 1.0)
    Vv = inputs.normal_f32_np(61, 4, (n, hkv, T, d), 1.0)
    S = torch.empty(n, hkv, d, d, device="cuda")
    z = torch.empty(n, hkv, d, device="cuda")
    bha.bha_state_prefill(dev_f32(Kv), dev_f32(Vv), S, z)
    torch.cuda.synchronize()
    rS, rz = oracle.state_prefill(Kv, Vv)
    check_rel("prefill_f32_S", host(S), rS, TOL_F32_REL)
    check_rel("prefill_f32_z", host(z), rz, TOL_F32_REL)


# ------------------------------------------------------------ prefix softmax

PREFIX_CASES = [  # (n, hq, hkv, b, P, cap)
    (2, 16, 4, 32, 0, 16),
    (2, 16, 4, 32, 1, 8),
    (2, 16, 4, 32, 127, 200),
    (2, 16, 4, 32, 128, 128),
    (2, 16, 4, 32, 1000, 1100),
    (1, 8, 2, 17, 4096, 4096),
    (1, 4, 4, 1, 300, 300),
    (1, 8, 1, 33, 777, 800),
]


@pytest.mark.parametrize("case", PREFIX_CASES, ids=lambda c: "n%d_hq%d_hkv%d_b%d_P%d" % c[:5])
def test_prefix_bf16(case):
    import torch
    n, hq, hkv, b, P, cap = case
    seed = 400 + P + b
    Q, Qv = bf16_case((seed, 0), (n, hq, b, 128), STD)
    K, Kv = bf16_case((seed, 1), (n, hkv, b, 128), STD)
    V, Vv = bf16_case((seed, 2), (n, hkv, b, 128), STD)
    Kc, Kcv = bf16_case((seed, 7), (n, hkv, cap, 128), STD)
    Vc, Vcv = bf16_case((seed, 8), (n, hkv, cap, 128), STD)
    Y = Guarded((n, hq, b, 128), torch.bfloat16)
    need = bha.bha_prefix_softmax_workspace_size(n, hq, hkv, b, 128, P)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda") if need else None
    bha.bha_prefix_softmax(Q, Kc, Vc, P, K, V, Y.t, workspace=ws)
    torch.cuda.synchronize()
    assert Y.intact() and Y.no_nan()
    ref = oracle.prefix_softmax(Qv, Kcv, Vcv, P, Kv, Vv)
    check_bf16("prefix_bf16", host(Y.t), ref, case=case, ws=need)


def test_prefix_bf16_large_scores():
    """Unit-variance inputs: row maxima grow across key tiles, exercising the
    accumulator rescale."""
    import torch
    n, hq, hkv, b, P = 1, 4, 1, 32, 2000
    Q, Qv = bf16_case((9, 0), (n, hq, b, 128), 1.0)
    K, Kv = bf16_case((9, 1), (n, hkv, b, 128), 1.0)
    V, Vv = bf16_case((9, 2), (n, hkv, b, 128), 1.0)
    Kc, Kcv = bf16_case((9, 7), (n, hkv, P, 128), 1.0)
    Vc, Vcv = bf16_case((9, 8), (n, hkv, P, 128), 1.0)
    Y = torch.empty(n, hq, b, 128, dtype=torch.bfloat16, device="cuda")
    need = bha.bha_prefix_softmax_workspace_size(n, hq, hkv, b, 128, P)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda") if need else None
    bha.bha_prefix_softmax(Q, Kc, Vc, P, K, V, Y, scale=0.25, workspace=ws)
    torch.cuda.synchronize()
    ref = oracle.prefix_softmax(Qv, Kcv, Vcv, P, Kv, Vv, scale=0.25)
    check_bf16("prefix_bf16_large", host(Y), ref)


def test_prefix_f32():
    import torch
    n, hq, hkv, b, P, cap, d = 2, 4, 2, 5, 300, 310, 16
    Qv = inputs.normal_f32_np(71, 0, (n, hq, b, d), 1.0)
    Kv = inputs.normal_f32_np(71, 1, (n, hkv, b, d), 1.0)
    Vv = inputs.normal_f32_np(71, 2, (n, hkv, b, d), 1.0)
    Kcv = inputs.normal_f32_np(71, 7, (n, hkv, cap, d), 1.0)
    Vcv = inputs.normal_f32_np(71, 8, (n, hkv, cap, d), 1.0)
    Y = torch.empty(n, hq, b, d, device="cuda")
    bha.bha_prefix_softmax(dev_f32(Qv), dev_f32(Kcv), dev_f32(Vcv), P, dev_f32(Kv), dev_f32(Vv), Y)
    torch.cuda.synchronize()
    ref = oracle.prefix_softmax(Qv, Kcv, Vcv, P, Kv, Vv)
    check_rel("prefix_f32", host(Y), ref, TOL_F32_REL)


def test_prefix_p0_equals_step_with_zero_state():
    import torch
    n, hq, hkv, b = 2, 16, 4, 32
    Q, _ = bf16_case((5, 0), (n, hq, b, 128), STD)
    K, _ = bf16_case((5, 1), (n, hkv, b, 128), STD)
    V, _ = bf16_case((5, 2), (n, hkv, b, 128), STD)
    Y1 = torch.empty(n, hq, b, 128, dtype=torch.bfloat16, device="cuda")
    Y2 = torch.empty_like(Y1)
    Kc = torch.zeros(n, hkv, 8, 128, dtype=torch.bfloat16, device="cuda")
    bha.bha_prefix_softmax(Q, Kc, Kc, 0, K, V, Y1)
    bha.bha_hybrid_step(Q, K, V, torch.zeros(n, hkv, 128, 128, device="cuda"), Y2)
    torch.cuda.synchronize()
    assert rel_l2(host(Y1), host(Y2)) < 1e-2


# ------------------------------------------------------------ fused last step + commit

FUSED_CASES = [  # (n, hq, hkv, b): the first five run as one kernel in the default mode
    (2, 16, 4, 32), (3, 4, 4, 32), (2, 8, 2, 17), (2, 8, 2, 10), (1, 4, 1, 1),
    (2, 8, 1, 33),   # G*b = 264 rows: step + commit kernels
    (1, 16, 4, 64),  # 256 rows
    (38, 16, 4, 32), # 152 unit rows: the fused kernel on whole units (the five above
                     # run as column halves)
]


@pytest.mark.parametrize("mode", ["default", "default_noz", "shared"])
@pytest.mark.parametrize("case", FUSED_CASES, ids=lambda c: "n%d_hq%d_hkv%d_b%d" % c)
def test_step_commit_bf16(case, mode):
    """Y from the state before the block, then S += phi(K)^T V, z += sum phi(k)
    -- against the oracle's step followed by its commit."""
    import torch
    n, hq, hkv, b = case
    seed = 600 + b
    shared = mode == "shared"
    Q, Qv = bf16_case((seed, 0), (n, hq, b, 128), STD)
    K, Kv = bf16_case((seed, 1), (n, hkv, b, 128), STD)
    V, Vv = bf16_case((seed, 2), (n, hkv, b, 128), STD)
    Sv, zv = inputs.synthetic_state_np(seed, n, hkv, 128, 4096, STD)
    S = dev_f32(Sv)
    z = None if mode == "default_noz" else dev_f32(zv)
    Y = Guarded((n, hq, b, 128), torch.bfloat16)
    bha.bha_hybrid_step_commit(Q, K, V, S, Y.t, z=z,
                               flags=bha.BHA_FLAG_SHARED_DENOM if shared else 0)
    torch.cuda.synchronize()
    assert Y.intact() and Y.no_nan()
    check_bf16("step_commit_y", host(Y.t), oracle.hybrid_step(Qv, Kv, Vv, Sv, zv, shared=shared),
               case=case, mode=mode)
    rS, rz = oracle.state_commit(Sv, zv, Kv, Vv)
    check_rel("step_commit_S", host(S), rS, TOL_STATE_REL, case=case, mode=mode)
    if z is not None:
        check_rel("step_commit_z", host(z), rz, TOL_STATE_REL, case=case, mode=mode)


def test_step_commit_f32():
    import torch
    n, hq, hkv, b, d = 2, 4, 2, 7, 16
    Qv = inputs.normal_f32_np(81, 0, (n, hq, b, d), 1.0)
    Kv = inputs.normal_f32_np(81, 1, (n, hkv, b, d), 1.0)
    Vv = inputs.normal_f32_np(81, 2, (n, hkv, b, d), 1.0)
    Sv = inputs.normal_f32_np(81, 3, (n, hkv, d, d), 1.0)
    zv = np.abs(inputs.normal_f32_np(81, 4, (n, hkv, d), 1.0))
    S, z = dev_f32(Sv), dev_f32(zv)
    Y = torch.empty(n, hq, b, d, device="cuda")
    bha.bha_hybrid_step_commit(dev_f32(Qv), dev_f32(Kv), dev_f32(Vv), S, Y, z=z)
    torch.cuda.synchronize()
    check_rel("step_commit_f32_y", host(Y), oracle.hybrid_step(Qv, Kv, Vv, Sv, zv), TOL_F32_REL)
    rS, rz = oracle.state_commit(Sv, zv, Kv, Vv)
    check_rel("step_commit_f32_S", host(S), rS, TOL_F32_REL)
    check_rel("step_commit_f32_z", host(z), rz, TOL_F32_REL)
