"""GPU parity of ragged and paged batches, through the C ABI, against the fp64
oracle: the exact path over a paged KV cache with per-request cache lengths
(`bha_prefix_softmax_paged`) and prefill of prompts of different lengths
(`bha_state_prefill_ragged`).  The summary page pairs the method with
KV-cache management; its related work names PagedAttention.

Pool slots past a request's cache and padding rows past a prompt hold NaN:
the kernels must neither read them into a result nor let them through a
zero weight.  Page tables are random permutations with unused entries -1.
"""
import math

import numpy as np
import pytest

import oracle
from block_hybrid_linear_b200 import inputs
import block_hybrid_linear_b200 as bha

from gpu_util import (TOL_BF16_ABS, TOL_BF16_REL, TOL_F32_REL, TOL_STATE_REL, Guarded,
                      dev_bf16, dev_f32, host, log_parity, max_abs, rel_l2)

pytestmark = pytest.mark.gpu

STD = 1.0 / math.sqrt(128)
BF16_NAN = np.uint16(0x7FC0)
TOL_STATE_FMAP_REL = 5e-3


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


def dev_i32(x):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.int32)).cuda()


def check(name, got, ref, tol_rel, tol_abs=None, **kw):
    e_rel, e_abs = rel_l2(got, ref), max_abs(got, ref)
    log_parity(name, rel_l2=e_rel, max_abs=e_abs, **kw)
    assert e_rel <= tol_rel, (name, e_rel)
    if tol_abs is not None:
        assert e_abs <= tol_abs, (name, e_abs)


def paged_pool(seed, P_lens, hkv, ps, d, max_pages, dtype):
    """A pool holding each request's cache in random pages (other slots NaN),
    its page table (unused entries -1), and the pool's values."""
    rng = np.random.default_rng(seed)
    need = [(P + ps - 1) // ps for P in P_lens]
    num_pages = sum(need) + 3
    order = list(rng.permutation(num_pages))
    table = np.full((len(P_lens), max_pages), -1, dtype=np.int32)
    shape = (num_pages, hkv, ps, d)
    if dtype == "bf16":
        kb, kv = inputs.normal_bf16_np(seed, inputs.TID_KC, shape, STD)
        vb, vv = inputs.normal_bf16_np(seed, inputs.TID_VC, shape, STD)
    else:
        kv = inputs.normal_f32_np(seed, inputs.TID_KC, shape, 1.0)
        vv = inputs.normal_f32_np(seed, inputs.TID_VC, shape, 1.0)
        kb, vb = kv.copy(), vv.copy()
    used = np.zeros((num_pages, ps), dtype=bool)
    for i, P in enumerate(P_lens):
        for pg in range(need[i]):
            p = int(order.pop())
            table[i, pg] = p
            used[p, :min(ps, P - pg * ps)] = True
    nan = BF16_NAN if dtype == "bf16" else np.float32(np.nan)
    for arr in (kb, vb):
        arr.transpose(0, 2, 1, 3)[~used] = nan
    return kb, vb, kv, vv, table, num_pages


PAGED_CASES = [  # (n, hq, hkv, b, page_size, P_lens, max_pages)
    (3, 16, 4, 32, 128, [0, 200, 1000], 10),        # one tile per page, a request with no cache
    (4, 8, 2, 17, 16, [5, 0, 130, 700], 48),        # 8 pages per tile, ragged tails
    (2, 8, 2, 33, 64, [64, 4133], 80),              # several chunks; a chunk past request 0's cache
    (2, 16, 4, 64, 256, [300, 2500], 12),           # half a page per tile
    (1, 4, 1, 1, 32, [77], 3),                      # one active token
    (3, 16, 4, 32, 64, [0, 0, 0], 40),              # planned pieces, every cache empty
    (12, 16, 4, 32, 64, [9000] + [1, 2, 3, 5, 8, 13, 21, 34, 55, 89, 0], 150),  # one long
                                                    # request among tiny ones: 5 pieces + 11 single
]


@pytest.mark.parametrize("case", PAGED_CASES, ids=lambda c: "n%d_b%d_ps%d" % (c[0], c[3], c[4]))
def test_paged_prefix_bf16(case):
    import torch
    n, hq, hkv, b, ps, P_lens, max_pages = case
    seed = 1200 + ps + b
    kb, vb, kv, vv, table, num_pages = paged_pool(seed, P_lens, hkv, ps, 128, max_pages, "bf16")
    Qb, Qv = inputs.normal_bf16_np(seed, inputs.TID_Q, (n, hq, b, 128), STD)
    Kb, Kv = inputs.normal_bf16_np(seed, inputs.TID_K, (n, hkv, b, 128), STD)
    Vb, Vv = inputs.normal_bf16_np(seed, inputs.TID_V, (n, hkv, b, 128), STD)
    Y = Guarded((n, hq, b, 128), torch.bfloat16)
    need = bha.bha_prefix_softmax_paged_workspace_size(n, hq, hkv, b, 128, max_pages, ps)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda").fill_(255)
    bha.bha_prefix_softmax_paged(dev_bf16(Qb), dev_bf16(kb), dev_bf16(vb), dev_i32(table),
                                 dev_i32(P_lens), dev_bf16(Kb), dev_bf16(Vb), Y.t, workspace=ws)
    torch.cuda.synchronize()
    assert Y.intact() and Y.no_nan()
    ref = oracle.prefix_softmax_paged(Qv, kv, vv, table, P_lens, ps, Kv, Vv)
    check("paged_prefix_bf16", host(Y.t), ref, TOL_BF16_REL, TOL_BF16_ABS, case=str(case),
          ws=need)


def test_paged_prefix_planned_pieces_bf16():
    """A batch large enough that the device-side plan cuts long caches into
    pieces longer than the minimum (32 tiles of 64 keys): 32 requests with
    lengths drawn uniformly in [1, 6000] plus the edge lengths 0, 63, 64, 65
    and 6000, two query tiles per KV head.  Every output against the oracle."""
    import torch
    rng = np.random.default_rng(1250)
    n, hq, hkv, b, ps, max_pages = 32, 16, 4, 64, 64, 94
    P_lens = [0, 63, 64, 65, 6000] + [int(x) for x in rng.integers(1, 6001, n - 5)]
    kb, vb, kv, vv, table, num_pages = paged_pool(1250, P_lens, hkv, ps, 128, max_pages, "bf16")
    Qb, Qv = inputs.normal_bf16_np(1250, inputs.TID_Q, (n, hq, b, 128), STD)
    Kb, Kv = inputs.normal_bf16_np(1250, inputs.TID_K, (n, hkv, b, 128), STD)
    Vb, Vv = inputs.normal_bf16_np(1250, inputs.TID_V, (n, hkv, b, 128), STD)
    Y = Guarded((n, hq, b, 128), torch.bfloat16)
    need = bha.bha_prefix_softmax_paged_workspace_size(n, hq, hkv, b, 128, max_pages, ps)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda").fill_(255)
    bha.bha_prefix_softmax_paged(dev_bf16(Qb), dev_bf16(kb), dev_bf16(vb), dev_i32(table),
                                 dev_i32(P_lens), dev_bf16(Kb), dev_bf16(Vb), Y.t, workspace=ws)
    torch.cuda.synchronize()
    assert Y.intact() and Y.no_nan()
    ref = oracle.prefix_softmax_paged(Qv, kv, vv, table, P_lens, ps, Kv, Vv)
    check("paged_prefix_planned_bf16", host(Y.t), ref, TOL_BF16_REL, TOL_BF16_ABS, ws=need)


def test_paged_prefix_matches_contiguous_bf16():
    """A request's pages laid out in order reproduce the contiguous exact
    path on the same cache (both against the oracle's single definition)."""
    import torch
    n, hq, hkv, b, ps, P = 2, 16, 4, 32, 128, 1000
    Kc, Kcv = inputs.normal_bf16_np(1300, inputs.TID_KC, (n, hkv, P, 128), STD)
    Vc, Vcv = inputs.normal_bf16_np(1300, inputs.TID_VC, (n, hkv, P, 128), STD)
    Qb, Qv = inputs.normal_bf16_np(1300, inputs.TID_Q, (n, hq, b, 128), STD)
    Kb, Kv = inputs.normal_bf16_np(1300, inputs.TID_K, (n, hkv, b, 128), STD)
    Vb, Vv = inputs.normal_bf16_np(1300, inputs.TID_V, (n, hkv, b, 128), STD)
    npg = (P + ps - 1) // ps
    pool_k = np.zeros((n * npg, hkv, ps, 128), dtype=np.uint16)
    pool_v = np.zeros_like(pool_k)
    for i in range(n):
        for pg in range(npg):
            rows = min(ps, P - pg * ps)
            pool_k[i * npg + pg, :, :rows] = Kc[i, :, pg * ps:pg * ps + rows]
            pool_v[i * npg + pg, :, :rows] = Vc[i, :, pg * ps:pg * ps + rows]
    table = np.arange(n * npg, dtype=np.int32).reshape(n, npg)
    Yp = torch.empty(n, hq, b, 128, dtype=torch.bfloat16, device="cuda")
    Yc = torch.empty_like(Yp)
    need = bha.bha_prefix_softmax_paged_workspace_size(n, hq, hkv, b, 128, npg, ps)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    bha.bha_prefix_softmax_paged(dev_bf16(Qb), dev_bf16(pool_k), dev_bf16(pool_v),
                                 dev_i32(table), dev_i32([P] * n), dev_bf16(Kb), dev_bf16(Vb), Yp,
                                 workspace=ws)
    needc = bha.bha_prefix_softmax_workspace_size(n, hq, hkv, b, 128, P)
    wsc = torch.empty(max(needc, 16), dtype=torch.uint8, device="cuda")
    bha.bha_prefix_softmax(dev_bf16(Qb), dev_bf16(Kc), dev_bf16(Vc), P, dev_bf16(Kb),
                           dev_bf16(Vb), Yc, workspace=wsc)
    torch.cuda.synchronize()
    ref = oracle.prefix_softmax(Qv, Kcv, Vcv, P, Kv, Vv)
    check("paged_vs_oracle", host(Yp), ref, TOL_BF16_REL, TOL_BF16_ABS)
    check("contiguous_vs_oracle", host(Yc), ref, TOL_BF16_REL, TOL_BF16_ABS)
    check("paged_vs_contiguous", host(Yp), host(Yc), 5e-3)


def test_paged_prefix_f32():
    import torch
    n, hq, hkv, b, d, ps, P_lens, max_pages = 3, 4, 2, 7, 16, 16, [0, 21, 50], 5
    kb, vb, kv, vv, table, num_pages = paged_pool(1400, P_lens, hkv, ps, d, max_pages, "f32")
    Qv = inputs.normal_f32_np(1400, 0, (n, hq, b, d), 1.0)
    Kv = inputs.normal_f32_np(1400, 1, (n, hkv, b, d), 1.0)
    Vv = inputs.normal_f32_np(1400, 2, (n, hkv, b, d), 1.0)
    Y = Guarded((n, hq, b, d), torch.float32)
    bha.bha_prefix_softmax_paged(dev_f32(Qv), dev_f32(kb), dev_f32(vb), dev_i32(table),
                                 dev_i32(P_lens), dev_f32(Kv), dev_f32(Vv), Y.t)
    torch.cuda.synchronize()
    assert Y.intact() and Y.no_nan()
    ref = oracle.prefix_softmax_paged(Qv, kv, vv, table, P_lens, ps, Kv, Vv)
    check("paged_prefix_f32", host(Y.t), ref, TOL_F32_REL)


# ------------------------------------------------------------ ragged prefill

FMAPS = {"relu": bha.BHA_FMAP_RELU, "elu1": bha.BHA_FMAP_ELU1, "proj": bha.BHA_FMAP_RELU_PROJ}


@pytest.mark.parametrize("fmap", list(FMAPS), ids=list(FMAPS))
def test_ragged_prefill_bf16(fmap):
    import torch
    f = FMAPS[fmap]
    T_lens = [0, 1, 63, 64, 65, 1000, 4113]
    n, hkv, Tmax = len(T_lens), 2, max(T_lens)
    Kb, Kv = inputs.normal_bf16_np(1500, inputs.TID_KP, (n, hkv, Tmax, 128), STD)
    Vb, Vv = inputs.normal_bf16_np(1500, inputs.TID_VP, (n, hkv, Tmax, 128), STD)
    for i, T in enumerate(T_lens):
        Kb[i, :, T:] = BF16_NAN
        Vb[i, :, T:] = BF16_NAN
    W = Wv = None
    if f == bha.BHA_FMAP_RELU_PROJ:
        Wb, Wv = inputs.normal_bf16_np(1500, 90, (hkv, 128, 128), STD)
        W = dev_bf16(Wb)
    S = Guarded((n, hkv, 128, 128), torch.float32)
    z = Guarded((n, hkv, 128), torch.float32)
    need = bha.bha_state_prefill_workspace_size(n, hkv, Tmax, 128)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda").fill_(255)
    bha.bha_state_prefill_ragged(dev_bf16(Kb), dev_bf16(Vb), dev_i32(T_lens), S.t, z.t, fmap=f,
                                 W=W, workspace=ws)
    torch.cuda.synchronize()
    assert S.intact() and S.no_nan() and z.intact() and z.no_nan()
    rS, rz = oracle.state_prefill_ragged(Kv, Vv, T_lens, fmap=f, W=Wv)
    assert np.all(host(S.t)[0] == 0) and np.all(host(z.t)[0] == 0)
    tol = TOL_STATE_REL if f == bha.BHA_FMAP_RELU else TOL_STATE_FMAP_REL
    check("ragged_prefill_S", host(S.t), rS, tol, fmap=fmap, ws=need)
    check("ragged_prefill_z", host(z.t), rz, tol, fmap=fmap)


def test_ragged_prefill_f32():
    import torch
    T_lens = [0, 3, 40]
    n, hkv, Tmax, d = len(T_lens), 2, 40, 16
    Kv = inputs.normal_f32_np(1600, 3, (n, hkv, Tmax, d), 1.0)
    Vv = inputs.normal_f32_np(1600, 4, (n, hkv, Tmax, d), 1.0)
    Kd, Vd = Kv.copy(), Vv.copy()
    for i, T in enumerate(T_lens):
        Kd[i, :, T:] = np.nan
        Vd[i, :, T:] = np.nan
    S = torch.empty(n, hkv, d, d, device="cuda")
    z = torch.empty(n, hkv, d, device="cuda")
    bha.bha_state_prefill_ragged(dev_f32(Kd), dev_f32(Vd), dev_i32(T_lens), S, z)
    torch.cuda.synchronize()
    rS, rz = oracle.state_prefill_ragged(Kv, Vv, T_lens)
    check("ragged_prefill_f32_S", host(S), rS, TOL_F32_REL)
    check("ragged_prefill_f32_z", host(z), rz, TOL_F32_REL)
