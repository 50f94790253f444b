"""Host-side checks of the C ABI (no GPU needed, no kernel launched).

The library must load on a machine without a GPU driver, export every
symbol include/bha.h declares, and reject bad arguments before touching the
device.  Fake (never dereferenced) pointers stand in for device buffers.
"""
import ctypes
import os
import re

import pytest

import oracle
from block_hybrid_linear_b200 import _lib
from block_hybrid_linear_b200 import build as bha_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bha.h")

GAP = 1 << 36  # 16-byte aligned fake device addresses, 64 GiB apart
A, B, C, D, E, F = (GAP * k for k in range(1, 7))


@pytest.fixture(scope="module")
def L():
    bha_build.build()
    return _lib.lib()


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bha_\w+)\s*\(", text)))


def test_header_and_binding_agree():
    assert declared_symbols() == sorted(_lib.EXPORTED)


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), name


def test_status_strings(L):
    for code, name in [(0, "BHA_OK"), (-1, "BHA_ERR_INVALID_ARG"), (-2, "BHA_ERR_UNSUPPORTED"),
                       (-3, "BHA_ERR_MISALIGNED"), (-4, "BHA_ERR_WORKSPACE"),
                       (-5, "BHA_ERR_CUDA"), (-6, "BHA_ERR_TIMEOUT"), (-7, "BHA_ERR_DEVICE")]:
        assert _lib.status_string(code) == name
    assert _lib.status_string(12345) == "BHA_ERR_UNKNOWN"
    assert _lib.bha_version() == 1


@pytest.mark.parametrize("L_", [0, 1, 2, 3, 4, 5, 10, 31, 32, 33, 64, 1000])
@pytest.mark.parametrize("B_", [1, 2, 3, 4, 7, 32, 64])
def test_block_partition_bit_exact_vs_oracle(L, L_, B_):
    assert _lib.bha_block_partition(L_, B_) == oracle.block_partition(L_, B_)


def test_block_partition_worked_example(L):
    # paper-daily summary, worked example: L=10, B=4 -> tokens 1-4, 5-8, 9-10
    assert _lib.bha_block_partition(10, 4) == [0, 4, 8, 10]


def test_block_partition_errors(L):
    buf = (ctypes.c_int * 2)()
    assert L.bha_block_partition(10, 0, buf, 2) == _lib.BHA_ERR_INVALID_ARG
    assert L.bha_block_partition(-1, 4, buf, 2) == _lib.BHA_ERR_INVALID_ARG
    assert L.bha_block_partition(10, 4, None, 4) == _lib.BHA_ERR_INVALID_ARG
    assert L.bha_block_partition(10, 4, buf, 2) == _lib.BHA_ERR_WORKSPACE


def step(L, Q=A, K=B, V=C, S=D, z=None, Y=E, n=2, hq=16, hkv=4, b=32, d=128, scale=0.0,
         flags=0, dtype=_lib.BHA_BF16):
    return L.bha_hybrid_step(Q, K, V, S, z, Y, n, hq, hkv, b, d, scale, flags, dtype, None)


def test_step_validation(L):
    assert step(L, Q=None) == _lib.BHA_ERR_INVALID_ARG
    assert step(L, S=None) == _lib.BHA_ERR_INVALID_ARG
    assert step(L, Y=None) == _lib.BHA_ERR_INVALID_ARG
    assert step(L, hq=6, hkv=4) == _lib.BHA_ERR_INVALID_ARG          # hq % hkv
    assert step(L, hkv=0) == _lib.BHA_ERR_INVALID_ARG
    assert step(L, n=-1) == _lib.BHA_ERR_INVALID_ARG
    assert step(L, b=0) == _lib.BHA_ERR_INVALID_ARG
    assert step(L, b=65) == _lib.BHA_ERR_UNSUPPORTED
    assert step(L, d=64) == _lib.BHA_ERR_UNSUPPORTED                 # bf16 needs d=128
    assert step(L, d=130, dtype=_lib.BHA_F32) == _lib.BHA_ERR_UNSUPPORTED
    assert step(L, d=18, dtype=_lib.BHA_F32) == _lib.BHA_ERR_UNSUPPORTED
    assert step(L, dtype=7) == _lib.BHA_ERR_UNSUPPORTED
    assert step(L, flags=2) == _lib.BHA_ERR_INVALID_ARG
    assert step(L, flags=_lib.BHA_FLAG_SHARED_DENOM) == _lib.BHA_ERR_INVALID_ARG  # no z
    assert step(L, Q=A + 8) == _lib.BHA_ERR_MISALIGNED
    assert step(L, Y=E + 2) == _lib.BHA_ERR_MISALIGNED
    assert step(L, flags=1, z=F + 4) == _lib.BHA_ERR_MISALIGNED
    assert step(L, Y=A) == _lib.BHA_ERR_INVALID_ARG                  # Y aliases Q
    assert step(L, Y=B + 4096) == _lib.BHA_ERR_INVALID_ARG           # Y overlaps K
    assert step(L, n=0) == _lib.BHA_OK                               # empty: no launch


def test_step_commit_validation(L):
    f = lambda **kw: L.bha_hybrid_step_commit(kw.get("Q", A), kw.get("K", B), kw.get("V", C),
                                              kw.get("S", D), kw.get("z", None), kw.get("Y", E),
                                              2, 16, 4, 32, 128, 0.0, kw.get("flags", 0),
                                              _lib.BHA_BF16, None)
    assert f(S=None) == _lib.BHA_ERR_INVALID_ARG
    assert f(flags=1) == _lib.BHA_ERR_INVALID_ARG            # shared needs z
    assert f(S=B) == _lib.BHA_ERR_INVALID_ARG                # S overlaps K
    assert f(z=D + 64) == _lib.BHA_ERR_INVALID_ARG           # z overlaps S
    assert f(Y=D) == _lib.BHA_ERR_INVALID_ARG                # Y overlaps S
    assert f(S=D + 4) == _lib.BHA_ERR_MISALIGNED


def test_valid_call_without_device_reports_cuda_error(L):
    # Arguments are valid, so the call reaches the runtime, which has no GPU here.
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert step(L) == _lib.BHA_ERR_CUDA


def test_commit_validation(L):
    f = lambda **kw: L.bha_state_commit(kw.get("K", A), kw.get("V", B), kw.get("n", 2), 4,
                                        kw.get("b", 32), kw.get("d", 128),
                                        kw.get("dtype", _lib.BHA_BF16), kw.get("S", C),
                                        kw.get("z", None), None)
    assert f(K=None) == _lib.BHA_ERR_INVALID_ARG
    assert f(S=None) == _lib.BHA_ERR_INVALID_ARG
    assert f(b=65) == _lib.BHA_ERR_UNSUPPORTED
    assert f(d=96) == _lib.BHA_ERR_UNSUPPORTED
    assert f(S=C + 4) == _lib.BHA_ERR_MISALIGNED
    assert f(S=A) == _lib.BHA_ERR_INVALID_ARG     # S overlaps K
    assert f(z=C + 64) == _lib.BHA_ERR_INVALID_ARG  # z overlaps S
    assert f(n=0) == _lib.BHA_OK


def test_prefill_validation_and_workspace(L):
    need = L.bha_state_prefill_workspace_size(64, 4, 32768, 128, _lib.BHA_BF16)
    # 256 units x 8 chunks of 4096 tokens x (128 x 128 + 128) fp32
    assert need == 256 * 8 * (128 * 128 + 128) * 4
    assert L.bha_state_prefill_workspace_size(64, 4, 32768, 128, _lib.BHA_F32) == 0
    assert L.bha_state_prefill_workspace_size(64, 4, 0, 128, _lib.BHA_BF16) == 0
    big = GAP * 16
    f = lambda **kw: L.bha_state_prefill(kw.get("K", A), kw.get("V", big), 64, 4,
                                         kw.get("T", 32768), 128, _lib.BHA_BF16,
                                         kw.get("S", 2 * big), None, kw.get("ws", 3 * big),
                                         kw.get("ws_bytes", need), None)
    assert f(ws=None) == _lib.BHA_ERR_WORKSPACE
    assert f(ws_bytes=need - 16) == _lib.BHA_ERR_WORKSPACE
    assert f(T=-1) == _lib.BHA_ERR_INVALID_ARG
    assert f(K=None) == _lib.BHA_ERR_INVALID_ARG
    assert f(ws=3 * big + 8) == _lib.BHA_ERR_MISALIGNED


def test_prefix_validation_and_workspace(L):
    need = L.bha_prefix_softmax_workspace_size(64, 16, 4, 32, 128, 32768, _lib.BHA_BF16)
    assert need > 0 and need % 16 == 0
    assert L.bha_prefix_softmax_workspace_size(64, 16, 4, 32, 128, 32768, _lib.BHA_F32) == 0
    big = GAP * 16
    f = lambda **kw: L.bha_prefix_softmax(A, kw.get("Kc", big), kw.get("Vc", 2 * big),
                                          kw.get("P", 32768), kw.get("cap", 32768), B, C,
                                          kw.get("Y", D), 64, 16, 4, 32, 128, 0.0,
                                          _lib.BHA_BF16, kw.get("ws", 3 * big),
                                          kw.get("ws_bytes", need), None)
    assert f(cap=100) == _lib.BHA_ERR_INVALID_ARG    # P > cap
    assert f(P=-1) == _lib.BHA_ERR_INVALID_ARG
    assert f(Kc=None) == _lib.BHA_ERR_INVALID_ARG
    assert f(ws=None) == _lib.BHA_ERR_WORKSPACE
    assert f(Y=A) == _lib.BHA_ERR_INVALID_ARG        # Y aliases Q
    assert f(Y=big + 64) == _lib.BHA_ERR_INVALID_ARG  # Y inside the cache


def test_feature_map_validation(L):
    """The _fm entry points: unknown map, W present without the projected
    map or missing with it, misaligned W, W overlapping an output."""
    RELU, ELU1, PROJ = _lib.BHA_FMAP_RELU, _lib.BHA_FMAP_ELU1, _lib.BHA_FMAP_RELU_PROJ
    W = F

    def st(fmap, w, **kw):
        return L.bha_hybrid_step_fm(A, B, C, D, None, kw.get("Y", E), 2, 16, 4, 32, 128, 0.0,
                                    0, _lib.BHA_BF16, fmap, w, None)

    def cm(fmap, w, **kw):
        return L.bha_state_commit_fm(A, B, 2, 4, 32, 128, _lib.BHA_BF16, fmap, w,
                                     kw.get("S", C), kw.get("z", None), None)

    def pf(fmap, w, **kw):
        return L.bha_state_prefill_fm(A, B, 2, 4, 64, 128, _lib.BHA_BF16, fmap, w,
                                      kw.get("S", C), None, None, 0, None)

    def sc(fmap, w, **kw):
        return L.bha_hybrid_step_commit_fm(A, B, C, kw.get("S", D), None, E, 2, 16, 4, 32, 128,
                                           0.0, 0, _lib.BHA_BF16, fmap, w, None)

    for f in (st, cm, pf, sc):
        assert f(3, None) == _lib.BHA_ERR_INVALID_ARG       # unknown map
        assert f(-1, None) == _lib.BHA_ERR_INVALID_ARG
        assert f(RELU, W) == _lib.BHA_ERR_INVALID_ARG       # W without the projected map
        assert f(ELU1, W) == _lib.BHA_ERR_INVALID_ARG
        assert f(PROJ, None) == _lib.BHA_ERR_INVALID_ARG    # projected map without W
        assert f(PROJ, W + 8) == _lib.BHA_ERR_MISALIGNED
    assert st(PROJ, W, Y=W + 4096) == _lib.BHA_ERR_INVALID_ARG   # Y overlaps W
    assert cm(PROJ, W, S=W - 4096) == _lib.BHA_ERR_INVALID_ARG   # S overlaps W
    assert cm(PROJ, W, z=W + 256) == _lib.BHA_ERR_INVALID_ARG    # z overlaps W
    assert pf(PROJ, W, S=W + 16) == _lib.BHA_ERR_INVALID_ARG
    assert sc(PROJ, W, S=W + 16) == _lib.BHA_ERR_INVALID_ARG
    import torch
    if not torch.cuda.is_available():
        # valid arguments reach the runtime, which has no GPU here
        for f in (st, cm, pf, sc):
            for fmap, w in ((RELU, None), (ELU1, None), (PROJ, W)):
                assert f(fmap, w) == _lib.BHA_ERR_CUDA


def test_paged_prefix_validation(L):
    """bha_prefix_softmax_paged: page sizes, counts, alignment, aliasing and
    the workspace (sized for the longest cache)."""
    n, hq, hkv, b, d, maxp, ps = 4, 16, 4, 32, 128, 64, 128
    need = L.bha_prefix_softmax_paged_workspace_size(n, hq, hkv, b, d, maxp, ps, _lib.BHA_BF16)
    # at most one piece per 32 key tiles of the longest cache (8192 keys + the
    # block: 129 tiles of 64 keys -> 5 partial slots per unit row), then the
    # device-side plan: a 256-byte header and one 16-byte work item per slot
    items = n * hkv * 5
    assert need == items * (128 * 128 + 256) * 4 + 256 + items * 16
    assert L.bha_prefix_softmax_paged_workspace_size(n, hq, hkv, b, d, maxp, ps,
                                                     _lib.BHA_F32) == 0
    big = GAP * 16

    def f(**kw):
        return L.bha_prefix_softmax_paged(
            A, kw.get("Kp", big), kw.get("Vp", 2 * big), kw.get("num_pages", 1000),
            kw.get("ps", ps), kw.get("table", C), kw.get("maxp", maxp), kw.get("plens", D),
            B, E, kw.get("Y", F), kw.get("n", n), hq, hkv, b, d, 0.0,
            kw.get("dtype", _lib.BHA_BF16), kw.get("ws", 3 * big), kw.get("ws_bytes", need), None)

    for bad in (8, 48, 512, 0):
        assert f(ps=bad) == _lib.BHA_ERR_UNSUPPORTED, bad
    assert f(maxp=0) == _lib.BHA_ERR_INVALID_ARG
    assert f(num_pages=0) == _lib.BHA_ERR_INVALID_ARG
    assert f(table=None) == _lib.BHA_ERR_INVALID_ARG
    assert f(plens=None) == _lib.BHA_ERR_INVALID_ARG
    assert f(table=C + 2) == _lib.BHA_ERR_MISALIGNED
    assert f(plens=D + 1) == _lib.BHA_ERR_MISALIGNED
    assert f(Kp=big + 8) == _lib.BHA_ERR_MISALIGNED
    assert f(ws=None) == _lib.BHA_ERR_WORKSPACE
    assert f(ws_bytes=need - 16) == _lib.BHA_ERR_WORKSPACE
    assert f(Y=big + 4096) == _lib.BHA_ERR_INVALID_ARG      # Y inside the pool
    assert f(Y=C) == _lib.BHA_ERR_INVALID_ARG               # Y over the page table
    assert f(n=0) == _lib.BHA_OK
    import torch
    if not torch.cuda.is_available():
        assert f() == _lib.BHA_ERR_CUDA
        assert f(ps=16, dtype=_lib.BHA_F32) == _lib.BHA_ERR_CUDA


def test_ragged_prefill_validation(L):
    need = L.bha_state_prefill_workspace_size(4, 4, 4096, 128, _lib.BHA_BF16)
    big = GAP * 16

    def f(**kw):
        return L.bha_state_prefill_ragged(A, big, kw.get("tl", C), kw.get("n", 4), 4, 4096, 128,
                                          _lib.BHA_BF16, 0, None, kw.get("S", 2 * big), None,
                                          3 * big if need else None, need, None)

    assert f(tl=None) == _lib.BHA_ERR_INVALID_ARG
    assert f(tl=C + 2) == _lib.BHA_ERR_MISALIGNED
    assert f(S=C) == _lib.BHA_ERR_INVALID_ARG               # S over the lengths
    assert f(n=0, tl=None) == _lib.BHA_OK
    import torch
    if not torch.cuda.is_available():
        assert f() == _lib.BHA_ERR_CUDA


def test_reuse_validation_and_workspace(L):
    """bha_prefix_softmax_reuse: bf16 only, k >= 0, the cache and the active
    list required to be disjoint from the inputs and each other, and a
    workspace that covers both the dense first step and a selecting step."""
    n, hq, hkv, b, d, P, k = 64, 16, 4, 32, 128, 32768, 8
    need = L.bha_prefix_softmax_reuse_workspace_size(n, hq, hkv, b, d, P, k, _lib.BHA_BF16)
    assert need > 0 and need % 16 == 0
    assert L.bha_prefix_softmax_reuse_workspace_size(n, hq, hkv, b, d, P, k, _lib.BHA_F32) == 0
    assert L.bha_prefix_softmax_reuse_workspace_size(n, hq, hkv, b, d, P, -1,
                                                     _lib.BHA_BF16) == 0
    # the dense first step (every token active) needs at least the exact path's partials
    assert need >= L.bha_prefix_softmax_reuse_workspace_size(n, hq, hkv, b, d, P, 0,
                                                             _lib.BHA_BF16)
    big = GAP * 16
    Qp, O, Lp, act = GAP * 7, GAP * 8, GAP * 9, GAP * 10

    def f(**kw):
        return L.bha_prefix_softmax_reuse(
            kw.get("Q", A), kw.get("Qprev", Qp), kw.get("Kc", big), kw.get("Vc", 2 * big),
            kw.get("P", P), kw.get("cap", P), B, C, kw.get("Y", D), kw.get("O", O),
            kw.get("Lp", Lp), kw.get("act", act), kw.get("k", k), n, hq, hkv, b, d, 0.0,
            kw.get("dtype", _lib.BHA_BF16), kw.get("ws", 3 * big), kw.get("ws_bytes", need),
            None)
    # fp32 reference mode: validated like bf16, no workspace, reaches the runtime
    assert f(dtype=_lib.BHA_F32, ws=None, ws_bytes=0) == _lib.BHA_ERR_CUDA
    assert L.bha_prefix_softmax_reuse(A, Qp, big, 2 * big, P, P, B, C, D, O, Lp, act, k, n, 512,
                                      4, b, d, 0.0, _lib.BHA_BF16, 3 * big, need,
                                      None) == _lib.BHA_ERR_UNSUPPORTED   # hq * b > 8192
    assert f(k=-1) == _lib.BHA_ERR_INVALID_ARG
    assert f(cap=100) == _lib.BHA_ERR_INVALID_ARG
    assert f(O=None) == _lib.BHA_ERR_INVALID_ARG
    assert f(Lp=None) == _lib.BHA_ERR_INVALID_ARG
    assert f(Kc=None) == _lib.BHA_ERR_INVALID_ARG
    assert f(ws=None) == _lib.BHA_ERR_WORKSPACE
    assert f(ws_bytes=need - 16) == _lib.BHA_ERR_WORKSPACE
    assert f(Y=A) == _lib.BHA_ERR_INVALID_ARG         # Y aliases Q
    assert f(Y=O) == _lib.BHA_ERR_INVALID_ARG         # Y aliases the cache
    assert f(O=Qp) == _lib.BHA_ERR_INVALID_ARG        # the cache aliases Qprev
    assert f(Lp=O + 64) == _lib.BHA_ERR_INVALID_ARG   # L_pre inside O_pre
    assert f(act=Lp) == _lib.BHA_ERR_INVALID_ARG      # the list over L_pre
    assert f(O=O + 8) == _lib.BHA_ERR_MISALIGNED
    assert f(act=act + 2) == _lib.BHA_ERR_MISALIGNED
    assert f(ws=big + 64) == _lib.BHA_ERR_INVALID_ARG  # workspace inside the cache
    # without a device the valid call gets as far as the runtime
    assert f() == _lib.BHA_ERR_CUDA
    assert f(Qprev=None, act=None) == _lib.BHA_ERR_CUDA
    assert f(Kc=None, Vc=None, P=0, cap=0) == _lib.BHA_ERR_CUDA


def test_product_path_and_oracle_share_nothing():
    """The CUDA package never imports or loads the oracle, and the oracle never
    imports the package (the seeded input generators live in the package's
    `inputs` module, which holds no arithmetic of the method and is imported by
    tests and the benchmark, not by the oracle)."""
    pkg = os.path.join(ROOT, "block_hybrid_linear_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), f
                assert "liboracle" not in text and "bha_oracle" not in text, f
    odir = os.path.join(ROOT, "oracle")
    for f in os.listdir(odir):
        if f.endswith((".py", ".c", ".h")):
            text = open(os.path.join(odir, f)).read()
            assert not re.search(r"^\s*(import|from)\s+block_hybrid_linear_b200\b", text, re.M), f
            assert "libbha" not in text and "#include \"bha" not in text, f
