"""The allocation-free prefill entry point, against the regular one.

bha_state_prefill_noalloc is for callers that cannot allocate device memory
(plugins in a host application that owns all device memory, runtimes that
forbid allocation while serving): it takes the prefill's chunk workspace
from the library's own fixed device array instead of a caller buffer.  This
file is collected last so that, if it fails, a run stopping at the first
failure has run every other test; it passes alone in a fresh process too
(the first call does the one-time set-up).
"""
import ctypes
import math

import numpy as np
import pytest

import block_hybrid_linear_b200 as bha
from block_hybrid_linear_b200 import _lib

from gpu_util import TOL_STATE_REL, bf16_case, host, rel_l2

pytestmark = pytest.mark.gpu

STD = 1.0 / math.sqrt(128)


def test_noalloc_prefill_matches_workspace_prefill_twice():
    """Two calls in a row, the second smaller than the first: both run the same
    kernels, plan and fixed-order chunk reduce as the workspace prefill, so the
    states must be bit-identical; the second call also shows that partials a
    larger earlier call left in the shared array are never read."""
    import torch
    from block_hybrid_linear_b200 import build
    build.build()
    for call, (n, hkv, T) in enumerate(((2, 2, 5000), (1, 2, 3000))):
        need = bha.bha_state_prefill_workspace_size(n, hkv, T, 128)
        assert 0 < need <= 32 << 20   # uses the scratch, within its limit
        K, _ = bf16_case((900 + call, 3), (n, hkv, T, 128), STD)
        V, _ = bf16_case((900 + call, 4), (n, hkv, T, 128), STD)
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        S_ref = torch.empty(n, hkv, 128, 128, device="cuda")
        z_ref = torch.empty(n, hkv, 128, device="cuda")
        bha.bha_state_prefill(K, V, S_ref, z_ref, workspace=ws)
        S = torch.full((n, hkv, 128, 128), float("nan"), device="cuda")
        z = torch.full((n, hkv, 128), float("nan"), device="cuda")
        bha.bha_state_prefill_noalloc(K, V, S, z)
        torch.cuda.synchronize()
        assert rel_l2(host(S), host(S_ref)) <= TOL_STATE_REL
        assert rel_l2(host(z), host(z_ref)) <= TOL_STATE_REL
        assert torch.equal(S, S_ref) and torch.equal(z, z_ref), call
    assert bha.bha_device_error(True) == 0


def test_noalloc_prefill_rejects_sizes_beyond_the_scratch():
    import torch
    # 64 requests x 4 KV heads x 32768 tokens need ~135 MB of chunk partials
    need = bha.bha_state_prefill_workspace_size(64, 4, 32768, 128)
    assert need > 32 << 20
    K = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    S = torch.empty(16, device="cuda")
    rc = _lib.lib().bha_state_prefill_noalloc(
        ctypes.c_void_p(K.data_ptr()), ctypes.c_void_p(K.data_ptr()), 64, 4, 32768, 128,
        _lib.BHA_BF16, ctypes.c_void_p(S.data_ptr()), None, None)
    assert rc == _lib.BHA_ERR_WORKSPACE
