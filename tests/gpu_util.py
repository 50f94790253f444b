"""Helpers for the GPU parity tests: device copies of seeded inputs, error
metrics, guard-canary buffers and a parity log."""
import json
import os

import numpy as np

from block_hybrid_linear_b200 import inputs

# tolerances of the contract (relative L2 in bf16 mode also has a max-abs bound)
TOL_BF16_REL = 1e-2
TOL_BF16_ABS = 3e-2
TOL_F32_REL = 1e-4
# fp32 prefix state built from bf16 K/V with fp32 accumulation
TOL_STATE_REL = 1e-4


def dev_bf16(bits):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def dev_f32(x):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def host(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64).ravel()
    b = np.asarray(b, dtype=np.float64).ravel()
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def max_abs(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.max(np.abs(a - b))) if a.size else 0.0


def log_parity(name, **fields):
    path = os.environ.get("BHA_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(dict(test=name, **fields)) + "\n")


def bf16_case(seed, shape, std):
    bits, vals = inputs.normal_bf16_np(seed[0], seed[1], shape, std)
    return dev_bf16(bits), vals


class Guarded:
    """An output tensor inside a larger buffer with canaries on both sides,
    NaN-filled before the launch."""

    CANARY = 4096  # elements each side

    def __init__(self, shape, dtype):
        import torch
        numel = int(np.prod(shape))
        self.buf = torch.empty(numel + 2 * self.CANARY, dtype=dtype, device="cuda")
        self.buf.fill_(float("nan"))
        self.buf[: self.CANARY].fill_(-4096.0)
        self.buf[-self.CANARY:].fill_(-4096.0)
        self.t = self.buf[self.CANARY: self.CANARY + numel].view(*shape)

    def intact(self):
        import torch
        lo = self.buf[: self.CANARY].float()
        hi = self.buf[-self.CANARY:].float()
        return bool(torch.all(lo == -4096.0)) and bool(torch.all(hi == -4096.0))

    def no_nan(self):
        import torch
        return not bool(torch.isnan(self.t.float()).any())
