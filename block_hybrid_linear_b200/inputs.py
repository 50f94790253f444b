"""Seeded synthetic inputs and workload shapes for block-hybrid attention.

This module holds no arithmetic of the method: it only draws random numbers,
rounds them to bf16, and describes the workloads' shapes.  It serves both the
CUDA path's callers (tests, benchmark) and the CPU oracle's callers, so that
both sides see identical inputs.

Two generators:

* ``normal_*_np`` -- NumPy ``default_rng(SeedSequence([seed, tensor_id,
  row]))`` with one independent stream per leading-dimension row, so any
  sampled batch row can be regenerated on its own.  float32 normals scaled by
  ``std``; bf16 values are the round-to-nearest-even of those float32 values.
* ``normal_bf16_torch`` -- the same distribution drawn by torch's generator
  on a device, for bulk benchmark data (gigabytes) where the host would take
  too long.  Values differ from the NumPy stream but are equally seeded.

The pages measure on HumanEval, MBPP+ and CMATH with trained LLaDA models;
those datasets and weights are not available, so Gaussian Q/K/V of the
attention layer's shape stand in for real activations.  The path is dense
and fixed-shape, so timing does not depend on the values.
"""
import math

import numpy as np

# tensor ids of the seeded streams
TID_Q, TID_K, TID_V, TID_KP, TID_VP, TID_S, TID_Z, TID_KC, TID_VC = range(9)


def step_tid(base_tid: int, blk: int, step: int, steps_per_block: int = 8):
    """Stream id of a per-(block, denoising step) tensor."""
    return base_tid + 16 * (blk * steps_per_block + step + 1)


def f32_to_bf16_bits(x):
    """Round float32 -> bf16 bit patterns, round-to-nearest-even (finite x)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits):
    """Exact widening of bf16 bit patterns to float32."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32)
    return (b << np.uint32(16)).view(np.float32)


def _rows_normal_f32(seed, tid, shape, std, row_offset=0):
    shape = tuple(int(s) for s in shape)
    out = np.empty(shape, dtype=np.float32)
    if len(shape) == 0 or shape[0] == 0:
        return out
    for r in range(shape[0]):
        rng = np.random.default_rng(
            np.random.SeedSequence([int(seed), int(tid), int(r + row_offset)]))
        out[r] = rng.standard_normal(shape[1:], dtype=np.float32) * np.float32(std)
    return out


def normal_f32_np(seed, tid, shape, std=1.0, row_offset=0):
    """float32 N(0, std^2) with one stream per leading row."""
    return _rows_normal_f32(seed, tid, shape, std, row_offset)


def normal_bf16_np(seed, tid, shape, std=1.0, row_offset=0):
    """bf16 N(0, std^2): returns (bits uint16, exact values as float32)."""
    x = _rows_normal_f32(seed, tid, shape, std, row_offset)
    bits = f32_to_bf16_bits(x)
    return bits, bf16_bits_to_f32(bits)


def normal_bf16_torch(seed, tid, shape, std, device):
    """bf16 N(0, std^2) drawn on ``device`` with a seeded torch generator."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1000003 + int(tid) * 7919) % (2 ** 63))
    x = torch.randn(tuple(int(s) for s in shape), generator=g, device=device,
                    dtype=torch.float32)
    x.mul_(float(std))
    return x.to(torch.bfloat16)


def synthetic_state_np(seed, n, hkv, d, T, sigma):
    """A prefix state with the statistics of a T-token prefill of N(0, sigma^2)
    keys and values, drawn directly (no arithmetic of the method).

    Entries of S are ~ N(0, T * sigma^4 / 2); entries of z are the mean
    T * sigma / sqrt(2 pi) plus N(0, T * sigma^2 * (1/2 - 1/(2 pi))) noise.
    Returns float32 (S [n, hkv, d, d], z [n, hkv, d]).
    """
    s_std = math.sqrt(max(T, 1) * sigma ** 4 / 2.0)
    S = normal_f32_np(seed, TID_S, (n, hkv, d, d), s_std)
    z_mean = T * sigma / math.sqrt(2.0 * math.pi)
    z_std = math.sqrt(max(T, 1) * sigma ** 2 * (0.5 - 1.0 / (2.0 * math.pi)))
    z = normal_f32_np(seed, TID_Z, (n, hkv, d), z_std) + np.float32(z_mean)
    return S, np.abs(z).astype(np.float32)


# Workloads by name: the worked example and the four attention-layer
# workloads of a 16B dLLM (16 query / 4 KV heads, head dim 128, active block 32).
WORKLOADS = {
    "worked-example": dict(n=1, hq=1, hkv=1, d=16, L=10, B=4, dtype="f32", std=1.0,
                           seed=1000),
    "single-step": dict(n=8, hq=16, hkv=4, d=128, b=32, P=4096, dtype="bf16",
                        std=1.0 / math.sqrt(128), seed=2000),
    "generation-loop": dict(n=32, hq=16, hkv=4, d=128, b=32, prompt=1024, blocks=32, steps=8,
                            dtype="bf16", std=1.0 / math.sqrt(128), seed=3000),
    "long-prefix": dict(n=64, hq=16, hkv=4, d=128, b=32, P=32768, dtype="bf16",
                        std=1.0 / math.sqrt(128), seed=4000),
    "stack-sweep": dict(layers=20, hybrid_layers=6, hq=16, hkv=4, d=128, b=32, P=8192,
                        dtype="bf16", std=1.0 / math.sqrt(128), seed=5000),
}
