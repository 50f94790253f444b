"""Pins of the fp64 CPU oracle against what the pages and the mathematics fix.

None of these checks re-types the oracle's own formula: each compares the
oracle with an independent statement of the same fact -- a library routine
(torch's scaled_dot_product_attention on CPU in float64, NumPy matmul), a
brute-force sum over individual prefix tokens, a closed form or special case,
an invariant (additivity, order invariance, linearity), or the worked example
of the paper-daily summary page of "Retrofitting Linear Attention into
Diffusion Language Models" (section 具体技术细节示例).

Each pin is a function of the implementation under test, so that the same
pins can be shown to fail on planted mistakes (see ``test_pins_catch_*``).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from block_hybrid_linear_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TOL = 1e-10


def relu(x):
    return np.maximum(x, 0.0)


def sdpa(Q, K, V, scale=None):
    """Library softmax attention (torch, CPU, float64), GQA by contiguous
    head grouping (query head h uses KV head h // G), no mask."""
    q = torch.from_numpy(np.asarray(Q, dtype=np.float64))
    k = torch.from_numpy(np.asarray(K, dtype=np.float64))
    v = torch.from_numpy(np.asarray(V, dtype=np.float64))
    G = q.shape[1] // k.shape[1]
    k = k.repeat_interleave(G, dim=1)
    v = v.repeat_interleave(G, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(
        q, k, v, scale=scale).numpy()


def rnd(seed, shape, std=1.0):
    return inputs.normal_f32_np(seed, 0, shape, std).astype(np.float64)


def relerr(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = max(np.linalg.norm(b.ravel()), 1e-300)
    return float(np.linalg.norm((a - b).ravel()) / den)


class Impl:
    """Bundle of the oracle routines a pin exercises (real or mutant)."""

    def __init__(self, step=None, prefill=None, commit=None, prefix=None):
        self.step = step or oracle.hybrid_step
        self.prefill = prefill or oracle.state_prefill
        self.commit = commit or oracle.state_commit
        self.prefix = prefix or oracle.prefix_softmax


REAL = Impl()


# ---------------------------------------------------------------- pins ------

def pin_zero_prefix_is_softmax(impl, shared=False):
    """S = 0 (and z = 0): the hybrid output is textbook softmax attention."""
    n, hq, hkv, b, d = 2, 4, 2, 7, 16
    Q, K, V = rnd(1, (n, hq, b, d)), rnd(2, (n, hkv, b, d)), rnd(3, (n, hkv, b, d))
    S = np.zeros((n, hkv, d, d))
    z = np.zeros((n, hkv, d))
    y = impl.step(Q, K, V, S, z, 0.0, shared)
    return relerr(y, sdpa(Q, K, V, scale=1.0 / math.sqrt(d)))


def pin_linear_term_bruteforce(impl):
    """y - softmax part == sum over prefix tokens t of (phi(q).phi(k_t)) v_t,
    summed token by token (no state S), for a prefix S built by prefill."""
    n, hq, hkv, b, d, T = 1, 4, 2, 5, 8, 9
    Q, K, V = rnd(11, (n, hq, b, d)), rnd(12, (n, hkv, b, d)), rnd(13, (n, hkv, b, d))
    Kp, Vp = rnd(14, (n, hkv, T, d)), rnd(15, (n, hkv, T, d))
    S, z = impl.prefill(Kp, Vp)
    y = impl.step(Q, K, V, S, z, 0.0, False)
    soft = sdpa(Q, K, V, scale=1.0 / math.sqrt(d))
    G = hq // hkv
    lin = np.zeros_like(soft)
    for h in range(hq):
        g = h // G
        for i in range(b):
            fq = relu(Q[0, h, i])
            for t in range(T):
                lin[0, h, i] += float(fq @ relu(Kp[0, g, t])) * Vp[0, g, t]
    return relerr(y - soft, lin)


def pin_associativity(impl):
    """phi(Q)(phi(K)^T V) == (phi(Q) phi(K)^T) V, the right side by NumPy."""
    n, hq, hkv, b, d, T = 2, 2, 1, 6, 12, 20
    Q, K, V = rnd(21, (n, hq, b, d)), rnd(22, (n, hkv, b, d)), rnd(23, (n, hkv, b, d))
    Kp, Vp = rnd(24, (n, hkv, T, d)), rnd(25, (n, hkv, T, d))
    S, z = impl.prefill(Kp, Vp)
    y = impl.step(Q, K, V, S, z, 0.0, False)
    y0 = impl.step(Q, K, V, np.zeros_like(S), z, 0.0, False)
    G = hq // hkv
    A = relu(Q) @ np.swapaxes(relu(Kp), -1, -2).repeat(G, axis=1)
    expect = A @ Vp.repeat(G, axis=1)
    return relerr(y - y0, expect)


def pin_prefill_matches_numpy(impl):
    """S = relu(K)^T V and z = column sums of relu(K), by NumPy."""
    Kp, Vp = rnd(31, (3, 2, 33, 16)), rnd(32, (3, 2, 33, 16))
    S, z = impl.prefill(Kp, Vp)
    eS = np.swapaxes(relu(Kp), -1, -2) @ Vp
    ez = relu(Kp).sum(axis=-2)
    return max(relerr(S, eS), relerr(z, ez))


def pin_prefill_equals_commits(impl):
    """Worked example: S_{1,2} = S_1 + S_2; prefill over blocks 1..k equals
    committing them one by one from zero, in any block order."""
    d, B, nblk = 8, 4, 3
    Kp, Vp = rnd(41, (2, 1, B * nblk, d)), rnd(42, (2, 1, B * nblk, d))
    S_all, z_all = impl.prefill(Kp, Vp)
    worst = 0.0
    for order in ([0, 1, 2], [2, 0, 1], [1, 2, 0]):
        S = np.zeros((2, 1, d, d))
        z = np.zeros((2, 1, d))
        for blk in order:
            sl = slice(blk * B, (blk + 1) * B)
            S, z = impl.commit(S, z, Kp[:, :, sl], Vp[:, :, sl])
        worst = max(worst, relerr(S, S_all), relerr(z, z_all))
    return worst


def pin_b1_softmax_is_v(impl):
    """One active token: its softmax weight is exactly 1, so y = v (S = 0)."""
    n, hq, hkv, d = 2, 4, 2, 16
    Q, K, V = rnd(51, (n, hq, 1, d)), rnd(52, (n, hkv, 1, d)), rnd(53, (n, hkv, 1, d))
    y = impl.step(Q, K, V, np.zeros((n, hkv, d, d)), None, 0.0, False)
    return relerr(y, V.repeat(hq // hkv, axis=1))


def pin_negative_queries_kill_linear(impl):
    """phi(q) = 0 for all-negative q: the linear term vanishes for any S."""
    n, hq, hkv, b, d = 1, 2, 1, 5, 8
    Q = -np.abs(rnd(61, (n, hq, b, d))) - 0.1
    K, V = rnd(62, (n, hkv, b, d)), rnd(63, (n, hkv, b, d))
    S = rnd(64, (n, hkv, d, d), 10.0)
    return relerr(impl.step(Q, K, V, S, None, 0.0, False),
                  sdpa(Q, K, V, scale=1.0 / math.sqrt(d)))


def pin_constant_keys_mean(impl):
    """All block keys equal: uniform weights, so y = mean of V (S = 0)."""
    n, hq, hkv, b, d = 1, 2, 1, 6, 8
    Q = rnd(71, (n, hq, b, d))
    K = np.broadcast_to(rnd(72, (n, hkv, 1, d)), (n, hkv, b, d)).copy()
    V = rnd(73, (n, hkv, b, d))
    y = impl.step(Q, K, V, np.zeros((n, hkv, d, d)), None, 0.0, False)
    expect = np.broadcast_to(V.mean(axis=2, keepdims=True), (n, hkv, b, d))
    return relerr(y, expect.repeat(hq, axis=1))


def pin_linear_in_S(impl):
    """y(S1 + S2) - y(0) = (y(S1) - y(0)) + (y(S2) - y(0))."""
    n, hq, hkv, b, d = 1, 4, 2, 3, 8
    Q, K, V = rnd(81, (n, hq, b, d)), rnd(82, (n, hkv, b, d)), rnd(83, (n, hkv, b, d))
    S1, S2 = rnd(84, (n, hkv, d, d)), rnd(85, (n, hkv, d, d))
    f = lambda S: impl.step(Q, K, V, S, None, 0.0, False)
    y0 = f(np.zeros_like(S1))
    return relerr(f(S1 + S2) - y0, (f(S1) - y0) + (f(S2) - y0))


def pin_gqa_head_map(impl):
    """Query head h uses KV head h // G: compare each head with a 1-head call
    whose KV tensors are that KV head's."""
    n, hq, hkv, b, d = 1, 6, 2, 4, 8
    Q, K, V = rnd(91, (n, hq, b, d)), rnd(92, (n, hkv, b, d)), rnd(93, (n, hkv, b, d))
    S = rnd(94, (n, hkv, d, d))
    y = impl.step(Q, K, V, S, None, 0.0, False)
    worst = 0.0
    for h in range(hq):
        g = h // (hq // hkv)
        yh = impl.step(Q[:, h:h + 1], K[:, g:g + 1], V[:, g:g + 1],
                       S[:, g:g + 1], None, 0.0, False)
        worst = max(worst, relerr(y[:, h:h + 1], yh))
    return worst


def pin_shared_bruteforce(impl):
    """Shared denominator: y = sum_j w_j v_j / sum_j w_j, with w = exp(s_j)
    over block tokens and w = phi(q).phi(k_t) over prefix tokens, summed token
    by token (no S, z, max shift)."""
    n, hq, hkv, b, d, T = 1, 2, 1, 4, 8, 6
    Q, K, V = rnd(101, (n, hq, b, d)), rnd(102, (n, hkv, b, d)), rnd(103, (n, hkv, b, d))
    Kp, Vp = rnd(104, (n, hkv, T, d)), rnd(105, (n, hkv, T, d))
    S, z = impl.prefill(Kp, Vp)
    y = impl.step(Q, K, V, S, z, 0.0, True)
    expect = np.zeros_like(y)
    sc = 1.0 / math.sqrt(d)
    for h in range(hq):
        for i in range(b):
            q = Q[0, h, i]
            num = np.zeros(d)
            den = 0.0
            for j in range(b):
                w = math.exp(sc * float(q @ K[0, 0, j]))
                num += w * V[0, 0, j]
                den += w
            for t in range(T):
                w = float(relu(q) @ relu(Kp[0, 0, t]))
                num += w * Vp[0, 0, t]
                den += w
            expect[0, h, i] = num / den
    return relerr(y, expect)


def pin_prefix_softmax_sdpa(impl):
    """Exact prefix softmax == library attention over [cache[:P] || block];
    cache slots past P are ignored."""
    n, hq, hkv, b, d, P, cap = 2, 4, 2, 5, 16, 11, 14
    Q, K, V = rnd(111, (n, hq, b, d)), rnd(112, (n, hkv, b, d)), rnd(113, (n, hkv, b, d))
    Kc, Vc = rnd(114, (n, hkv, cap, d)), rnd(115, (n, hkv, cap, d))
    Kc[:, :, P:] = 1e3
    Vc[:, :, P:] = -1e3
    y = impl.prefix(Q, Kc, Vc, P, K, V)
    Kall = np.concatenate([Kc[:, :, :P], K], axis=2)
    Vall = np.concatenate([Vc[:, :, :P], V], axis=2)
    return relerr(y, sdpa(Q, Kall, Vall, scale=1.0 / math.sqrt(d)))


def pin_prefix_softmax_p0(impl):
    """P = 0: exact prefix softmax equals the hybrid step with S = 0."""
    n, hq, hkv, b, d = 1, 4, 1, 6, 8
    Q, K, V = rnd(121, (n, hq, b, d)), rnd(122, (n, hkv, b, d)), rnd(123, (n, hkv, b, d))
    Kc = np.zeros((n, hkv, 4, d))
    y = impl.prefix(Q, Kc, Kc, 0, K, V)
    y2 = impl.step(Q, K, V, np.zeros((n, hkv, d, d)), None, 0.0, False)
    return relerr(y, y2)


ALL_PINS = [
    pin_zero_prefix_is_softmax, pin_linear_term_bruteforce, pin_associativity,
    pin_prefill_matches_numpy, pin_prefill_equals_commits, pin_b1_softmax_is_v,
    pin_negative_queries_kill_linear, pin_constant_keys_mean, pin_linear_in_S,
    pin_gqa_head_map, pin_shared_bruteforce, pin_prefix_softmax_sdpa,
    pin_prefix_softmax_p0,
]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    assert pin(REAL) < TOL


def test_zero_prefix_shared_is_softmax():
    assert pin_zero_prefix_is_softmax(REAL, shared=True) < TOL


def test_scale_argument():
    """An explicit scale replaces 1/sqrt(d) (checked against the library)."""
    Q, K, V = rnd(131, (1, 2, 5, 8)), rnd(132, (1, 1, 5, 8)), rnd(133, (1, 1, 5, 8))
    y = oracle.hybrid_step(Q, K, V, np.zeros((1, 1, 8, 8)), None, 0.37)
    assert relerr(y, sdpa(Q, K, V, scale=0.37)) < TOL


# ------------------------------------------------- the worked example ------

def test_block_partition_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    assert oracle.block_partition(g["L"], g["B"]) == g["bounds"]
    one_based = [[a + 1, b] for a, b in zip(g["bounds"][:-1], g["bounds"][1:])]
    assert one_based == g["blocks_1based"]


@pytest.mark.parametrize("L", [0, 1, 3, 4, 5, 31, 32, 33, 100])
@pytest.mark.parametrize("B", [1, 2, 4, 7, 32])
def test_block_partition_invariants(L, B):
    bounds = oracle.block_partition(L, B)
    assert bounds[0] == 0 and bounds[-1] == L
    sizes = np.diff(bounds)
    assert len(sizes) == (L + B - 1) // B
    assert all(s == B for s in sizes[:-1])
    if L:
        assert 1 <= sizes[-1] <= B


def test_block_partition_rejects_bad_args():
    with pytest.raises(ValueError):
        oracle.block_partition(10, 0)


def test_worked_example_structure():
    """L=10, B=4, d=16, phi=ReLU, fp32 N(0,1) inputs from seed: block 1 is
    softmax only; block 2 adds phi(Q_2) S_1; block 3 uses S_1 + S_2."""
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    cfg = inputs.WORKLOADS["worked-example"]
    d, L = cfg["d"], g["L"]
    bounds = oracle.block_partition(L, g["B"])
    seq_q = inputs.normal_f32_np(cfg["seed"], inputs.TID_Q, (1, 1, L, d)).astype(np.float64)
    seq_k = inputs.normal_f32_np(cfg["seed"], inputs.TID_K, (1, 1, L, d)).astype(np.float64)
    seq_v = inputs.normal_f32_np(cfg["seed"], inputs.TID_V, (1, 1, L, d)).astype(np.float64)
    blocks = [(a, b) for a, b in zip(bounds[:-1], bounds[1:])]
    Qs = [[seq_q[:, :, a:b]] for a, b in blocks]
    Ks = [[seq_k[:, :, a:b]] for a, b in blocks]
    Vs = [[seq_v[:, :, a:b]] for a, b in blocks]
    outs, S_final, _ = oracle.generate(Qs, Ks, Vs)
    sc = 1.0 / math.sqrt(d)
    for bi, prev in enumerate(g["previous_blocks"]):
        a, b = blocks[bi]
        soft = sdpa(Qs[bi][0], Ks[bi][0], Vs[bi][0], scale=sc)
        lin = np.zeros_like(soft)
        prev_tokens = [t for pb in prev for t in range(*blocks[pb - 1])]
        for i in range(b - a):
            fq = relu(seq_q[0, 0, a + i])
            for t in prev_tokens:
                lin[0, 0, i] += float(fq @ relu(seq_k[0, 0, t])) * seq_v[0, 0, t]
        if not prev:
            assert relerr(outs[bi][0], soft) < TOL      # block 1: softmax only
        assert relerr(outs[bi][0], soft + lin) < TOL
    S1, _ = oracle.state_prefill(seq_k[:, :, 0:4], seq_v[:, :, 0:4])
    S2, _ = oracle.state_prefill(seq_k[:, :, 4:8], seq_v[:, :, 4:8])
    S12, _ = oracle.state_prefill(seq_k[:, :, 0:8], seq_v[:, :, 0:8])
    assert relerr(S12, S1 + S2) < TOL                    # S_{1,2} = S_1 + S_2
    S123, _ = oracle.state_prefill(seq_k, seq_v)
    assert relerr(S_final, S123) < TOL


def test_threads_do_not_change_results():
    Q, K, V = rnd(141, (3, 4, 9, 16)), rnd(142, (3, 2, 9, 16)), rnd(143, (3, 2, 9, 16))
    S = rnd(144, (3, 2, 16, 16))
    oracle.set_threads(1)
    y1 = oracle.hybrid_step(Q, K, V, S)
    oracle.set_threads(4)
    y4 = oracle.hybrid_step(Q, K, V, S)
    oracle.set_threads(1)
    assert np.array_equal(y1, y4)


# ------------------------------------------- planted mistakes are caught ----

def _mutant_step_transposed_S(Q, K, V, S, z=None, scale=0.0, shared=False):
    return oracle.hybrid_step(Q, K, V, np.swapaxes(S, -1, -2), z, scale, shared)


def _mutant_step_no_scale(Q, K, V, S, z=None, scale=0.0, shared=False):
    return oracle.hybrid_step(Q, K, V, S, z, 1.0, shared)


def _mutant_step_dropped_linear(Q, K, V, S, z=None, scale=0.0, shared=False):
    return oracle.hybrid_step(Q, K, V, np.zeros_like(S), z, scale, shared)


def _mutant_step_wrong_gqa(Q, K, V, S, z=None, scale=0.0, shared=False):
    hq, hkv = Q.shape[1], K.shape[1]
    out = np.zeros(Q.shape)
    for h in range(hq):
        g = h % hkv                                   # interleaved, not grouped
        zz = None if z is None else z[:, g:g + 1]
        out[:, h:h + 1] = oracle.hybrid_step(Q[:, h:h + 1], K[:, g:g + 1],
                                             V[:, g:g + 1], S[:, g:g + 1], zz,
                                             scale, shared)
    return out


def _mutant_prefill_no_relu(K, V, with_z=True):
    Kpos = np.abs(np.asarray(K, dtype=np.float64))   # |k| instead of relu(k)
    return oracle.state_prefill(Kpos, V, with_z)


def _mutant_commit_sign(S, z, Kb, Vb):
    S2, z2 = oracle.state_commit(S, z, Kb, Vb)
    return 2 * np.asarray(S) - S2, z2


def _mutant_prefix_drops_block(Q, Kc, Vc, P, K, V, scale=0.0):
    return oracle.prefix_softmax(Q, Kc, Vc, P, K * 0.0, V, scale)


MUTANTS = {
    "transposed_S": Impl(step=_mutant_step_transposed_S),
    "no_scale": Impl(step=_mutant_step_no_scale),
    "dropped_linear": Impl(step=_mutant_step_dropped_linear),
    "wrong_gqa": Impl(step=_mutant_step_wrong_gqa),
    "prefill_no_relu": Impl(prefill=_mutant_prefill_no_relu),
    "commit_sign": Impl(commit=_mutant_commit_sign),
    "prefix_drops_block_scores": Impl(prefix=_mutant_prefix_drops_block),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name):
    """At least one pin fails (by far) on each planted mistake."""
    impl = MUTANTS[name]
    errs = []
    for pin in ALL_PINS:
        try:
            errs.append(pin(impl))
        except Exception:
            errs.append(float("inf"))
    assert max(errs) > 1e-3, (name, errs)


# ------------------------------------------------------- other feature maps
# The method details speak of kernel-function approximations and the future
# work lists better kernels; these pins cover the two extra maps the oracle
# provides: elu(x) + 1 and a learned projection relu(x W) (one W per KV head).

def np_elu1(x):
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def np_relu_proj(x, W):
    return np.maximum(x @ W, 0.0)


def _bruteforce_linear(Q, Kp, Vp, phi):
    """sum over prefix tokens t of (phi(q).phi(k_t)) v_t, token by token."""
    n, hq, b, d = Q.shape
    hkv = Kp.shape[1]
    G = hq // hkv
    out = np.zeros(Q.shape)
    for ni in range(n):
        for h in range(hq):
            g = h // G
            fk = phi(Kp[ni, g], g)
            for i in range(b):
                fq = phi(Q[ni, h, i][None], g)[0]
                for t in range(Kp.shape[2]):
                    out[ni, h, i] += float(fq @ fk[t]) * Vp[ni, g, t]
    return out


def pin_fmap_linear_bruteforce(impl_step, impl_prefill, fmap, W, phi):
    n, hq, hkv, b, d, T = 1, 4, 2, 3, 8, 7
    Q, K, V = rnd(151, (n, hq, b, d)), rnd(152, (n, hkv, b, d)), rnd(153, (n, hkv, b, d))
    Kp, Vp = rnd(154, (n, hkv, T, d)), rnd(155, (n, hkv, T, d))
    S, z = impl_prefill(Kp, Vp, fmap=fmap, W=W)
    y = impl_step(Q, K, V, S, z, fmap=fmap, W=W)
    soft = sdpa(Q, K, V, scale=1.0 / math.sqrt(d))
    return relerr(y - soft, _bruteforce_linear(Q, Kp, Vp, phi))


def test_elu1_linear_term_bruteforce():
    e = pin_fmap_linear_bruteforce(oracle.hybrid_step, oracle.state_prefill,
                                   oracle.FMAP_ELU1, None, lambda x, g: np_elu1(x))
    assert e < TOL


def test_relu_proj_linear_term_bruteforce():
    W = rnd(160, (2, 8, 8), 0.5)
    e = pin_fmap_linear_bruteforce(oracle.hybrid_step, oracle.state_prefill,
                                   oracle.FMAP_RELU_PROJ, W, lambda x, g: np_relu_proj(x, W[g]))
    assert e < TOL


def test_relu_proj_identity_is_relu():
    """W = I: the projected map is ReLU exactly."""
    d = 8
    W = np.broadcast_to(np.eye(d), (2, d, d)).copy()
    Q, K, V = rnd(161, (2, 4, 5, d)), rnd(162, (2, 2, 5, d)), rnd(163, (2, 2, 5, d))
    Kp, Vp = rnd(164, (2, 2, 9, d)), rnd(165, (2, 2, 9, d))
    S1, z1 = oracle.state_prefill(Kp, Vp)
    S2, z2 = oracle.state_prefill(Kp, Vp, fmap=oracle.FMAP_RELU_PROJ, W=W)
    assert np.array_equal(S1, S2) and np.array_equal(z1, z2)
    y1 = oracle.hybrid_step(Q, K, V, S1, z1, shared=True)
    y2 = oracle.hybrid_step(Q, K, V, S2, z2, shared=True, fmap=oracle.FMAP_RELU_PROJ, W=W)
    assert np.array_equal(y1, y2)


def test_relu_proj_permutation_leaves_output_unchanged():
    """W = a permutation P: phi(q) phi(K)^T = relu(q) P P^T relu(K)^T, so the
    linear term (and y) equal the plain ReLU ones while S is permuted."""
    d = 8
    perm = np.random.default_rng(7).permutation(d)
    P = np.eye(d)[:, perm]
    W = np.stack([P, P])
    Q, K, V = rnd(171, (1, 4, 5, d)), rnd(172, (1, 2, 5, d)), rnd(173, (1, 2, 5, d))
    Kp, Vp = rnd(174, (1, 2, 9, d)), rnd(175, (1, 2, 9, d))
    S1, _ = oracle.state_prefill(Kp, Vp)
    S2, _ = oracle.state_prefill(Kp, Vp, fmap=oracle.FMAP_RELU_PROJ, W=W)
    assert relerr(S2, S1[..., perm, :]) < TOL
    y1 = oracle.hybrid_step(Q, K, V, S1)
    y2 = oracle.hybrid_step(Q, K, V, S2, fmap=oracle.FMAP_RELU_PROJ, W=W)
    assert relerr(y2, y1) < TOL


def test_elu1_special_values():
    """phi(0) = e^0 = 1, phi(x) = x + 1 for x > 0, phi(x) in (0, 1) for x < 0:
    one token with k = (0, 2, -1, ...) gives S rows scaled by those values."""
    d = 4
    k = np.array([[[[0.0, 2.0, -1.0, 3.5]]]])
    v = np.array([[[[1.0, -2.0, 0.5, 4.0]]]])
    S, z = oracle.state_prefill(k, v, fmap=oracle.FMAP_ELU1)
    phi = np.array([1.0, 3.0, math.exp(-1.0), 4.5])
    assert np.allclose(S[0, 0], np.outer(phi, v[0, 0, 0]), rtol=0, atol=1e-15)
    assert np.allclose(z[0, 0], phi, rtol=0, atol=1e-15)


def test_fmap_prefill_equals_commits_and_order_invariance():
    d, B = 8, 4
    W = rnd(180, (1, d, d), 0.5)
    Kp, Vp = rnd(181, (2, 1, 3 * B, d)), rnd(182, (2, 1, 3 * B, d))
    for fmap, w in ((oracle.FMAP_ELU1, None), (oracle.FMAP_RELU_PROJ, W)):
        S_all, z_all = oracle.state_prefill(Kp, Vp, fmap=fmap, W=w)
        for order in ([0, 1, 2], [2, 1, 0]):
            S = np.zeros((2, 1, d, d))
            z = np.zeros((2, 1, d))
            for blk in order:
                sl = slice(blk * B, (blk + 1) * B)
                S, z = oracle.state_commit(S, z, Kp[:, :, sl], Vp[:, :, sl], fmap, w)
            assert relerr(S, S_all) < TOL and relerr(z, z_all) < TOL


def test_fmap_pins_catch_planted_mistakes():
    """Transposed projection, and ELU without the +1, fail the brute force."""
    W = rnd(160, (2, 8, 8), 0.5)
    wt = np.swapaxes(W, -1, -2).copy()
    bad_step = lambda Q, K, V, S, z, fmap, W: oracle.hybrid_step(Q, K, V, S, z, fmap=fmap, W=wt)
    e = pin_fmap_linear_bruteforce(bad_step, oracle.state_prefill, oracle.FMAP_RELU_PROJ, W,
                                   lambda x, g: np_relu_proj(x, W[g]))
    assert e > 1e-3
    e2 = pin_fmap_linear_bruteforce(oracle.hybrid_step, oracle.state_prefill,
                                    oracle.FMAP_ELU1, None,
                                    lambda x, g: np_elu1(x) - 1.0)   # elu without +1
    assert e2 > 1e-3


# ------------------------------------------------------------ ragged and paged batches
# Per-request prefix lengths over a paged KV cache (the summary page pairs the
# method with KV-cache management; its related work names PagedAttention) and
# prompts of different lengths.

def _scatter_pages(caches, page_size, num_pages, rng, fill=np.nan):
    """Writes per-request contiguous caches [hkv, P_i, d] into a pool of pages
    at random distinct page numbers; returns (pool, table)."""
    hkv, d = caches[0].shape[0], caches[0].shape[2]
    pool = np.full((num_pages, hkv, page_size, d), fill)
    free = list(rng.permutation(num_pages))
    max_pages = max(1, max((c.shape[1] + page_size - 1) // page_size for c in caches))
    table = np.full((len(caches), max_pages), -1, dtype=np.int64)
    for i, c in enumerate(caches):
        for pg in range((c.shape[1] + page_size - 1) // page_size):
            p = free.pop()
            table[i, pg] = p
            rows = c[:, pg * page_size:(pg + 1) * page_size, :]
            pool[p, :, :rows.shape[1], :] = rows
    return pool, table


def _paged_case(seed, P_lens, page_size, n_extra_pages=5):
    rng = np.random.default_rng(seed)
    n, hq, hkv, b, d = len(P_lens), 4, 2, 5, 16
    Kc = [rng.standard_normal((hkv, P, d)) for P in P_lens]
    Vc = [rng.standard_normal((hkv, P, d)) for P in P_lens]
    pages = sum((P + page_size - 1) // page_size for P in P_lens) + n_extra_pages
    rng2 = np.random.default_rng(seed + 1)
    Kpool, table = _scatter_pages(Kc, page_size, pages, rng2)
    rng2 = np.random.default_rng(seed + 1)      # same page choice for V
    Vpool, table_v = _scatter_pages(Vc, page_size, pages, rng2)
    assert np.array_equal(table, table_v)
    Q = rng.standard_normal((n, hq, b, d))
    K = rng.standard_normal((n, hkv, b, d))
    V = rng.standard_normal((n, hkv, b, d))
    return Q, K, V, Kc, Vc, Kpool, Vpool, table


@pytest.mark.parametrize("page_size", [1, 4, 16])
def test_paged_prefix_equals_sdpa_per_request(page_size):
    """Each request's output equals library softmax attention over its own
    cache followed by its block; unused pool slots hold NaN and must not
    matter."""
    P_lens = [0, 7, 16, 33]
    Q, K, V, Kc, Vc, Kpool, Vpool, table = _paged_case(11, P_lens, page_size)
    Y = oracle.prefix_softmax_paged(Q, Kpool, Vpool, table, P_lens, page_size, K, V)
    assert np.all(np.isfinite(Y))
    for i, P in enumerate(P_lens):
        ref = sdpa(Q[i:i + 1], np.concatenate([Kc[i][None], K[i:i + 1]], axis=2),
                   np.concatenate([Vc[i][None], V[i:i + 1]], axis=2))
        np.testing.assert_allclose(Y[i:i + 1], ref, rtol=1e-12, atol=1e-12)


def test_paged_prefix_page_order_invariance():
    """Renumbering the pool's pages (and the table with them) changes nothing."""
    P_lens = [5, 20, 13]
    Q, K, V, _, _, Kpool, Vpool, table = _paged_case(12, P_lens, 4)
    Y = oracle.prefix_softmax_paged(Q, Kpool, Vpool, table, P_lens, 4, K, V)
    perm = np.random.default_rng(3).permutation(Kpool.shape[0])
    inv = np.argsort(perm)
    table2 = np.where(table >= 0, inv[np.maximum(table, 0)], -1)
    Y2 = oracle.prefix_softmax_paged(Q, Kpool[perm], Vpool[perm], table2, P_lens, 4, K, V)
    assert np.array_equal(Y, Y2)


def test_paged_prefix_page_size_invariance():
    """The same caches laid out in pages of 1, 4 and 16 tokens (each in its own
    random page order) give bit-identical outputs: the result depends on the
    tokens a request sees, not on how its pages cut them."""
    P_lens = [0, 9, 31, 16]
    outs = []
    for ps in (1, 4, 16):
        Q, K, V, _, _, Kpool, Vpool, table = _paged_case(14, P_lens, ps)
        outs.append(oracle.prefix_softmax_paged(Q, Kpool, Vpool, table, P_lens, ps, K, V))
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])


def test_paged_prefix_pins_catch_planted_mistakes():
    """A gather reading the wrong row of a page, or every request through
    request 0's table, fails the per-request SDPA pin."""
    P_lens = [6, 11]
    Q, K, V, Kc, Vc, Kpool, Vpool, table = _paged_case(13, P_lens, 4)

    def check(gather):
        for i, (kc, vc) in enumerate(gather):
            ref = sdpa(Q[i:i + 1], np.concatenate([Kc[i][None], K[i:i + 1]], axis=2),
                       np.concatenate([Vc[i][None], V[i:i + 1]], axis=2))
            got = oracle.prefix_softmax(Q[i:i + 1], kc[None], vc[None], kc.shape[1],
                                        K[i:i + 1], V[i:i + 1])
            if not np.allclose(got, ref, rtol=1e-9, atol=1e-9):
                return False
        return True

    good = oracle.paged_cache(Kpool, Vpool, table, P_lens, 4)
    assert check(good)
    shifted = [(np.stack([Kpool[table[i][t // 4], :, (t + 1) % 4] for t in range(P)], 1),
                np.stack([Vpool[table[i][t // 4], :, (t + 1) % 4] for t in range(P)], 1))
               for i, P in enumerate(P_lens)]
    assert not check(shifted)
    wrong_table = oracle.paged_cache(Kpool, Vpool, [table[0], table[0]], [6, 6], 4)
    assert not check(wrong_table)


def test_ragged_prefill_equals_per_request_numpy():
    """Request i folds exactly its first T_i tokens; padding rows hold NaN."""
    rng = np.random.default_rng(21)
    n, hkv, Tmax, d = 4, 2, 40, 16
    T_lens = [0, 1, 17, 40]
    K = rng.standard_normal((n, hkv, Tmax, d))
    V = rng.standard_normal((n, hkv, Tmax, d))
    for i, T in enumerate(T_lens):
        K[i, :, T:] = np.nan
        V[i, :, T:] = np.nan
    S, z = oracle.state_prefill_ragged(K, V, T_lens)
    for i, T in enumerate(T_lens):
        fk = np.maximum(K[i, :, :T], 0.0)
        np.testing.assert_allclose(S[i], np.einsum("htr,htc->hrc", fk, V[i, :, :T]),
                                   rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(z[i], fk.sum(axis=1), rtol=1e-12, atol=1e-12)
    assert np.all(S[0] == 0) and np.all(z[0] == 0)
