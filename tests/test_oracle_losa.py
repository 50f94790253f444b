"""Pins of the oracle's reuse of prefix attention for stable tokens.

The method is the LoSA page's (gist.science explainer of arXiv 2604.12056,
section "3. 方法论 LoSA": locality pruning by the MSE of each token's query
between consecutive denoising steps, top-k active tokens, reuse of the
previous step's prefix output and log-normaliser for the stable ones, a dense
first step; "技术细节": prefix and block attention merged by online softmax,
b x (d + 1) cached values per head), applied to the exact path with a dense
prefix pass over the active tokens.

Each pin states the fact independently of the oracle's code: the exact path
it must reduce to (itself pinned against torch SDPA), torch SDPA and
``torch.logsumexp`` over the prefix alone, a brute-force joint sum that mixes
the previous step's query (prefix) with this step's (block), and a NumPy sort
of NumPy-computed scores for the selection.  The same pins fail on planted
mistakes (``test_losa_pins_catch_planted_mistakes``).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from block_hybrid_linear_b200 import inputs

TOL = 1e-10


def rnd(seed, shape, std=1.0):
    return inputs.normal_f32_np(seed, 0, shape, std).astype(np.float64)


def sdpa(Q, K, V):
    q = torch.from_numpy(np.asarray(Q, dtype=np.float64))
    k = torch.from_numpy(np.asarray(K, dtype=np.float64))
    v = torch.from_numpy(np.asarray(V, dtype=np.float64))
    G = q.shape[1] // k.shape[1]
    k = k.repeat_interleave(G, dim=1)
    v = v.repeat_interleave(G, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(q, k, v).numpy()


def relerr(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-300))


def case(seed, n=2, hq=4, hkv=2, b=6, d=8, P=9, cap=12):
    Q = rnd(seed, (n, hq, b, d))
    Kc, Vc = rnd(seed + 1, (n, hkv, cap, d)), rnd(seed + 2, (n, hkv, cap, d))
    K, V = rnd(seed + 3, (n, hkv, b, d)), rnd(seed + 4, (n, hkv, b, d))
    return Q, Kc, Vc, P, K, V


def np_scores(Q, Qprev):
    """MSE of each token's query change over every head and dimension."""
    diff = np.asarray(Q, np.float64) - np.asarray(Qprev, np.float64)
    return (diff ** 2).mean(axis=(1, 3))     # [n, b]


def np_topk(score, k):
    """Top k by a stable NumPy sort (ties keep the lower index first)."""
    order = np.argsort(-score, axis=1, kind="stable")
    return np.sort(order[:, :k], axis=1)


# ---- the implementation under test (the oracle, or a planted mistake) ----

class Impl:
    def __init__(self, step=None, select=None):
        self.step = step or oracle.losa_step
        self.select = select or (lambda Q, Qp, k: oracle.losa_select(Q, Qp, k)[0])


def pin_first_step_is_exact(impl):
    """The block's first step is dense: y = exact softmax over [cache || block]."""
    worst = 0.0
    for P in (0, 1, 9):
        Q, Kc, Vc, _, K, V = case(10 + P, P=P)
        Y, _, _, _ = impl.step(Q, None, Kc, Vc, P, K, V)
        worst = max(worst, relerr(Y, sdpa(Q, np.concatenate([Kc[:, :, :P], K], 2),
                                          np.concatenate([Vc[:, :, :P], V], 2))))
    return worst


def pin_all_active_is_exact(impl):
    """k = b at a later step recomputes every token: y = the exact path."""
    Q0, Kc, Vc, P, K, V = case(20)
    Y0, O, L, _ = impl.step(Q0, None, Kc, Vc, P, K, V)
    Q1 = rnd(21, Q0.shape)
    Y1, _, _, _ = impl.step(Q1, Q0, Kc, Vc, P, K, V, O, L, k=Q0.shape[2])
    return relerr(Y1, oracle.prefix_softmax(Q1, Kc, Vc, P, K, V))


def pin_unchanged_queries_reuse_exactly(impl):
    """If a token's query is unchanged, its cached prefix part is exact: after
    a dense step with Q, a step with the same Q and a new block K, V gives the
    exact path for any k -- also after an intermediate step that changed Q
    with every token active (the cache must hold that step's prefix part)."""
    Q0, Kc, Vc, P, K, V = case(30)
    b = Q0.shape[2]
    K2, V2 = rnd(31, K.shape), rnd(32, V.shape)
    worst = 0.0
    for k in (0, 2):
        _, O, L, _ = impl.step(Q0, None, Kc, Vc, P, K, V)
        Y, _, _, _ = impl.step(Q0, Q0, Kc, Vc, P, K2, V2, O, L, k=k)
        worst = max(worst, relerr(Y, oracle.prefix_softmax(Q0, Kc, Vc, P, K2, V2)))
        Q1 = rnd(33, Q0.shape)
        _, O1, L1, _ = impl.step(Q1, Q0, Kc, Vc, P, K, V, O, L, k=b)
        Y, _, _, _ = impl.step(Q1, Q1, Kc, Vc, P, K2, V2, O1, L1, k=k)
        worst = max(worst, relerr(Y, oracle.prefix_softmax(Q1, Kc, Vc, P, K2, V2)))
    return worst


def brute_mixed(q_prefix, q_block, Kc, Vc, P, K, V, scale):
    """One output row as a single joint softmax sum whose prefix scores use
    q_prefix and whose block scores use q_block (no log-sum-exp merge)."""
    s = np.concatenate([scale * Kc[:P] @ q_prefix, scale * K @ q_block])
    w = np.exp(s - s.max())
    return (w[:, None] * np.concatenate([Vc[:P], V])).sum(0) / w.sum()


def pin_stable_tokens_keep_previous_prefix(impl):
    """A stable token's output mixes the previous step's prefix attention with
    this step's block attention; an active token's is the exact path."""
    Q0, Kc, Vc, P, K, V = case(40)
    n, hq, b, d = Q0.shape
    G = hq // Kc.shape[1]
    scale = 1.0 / math.sqrt(d)
    _, O, L, _ = impl.step(Q0, None, Kc, Vc, P, K, V)
    Q1 = Q0 + 0.5 * rnd(41, Q0.shape)
    K1, V1 = rnd(42, K.shape), rnd(43, V.shape)
    worst = 0.0
    for k in (0, 2):
        Y, _, _, act = impl.step(Q1, Q0, Kc, Vc, P, K1, V1, O, L, k=k)
        want = np_topk(np_scores(Q1, Q0), k)
        for ni in range(n):
            for h in range(hq):
                g = h // G
                for i in range(b):
                    q_pre = Q1[ni, h, i] if i in want[ni] else Q0[ni, h, i]
                    ref = brute_mixed(q_pre, Q1[ni, h, i], Kc[ni, g], Vc[ni, g], P, K1[ni, g],
                                      V1[ni, g], scale)
                    worst = max(worst, relerr(Y[ni, h, i], ref))
    return worst


def pin_selection_is_numpy_topk(impl):
    """The active set is the top k of the NumPy MSE, ties to the lower index:
    compared as integers, bit-exact (returned as 0 or inf)."""
    for seed, (n, hq, b, d) in ((50, (3, 4, 9, 8)), (51, (2, 16, 32, 16)), (52, (1, 2, 64, 4))):
        Q, Qp = rnd(seed, (n, hq, b, d)), rnd(seed + 100, (n, hq, b, d))
        # exact ties: tokens 1 and 4 (and 6 where b allows) change identically
        Qp[:, :, 4] = Qp[:, :, 1] + (Q[:, :, 4] - Q[:, :, 1])
        for k in (0, 1, 2, 3, b // 2, b - 1, b, b + 3):
            got = np.asarray(impl.select(Q, Qp, k))
            want = np_topk(np_scores(Q, Qp), min(k, b))
            if got.shape != want.shape or not np.array_equal(got, want):
                return math.inf
    return 0.0


def pin_cache_holds_prefix_attention(impl):
    """Cached entries of an active token: the normalised softmax output over
    the prefix alone (torch SDPA) and its natural-log normaliser
    (torch.logsumexp of the scaled scores); b x (d + 1) values per head."""
    Q, Kc, Vc, P, K, V = case(60)
    n, hq, b, d = Q.shape
    _, O, L, _ = impl.step(Q, None, Kc, Vc, P, K, V)
    if O.shape != (n, hq, b, d) or L.shape != (n, hq, b):
        return math.inf
    err = relerr(O, sdpa(Q, Kc[:, :, :P], Vc[:, :, :P]))
    G = hq // Kc.shape[1]
    qt = torch.from_numpy(Q)
    kt = torch.from_numpy(Kc[:, :, :P]).repeat_interleave(G, dim=1)
    lse = torch.logsumexp(qt @ kt.transpose(-1, -2) / math.sqrt(d), dim=-1).numpy()
    return max(err, relerr(L, lse))


LOSA_PINS = [pin_first_step_is_exact, pin_all_active_is_exact,
             pin_unchanged_queries_reuse_exactly, pin_stable_tokens_keep_previous_prefix,
             pin_selection_is_numpy_topk, pin_cache_holds_prefix_attention]


@pytest.mark.parametrize("pin", LOSA_PINS, ids=lambda p: p.__name__)
def test_losa_pin(pin):
    assert pin(Impl()) <= TOL


def test_losa_empty_prefix_and_single_token_block():
    """P = 0 leaves only the block (y = block softmax, lse cached as -inf);
    b = 1 gives y = v blended with the prefix by the exact path."""
    Q, Kc, Vc, _, K, V = case(70, P=0)
    Y, O, L, _ = oracle.losa_step(Q, None, Kc, Vc, 0, K, V)
    assert relerr(Y, sdpa(Q, K, V)) <= TOL and np.all(np.isneginf(L)) and np.all(O == 0)
    Q1 = rnd(71, Q.shape)
    Y1, _, _, _ = oracle.losa_step(Q1, Q, Kc, Vc, 0, K, V, O, L, k=1)
    assert relerr(Y1, sdpa(Q1, K, V)) <= TOL
    Q, Kc, Vc, P, K, V = case(72, b=1)
    Y, O, L, _ = oracle.losa_step(Q, None, Kc, Vc, P, K, V)
    assert relerr(Y, oracle.prefix_softmax(Q, Kc, Vc, P, K, V)) <= TOL


def test_losa_block_loop_first_step_dense_then_selected():
    """losa_block: step 0 equals the exact path, later steps list k tokens."""
    n, hq, hkv, b, d, P = 2, 4, 2, 8, 8, 11
    Kc, Vc = rnd(80, (n, hkv, P, d)), rnd(81, (n, hkv, P, d))
    Qs = [rnd(82 + t, (n, hq, b, d)) for t in range(3)]
    Ks = [rnd(90 + t, (n, hkv, b, d)) for t in range(3)]
    Vs = [rnd(95 + t, (n, hkv, b, d)) for t in range(3)]
    outs, acts, O, L = oracle.losa_block(Qs, Ks, Vs, Kc, Vc, P, 3)
    assert relerr(outs[0], oracle.prefix_softmax(Qs[0], Kc, Vc, P, Ks[0], Vs[0])) <= TOL
    assert acts[0].shape == (n, b) and acts[1].shape == (n, 3) and acts[2].shape == (n, 3)
    assert np.array_equal(acts[2], np_topk(np_scores(Qs[2], Qs[1]), 3))


# ------------------------------------------------ planted mistakes caught ----

def _mut_least_changed(Q, Qprev, Kc, Vc, P, K, V, O=None, L=None, k=0, scale=0.0):
    if Qprev is None:
        return oracle.losa_step(Q, None, Kc, Vc, P, K, V, O, L, k, scale)
    n, b = Q.shape[0], Q.shape[2]
    act = np.sort(np.argsort(np_scores(Q, Qprev), axis=1, kind="stable")[:, :min(k, b)], 1)
    is_act = np.zeros((n, b), np.int64)
    for ni in range(n):
        is_act[ni, act[ni]] = 1
    return oracle.losa_apply(Q, Kc, Vc, P, K, V, is_act, O, L, scale) + (act,)


def _mut_select_least_changed(Q, Qp, k):
    return np.sort(np.argsort(np_scores(Q, Qp), axis=1, kind="stable")[:, :min(k, Q.shape[2])], 1)


def _mut_recompute_everything(Q, Qprev, Kc, Vc, P, K, V, O=None, L=None, k=0, scale=0.0):
    n, b = Q.shape[0], Q.shape[2]
    Y, O2, L2 = oracle.losa_apply(Q, Kc, Vc, P, K, V, np.ones((n, b), np.int64), O, L, scale)
    return Y, O2, L2, np.tile(np.arange(b), (n, 1))


def _mut_cache_not_updated(Q, Qprev, Kc, Vc, P, K, V, O=None, L=None, k=0, scale=0.0):
    Y, O2, L2, act = oracle.losa_step(Q, Qprev, Kc, Vc, P, K, V, O, L, k, scale)
    return (Y, O2, L2, act) if O is None else (Y, O, L, act)


def _mut_merge_ignores_normalisers(Q, Qprev, Kc, Vc, P, K, V, O=None, L=None, k=0, scale=0.0):
    _, O2, L2, act = oracle.losa_step(Q, Qprev, Kc, Vc, P, K, V, O, L, k, scale)
    ob = oracle.prefix_softmax(Q, Kc, Vc, 0, K, V, scale)     # the block alone
    Y = np.where(np.isneginf(L2)[..., None], ob, 0.5 * (O2 + ob))
    return Y, O2, L2, act


LOSA_MUTANTS = {
    "least_changed_tokens_active": Impl(step=_mut_least_changed, select=_mut_select_least_changed),
    "stable_tokens_recomputed": Impl(step=_mut_recompute_everything),
    "cache_not_updated": Impl(step=_mut_cache_not_updated),
    "merge_ignores_normalisers": Impl(step=_mut_merge_ignores_normalisers),
}


@pytest.mark.parametrize("name", sorted(LOSA_MUTANTS))
def test_losa_pins_catch_planted_mistakes(name):
    impl = LOSA_MUTANTS[name]
    errs = []
    for pin in LOSA_PINS:
        try:
            errs.append(pin(impl))
        except Exception:
            errs.append(math.inf)
    assert max(errs) > 1e-3, (name, errs)
