"""fp64 CPU oracle for block-hybrid attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg (and its ``--impl reference`` arm) may import this package.  The product
path (``block_hybrid_linear_b200``) never imports it, and this package never
imports the product path: the two share no code.

Method (paper "Retrofitting Linear Attention into Diffusion Language
Models", arXiv 2608.06628; paper-daily summary page, sections "核心公式与算法"
(core formula) and "具体技术细节示例" (worked example); fugumt abstract page):

    y = softmax(Q_a K_a^T * scale) V_a + phi(Q_a) S_p,
    S_p = sum over committed tokens of phi(k)^T v,   phi = ReLU.

Readings where the pages are silent or garbled (each listed in the design
notes): the feature term uses the active block's queries (the worked example
writes phi(Q_2) S_1); the softmax is scaled by 1/sqrt(d); attention inside
the block is bidirectional; the linear term is added unnormalised (weight 1)
unless the shared-denominator option is selected.

Every function takes float arrays (float32 values are widened to float64
exactly), returns float64, and computes the plain definition in
``bha_oracle.c``.  "parity unpinned": the shared-denominator variant is not
on the pages; it is pinned only by its reduction to softmax when S = z = 0
and by a brute-force restatement over prefix tokens.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        lp = ctypes.POINTER(ctypes.c_long)
        L = ctypes.c_long
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_set_threads.restype = ctypes.c_int
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = ctypes.c_int
        lib.oracle_state_prefill.argtypes = [dp, dp, L, L, L, dp, dp, ctypes.c_int, dp, L]
        lib.oracle_state_prefill.restype = None
        lib.oracle_state_commit.argtypes = [dp, dp, dp, dp, L, L, L, ctypes.c_int, dp, L]
        lib.oracle_state_commit.restype = None
        lib.oracle_hybrid_step.argtypes = [dp, dp, dp, dp, dp, dp, L, L, L, L,
                                           L, ctypes.c_double, ctypes.c_int, ctypes.c_int, dp]
        lib.oracle_hybrid_step.restype = None
        lib.oracle_prefix_softmax.argtypes = [dp, dp, dp, L, L, dp, dp, dp, L,
                                              L, L, L, L, ctypes.c_double]
        lib.oracle_prefix_softmax.restype = None
        lib.oracle_losa_select.argtypes = [dp, dp, L, L, L, L, L, lp, dp]
        lib.oracle_losa_select.restype = None
        lib.oracle_losa_apply.argtypes = [dp, dp, dp, L, L, dp, dp, lp, dp, dp, dp,
                                          L, L, L, L, L, ctypes.c_double]
        lib.oracle_losa_apply.restype = None
        lib.oracle_block_partition.argtypes = [L, L, lp]
        lib.oracle_block_partition.restype = L
        _lib = lib
    return _lib


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def set_threads(n: int) -> int:
    """OpenMP threads used by the oracle (parallel over independent units)."""
    return _load().oracle_set_threads(int(n))


def max_threads() -> int:
    return _load().oracle_max_threads()


FMAP_RELU, FMAP_ELU1, FMAP_RELU_PROJ = 0, 1, 2


def _proj(fmap, W, d, hkv=None):
    """(pointer array, number of projections) for the feature map; W must
    hold one d x d projection per KV head of the tensors it is used with."""
    if fmap != FMAP_RELU_PROJ:
        return None, 1
    W = _f64(W)
    assert W.ndim == 3 and W.shape[1:] == (d, d)
    assert hkv is None or W.shape[0] == hkv, "one projection per KV head"
    return W, W.shape[0]


def state_prefill(K, V, with_z=True, fmap=FMAP_RELU, W=None):
    """S = phi(K)^T V and z = sum_t phi(k_t) over a prompt.

    K, V: [..., T, d] (leading dims are independent units, e.g. [n, hkv];
    KV head fastest).  fmap / W: the feature map (W [hkv, d, d] for the
    projected map; unit u uses W[u % hkv]).
    Returns (S [..., d, d], z [..., d] or None).
    """
    K = _f64(K)
    V = _f64(V)
    assert K.shape == V.shape and K.ndim >= 2
    lead, (T, d) = K.shape[:-2], K.shape[-2:]
    units = int(np.prod(lead)) if lead else 1
    S = np.zeros(lead + (d, d))
    z = np.zeros(lead + (d,)) if with_z else None
    Wp, wu = _proj(fmap, W, d, K.shape[-3] if K.ndim >= 3 else 1)
    _load().oracle_state_prefill(_ptr(K), _ptr(V), units, T, d, _ptr(S),
                                 _ptr(z), int(fmap), _ptr(Wp), wu)
    return S, z


def state_commit(S, z, Kb, Vb, fmap=FMAP_RELU, W=None):
    """Return (S + phi(Kb)^T Vb, z + sum_t phi(kb_t)); inputs are not modified.

    S [..., d, d], z [..., d] or None, Kb/Vb [..., b, d]; fmap / W as for
    state_prefill.
    """
    S = _f64(S).copy()
    z = None if z is None else _f64(z).copy()
    Kb = _f64(Kb)
    Vb = _f64(Vb)
    lead, (b, d) = Kb.shape[:-2], Kb.shape[-2:]
    assert S.shape == lead + (d, d)
    units = int(np.prod(lead)) if lead else 1
    Wp, wu = _proj(fmap, W, d, Kb.shape[-3] if Kb.ndim >= 3 else 1)
    _load().oracle_state_commit(_ptr(S), _ptr(z), _ptr(Kb), _ptr(Vb), units,
                                b, d, int(fmap), _ptr(Wp), wu)
    return S, z


def hybrid_step(Q, K, V, S, z=None, scale=0.0, shared=False, fmap=FMAP_RELU,
                W=None):
    """Block-hybrid attention output for the active block.

    Q [n, hq, b, d]; K, V [n, hkv, b, d]; S [n, hkv, d, d]; z [n, hkv, d]
    (required when shared).  scale <= 0 means 1/sqrt(d).  fmap / W: the
    feature map (W [hkv, d, d]; query head h uses KV head h // G's W).
    Returns Y [n, hq, b, d] in float64.
    """
    Q, K, V, S = _f64(Q), _f64(K), _f64(V), _f64(S)
    n, hq, b, d = Q.shape
    hkv = K.shape[1]
    assert K.shape == (n, hkv, b, d) and V.shape == K.shape
    assert S.shape == (n, hkv, d, d) and hq % hkv == 0
    if shared:
        assert z is not None
    zz = None if z is None else _f64(z)
    Y = np.zeros((n, hq, b, d))
    Wp, _ = _proj(fmap, W, d, hkv)
    _load().oracle_hybrid_step(_ptr(Q), _ptr(K), _ptr(V), _ptr(S), _ptr(zz),
                               _ptr(Y), n, hq, hkv, b, d, float(scale),
                               1 if shared else 0, int(fmap), _ptr(Wp))
    return Y


def prefix_softmax(Q, Kc, Vc, P, K, V, scale=0.0):
    """Exact softmax attention of the active block over [cache[:P] || block].

    Q [n, hq, b, d]; Kc, Vc [n, hkv, cap, d] (first P tokens valid);
    K, V [n, hkv, b, d].  Returns Y [n, hq, b, d] in float64.
    """
    Q, Kc, Vc, K, V = _f64(Q), _f64(Kc), _f64(Vc), _f64(K), _f64(V)
    n, hq, b, d = Q.shape
    hkv, cap = Kc.shape[1], Kc.shape[2]
    assert 0 <= P <= cap and Kc.shape == (n, hkv, cap, d)
    Y = np.zeros((n, hq, b, d))
    _load().oracle_prefix_softmax(_ptr(Q), _ptr(Kc), _ptr(Vc), int(P), cap,
                                  _ptr(K), _ptr(V), _ptr(Y), n, hq, hkv, b, d,
                                  float(scale))
    return Y


def paged_cache(Kpool, Vpool, table, P_lens, page_size):
    """The cache each request sees through its page table: token t of
    request i is row t % page_size of page table[i][t // page_size] of the
    pool ([num_pages, hkv, page_size, d]).  Returns per-request lists of
    (Kc [hkv, P_i, d], Vc [hkv, P_i, d]) float64 arrays."""
    Kpool, Vpool = _f64(Kpool), _f64(Vpool)
    out = []
    for i, P in enumerate(P_lens):
        P = int(P)
        pages = [int(table[i][t // page_size]) for t in range(P)]
        rows = [t % page_size for t in range(P)]
        Kc = np.stack([Kpool[p, :, r, :] for p, r in zip(pages, rows)], axis=1) if P else \
            np.zeros((Kpool.shape[1], 0, Kpool.shape[3]))
        Vc = np.stack([Vpool[p, :, r, :] for p, r in zip(pages, rows)], axis=1) if P else \
            np.zeros((Vpool.shape[1], 0, Vpool.shape[3]))
        out.append((Kc, Vc))
    return out


def prefix_softmax_paged(Q, Kpool, Vpool, table, P_lens, page_size, K, V, scale=0.0):
    """Exact softmax attention of each request's active block over its own
    cache (its first P_lens[i] tokens, read through its page table) followed
    by the block.  Q [n, hq, b, d]; K, V [n, hkv, b, d].  Returns Y float64."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    Y = np.zeros(Q.shape)
    for i, (Kc, Vc) in enumerate(paged_cache(Kpool, Vpool, table, P_lens, page_size)):
        P = Kc.shape[1]
        Y[i:i + 1] = prefix_softmax(Q[i:i + 1], Kc[None], Vc[None], P, K[i:i + 1], V[i:i + 1],
                                    scale)
    return Y


def state_prefill_ragged(K, V, T_lens, with_z=True, fmap=FMAP_RELU, W=None):
    """Prefill of prompts of different lengths: request i folds its first
    T_lens[i] tokens of K, V ([n, hkv, Tmax, d]; rows past T_lens[i] are
    padding and ignored).  Returns (S [n, hkv, d, d], z [n, hkv, d] or None)."""
    K, V = _f64(K), _f64(V)
    n, hkv, _, d = K.shape
    S = np.zeros((n, hkv, d, d))
    z = np.zeros((n, hkv, d)) if with_z else None
    for i, T in enumerate(T_lens):
        T = int(T)
        Si, zi = state_prefill(K[i:i + 1, :, :T], V[i:i + 1, :, :T], with_z, fmap, W)
        S[i] = Si[0]
        if with_z:
            z[i] = zi[0]
    return S, z


def losa_select(Q, Qprev, k):
    """Locality scores and active tokens (LoSA page, 3. 方法论: 局部性剪枝).

    Q, Qprev [n, hq, b, d]: the block's queries at this and at the previous
    denoising step.  score[ni, i] is the MSE of token i's query change over
    all query heads and dimensions; the k tokens with the largest score (ties
    to the lower index) are active.  Returns (active [n, min(k, b)] int64,
    increasing token order; score [n, b] float64).
    """
    Q, Qprev = _f64(Q), _f64(Qprev)
    n, hq, b, d = Q.shape
    assert Qprev.shape == Q.shape
    k = max(0, min(int(k), b))
    active = np.zeros((n, max(k, 1)), dtype=np.int64)
    score = np.zeros((n, b))
    _load().oracle_losa_select(_ptr(Q), _ptr(Qprev), n, hq, b, d, k,
                               active.ctypes.data_as(ctypes.POINTER(ctypes.c_long)),
                               _ptr(score))
    return active[:, :k], score


def losa_apply(Q, Kc, Vc, P, K, V, is_active, O_pre, L_pre, scale=0.0):
    """Cache reuse and merge for a given active set (LoSA page, 缓存复用 and
    技术细节): active tokens get a dense prefix pass with this step's queries
    (their entries of the cache are replaced), stable tokens keep their cached
    prefix output and log-normaliser, and every token's block attention is
    merged with its prefix part by the online-softmax identity.

    is_active [n, b] (nonzero = active); O_pre [n, hq, b, d], L_pre [n, hq, b]
    (natural-log normalisers; may be None when every token is active).
    Returns (Y, O_pre, L_pre) as new float64 arrays.
    """
    Q, Kc, Vc, K, V = _f64(Q), _f64(Kc), _f64(Vc), _f64(K), _f64(V)
    n, hq, b, d = Q.shape
    hkv, cap = Kc.shape[1], Kc.shape[2]
    assert 0 <= P <= cap and Kc.shape == (n, hkv, cap, d) and hq % hkv == 0
    act = np.ascontiguousarray(np.asarray(is_active).reshape(n, b) != 0, dtype=np.int64)
    if O_pre is None:
        assert act.all(), "a cache is needed unless every token is active"
        O = np.zeros((n, hq, b, d))
        Lp = np.full((n, hq, b), -np.inf)
    else:
        O = _f64(O_pre).copy()
        Lp = _f64(L_pre).copy()
    Y = np.zeros((n, hq, b, d))
    _load().oracle_losa_apply(_ptr(Q), _ptr(Kc), _ptr(Vc), int(P), cap, _ptr(K), _ptr(V),
                              act.ctypes.data_as(ctypes.POINTER(ctypes.c_long)), _ptr(O),
                              _ptr(Lp), _ptr(Y), n, hq, hkv, b, d, float(scale))
    return Y, O, Lp


def losa_step(Q, Qprev, Kc, Vc, P, K, V, O_pre=None, L_pre=None, k=0, scale=0.0):
    """One denoising step of the exact path with reuse for stable tokens.

    Qprev None: the block's first step, dense (every token active, the LoSA
    page's 初始化策略).  Otherwise the k tokens whose queries changed most
    since Qprev are active.  Returns (Y, O_pre, L_pre, active [n, k'])."""
    n, hq, b, d = np.shape(Q)
    if Qprev is None:
        active = np.tile(np.arange(b, dtype=np.int64), (n, 1))
    else:
        active, _ = losa_select(Q, Qprev, k)
    is_active = np.zeros((n, b), dtype=np.int64)
    for ni in range(n):
        is_active[ni, active[ni]] = 1
    Y, O, Lp = losa_apply(Q, Kc, Vc, P, K, V, is_active, O_pre, L_pre, scale)
    return Y, O, Lp, active


def losa_block(Q_steps, K_steps, V_steps, Kc, Vc, P, k, scale=0.0):
    """The denoising steps of one block with reuse: the first step dense, each
    later step with the k most-changed tokens active.  Returns the outputs,
    the active sets of every step and the final cache (O_pre, L_pre)."""
    O = Lp = None
    outs, acts = [], []
    for t in range(len(Q_steps)):
        Y, O, Lp, act = losa_step(Q_steps[t], None if t == 0 else Q_steps[t - 1], Kc, Vc, P,
                                  K_steps[t], V_steps[t], O, Lp, k, scale)
        outs.append(Y)
        acts.append(act)
    return outs, acts, O, Lp


def block_partition(L: int, B: int):
    """Block boundaries [0, B, 2B, ..., L] (last block may be short)."""
    k_max = (L + B - 1) // B if B > 0 else 0
    out = (ctypes.c_long * (k_max + 2))()
    k = _load().oracle_block_partition(int(L), int(B), out)
    if k < 0:
        raise ValueError("bad block partition arguments")
    return [int(out[i]) for i in range(k + 1)]


def generate(Q_steps, K_steps, V_steps, K_prompt=None, V_prompt=None,
             scale=0.0, shared=False, fmap=FMAP_RELU, W=None, S0=None, z0=None):
    """Blockwise decoding loop of the worked example, on given inputs.

    Q_steps[blk][step] etc. hold the active block's tensors at each
    denoising step ([n, hq, b_blk, d] / [n, hkv, b_blk, d]).  The prompt
    (optional) is folded into S first -- or the state the prompt left
    (S0, z0, e.g. from state_prefill run piecewise) is given instead; every
    block's outputs use the state of all earlier blocks, and after its last
    step the block is committed with the K/V of that step.  Returns
    outputs[blk][step] and the final S, z.
    """
    first_k = K_steps[0][0]
    n, hkv, _, dd = first_k.shape
    if K_prompt is not None:
        assert S0 is None and z0 is None
        S, z = state_prefill(K_prompt, V_prompt, fmap=fmap, W=W)
    elif S0 is not None:
        S = _f64(S0)
        z = _f64(z0) if z0 is not None else np.zeros((n, hkv, dd))
    else:
        S = np.zeros((n, hkv, dd, dd))
        z = np.zeros((n, hkv, dd))
    outs = []
    for blk in range(len(Q_steps)):
        ob = []
        for st in range(len(Q_steps[blk])):
            ob.append(hybrid_step(Q_steps[blk][st], K_steps[blk][st],
                                  V_steps[blk][st], S, z, scale, shared, fmap, W))
        outs.append(ob)
        S, z = state_commit(S, z, K_steps[blk][-1], V_steps[blk][-1], fmap, W)
    return outs, S, z
