"""ctypes binding of ``libbha.so`` -- argument marshalling only.

Each ``bha_*`` function here has the name and meaning of the C entry point
declared in ``include/bha.h``: it reads sizes off the tensors' shapes,
passes raw device pointers and the current CUDA stream, and raises
``BhaError`` on a negative status.  All arithmetic runs in the library's
CUDA kernels; there is no fallback.  PyTorch supplies device memory and
streams only.
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbha.so")

BHA_OK = 0
BHA_ERR_INVALID_ARG = -1
BHA_ERR_UNSUPPORTED = -2
BHA_ERR_MISALIGNED = -3
BHA_ERR_WORKSPACE = -4
BHA_ERR_CUDA = -5
BHA_ERR_TIMEOUT = -6
BHA_ERR_DEVICE = -7
BHA_BF16 = 0
BHA_F32 = 1
BHA_FLAG_SHARED_DENOM = 1
BHA_FMAP_RELU = 0
BHA_FMAP_ELU1 = 1
BHA_FMAP_RELU_PROJ = 2

# every symbol include/bha.h declares
EXPORTED = [
    "bha_status_string", "bha_version", "bha_state_prefill_workspace_size",
    "bha_state_prefill", "bha_state_prefill_noalloc", "bha_state_commit", "bha_hybrid_step",
    "bha_hybrid_step_commit", "bha_state_prefill_fm", "bha_state_commit_fm",
    "bha_hybrid_step_fm", "bha_hybrid_step_commit_fm", "bha_prefix_softmax_paged_workspace_size",
    "bha_prefix_softmax_paged", "bha_state_prefill_ragged",
    "bha_prefix_softmax_workspace_size", "bha_prefix_softmax",
    "bha_prefix_softmax_reuse_workspace_size", "bha_prefix_softmax_reuse",
    "bha_block_partition", "bha_device_error", "bha_selftest_timeout",
]

_lib = None


class BhaError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__("%s failed: %s (%d)" % (where, status_string(status), status))


def lib():
    """Load libbha.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                "libbha.so is missing; build it with "
                "`python -m block_hybrid_linear_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, sz, fl, u = (ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t,
                            ctypes.c_float, ctypes.c_uint)
        L.bha_status_string.argtypes = [i]
        L.bha_status_string.restype = ctypes.c_char_p
        L.bha_version.argtypes = []
        L.bha_version.restype = i
        L.bha_state_prefill_workspace_size.argtypes = [i, i, i, i, i]
        L.bha_state_prefill_workspace_size.restype = sz
        L.bha_state_prefill.argtypes = [vp, vp, i, i, i, i, i, vp, vp, vp, sz, vp]
        L.bha_state_prefill.restype = i
        L.bha_state_prefill_noalloc.argtypes = [vp, vp, i, i, i, i, i, vp, vp, vp]
        L.bha_state_prefill_noalloc.restype = i
        L.bha_state_commit.argtypes = [vp, vp, i, i, i, i, i, vp, vp, vp]
        L.bha_state_commit.restype = i
        L.bha_hybrid_step.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, fl, u,
                                      i, vp]
        L.bha_hybrid_step.restype = i
        L.bha_hybrid_step_commit.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, fl, u,
                                             i, vp]
        L.bha_hybrid_step_commit.restype = i
        L.bha_state_prefill_fm.argtypes = [vp, vp, i, i, i, i, i, i, vp, vp, vp, vp, sz, vp]
        L.bha_state_prefill_fm.restype = i
        L.bha_state_commit_fm.argtypes = [vp, vp, i, i, i, i, i, i, vp, vp, vp, vp]
        L.bha_state_commit_fm.restype = i
        L.bha_hybrid_step_fm.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, fl, u, i, i,
                                         vp, vp]
        L.bha_hybrid_step_fm.restype = i
        L.bha_hybrid_step_commit_fm.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, fl, u,
                                                i, i, vp, vp]
        L.bha_hybrid_step_commit_fm.restype = i
        L.bha_prefix_softmax_paged_workspace_size.argtypes = [i, i, i, i, i, i, i, i]
        L.bha_prefix_softmax_paged_workspace_size.restype = sz
        L.bha_prefix_softmax_paged.argtypes = [vp, vp, vp, i, i, vp, i, vp, vp, vp, vp, i, i, i,
                                               i, i, fl, i, vp, sz, vp]
        L.bha_prefix_softmax_paged.restype = i
        L.bha_state_prefill_ragged.argtypes = [vp, vp, vp, i, i, i, i, i, i, vp, vp, vp, vp, sz,
                                               vp]
        L.bha_state_prefill_ragged.restype = i
        L.bha_prefix_softmax_workspace_size.argtypes = [i, i, i, i, i, i, i]
        L.bha_prefix_softmax_workspace_size.restype = sz
        L.bha_prefix_softmax.argtypes = [vp, vp, vp, i, i, vp, vp, vp, i, i, i, i,
                                         i, fl, i, vp, sz, vp]
        L.bha_prefix_softmax.restype = i
        L.bha_prefix_softmax_reuse_workspace_size.argtypes = [i, i, i, i, i, i, i, i]
        L.bha_prefix_softmax_reuse_workspace_size.restype = sz
        L.bha_prefix_softmax_reuse.argtypes = [vp, vp, vp, vp, i, i, vp, vp, vp, vp, vp, vp, i,
                                               i, i, i, i, i, fl, i, vp, sz, vp]
        L.bha_prefix_softmax_reuse.restype = i
        L.bha_block_partition.argtypes = [i, i, ctypes.POINTER(ctypes.c_int), i]
        L.bha_block_partition.restype = i
        L.bha_device_error.argtypes = [i]
        L.bha_device_error.restype = i
        L.bha_selftest_timeout.argtypes = [vp]
        L.bha_selftest_timeout.restype = i
        _lib = L
    return _lib


def status_string(status):
    return lib().bha_status_string(int(status)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    handle = getattr(stream, "cuda_stream", stream)
    return ctypes.c_void_p(int(handle))


def _dtype(t):
    import torch
    if t.dtype == torch.bfloat16:
        return BHA_BF16
    if t.dtype == torch.float32:
        return BHA_F32
    raise TypeError("Q/K/V must be bfloat16 or float32, got %s" % t.dtype)


def _check(status, where):
    if status != BHA_OK:
        raise BhaError(status, where)


def bha_version():
    return lib().bha_version()


def bha_block_partition(L, B):
    """Block boundaries [0, B, 2B, ..., L] of a length-L sequence."""
    k = (L + B - 1) // B if B > 0 and L >= 0 else 0
    buf = (ctypes.c_int * (k + 1))()
    rc = lib().bha_block_partition(int(L), int(B), buf, k + 1)
    if rc < 0:
        raise BhaError(rc, "bha_block_partition")
    return [int(buf[j]) for j in range(rc + 1)]


def bha_device_error(reset=True):
    """Synchronise and return the kernels' device error word (0 = none)."""
    return lib().bha_device_error(1 if reset else 0)


def bha_selftest_timeout(stream=None):
    """Launch the timeout self-test kernel (records BHA_ERR_TIMEOUT)."""
    _check(lib().bha_selftest_timeout(_stream(stream)), "bha_selftest_timeout")


def bha_state_prefill_workspace_size(n, hkv, T, d, dtype=BHA_BF16):
    return lib().bha_state_prefill_workspace_size(n, hkv, T, d, dtype)


def bha_state_prefill(K, V, S, z=None, workspace=None, stream=None):
    """S = phi(K)^T V, z = sum_t phi(k_t) over the prompt.  K, V: [n, hkv, T, d]."""
    n, hkv, T, d = K.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().bha_state_prefill(_ptr(K), _ptr(V), n, hkv, T, d, _dtype(K), _ptr(S),
                                   _ptr(z), _ptr(workspace), ws_bytes, _stream(stream)),
           "bha_state_prefill")


def bha_state_prefill_noalloc(K, V, S, z=None, stream=None):
    """bha_state_prefill with the library's fixed 32 MiB device scratch in
    place of a caller workspace (for callers that cannot allocate)."""
    n, hkv, T, d = K.shape
    _check(lib().bha_state_prefill_noalloc(_ptr(K), _ptr(V), n, hkv, T, d, _dtype(K), _ptr(S),
                                           _ptr(z), _stream(stream)),
           "bha_state_prefill_noalloc")


def bha_state_commit(Kb, Vb, S, z=None, stream=None):
    """S += phi(Kb)^T Vb, z += sum_t phi(kb_t).  Kb, Vb: [n, hkv, b, d]."""
    n, hkv, b, d = Kb.shape
    _check(lib().bha_state_commit(_ptr(Kb), _ptr(Vb), n, hkv, b, d, _dtype(Kb), _ptr(S),
                                  _ptr(z), _stream(stream)), "bha_state_commit")


def bha_hybrid_step(Q, K, V, S, Y, z=None, scale=0.0, flags=0, stream=None):
    """Y = softmax(Q K^T scale) V + phi(Q) S for the active block.

    Q, Y: [n, hq, b, d]; K, V: [n, hkv, b, d]; S: [n, hkv, d, d] fp32."""
    n, hq, b, d = Q.shape
    hkv = K.shape[1]
    _check(lib().bha_hybrid_step(_ptr(Q), _ptr(K), _ptr(V), _ptr(S), _ptr(z), _ptr(Y), n,
                                 hq, hkv, b, d, float(scale), int(flags), _dtype(Q),
                                 _stream(stream)), "bha_hybrid_step")


def bha_hybrid_step_commit(Q, K, V, S, Y, z=None, scale=0.0, flags=0, stream=None):
    """bha_hybrid_step, then S += phi(K)^T V and z += sum phi(k) (in place)."""
    n, hq, b, d = Q.shape
    hkv = K.shape[1]
    _check(lib().bha_hybrid_step_commit(_ptr(Q), _ptr(K), _ptr(V), _ptr(S), _ptr(z), _ptr(Y),
                                        n, hq, hkv, b, d, float(scale), int(flags), _dtype(Q),
                                        _stream(stream)), "bha_hybrid_step_commit")


def bha_state_prefill_fm(K, V, S, z=None, fmap=BHA_FMAP_RELU, W=None, workspace=None,
                         stream=None):
    """bha_state_prefill with feature map ``fmap``; W: [hkv, d, d] in K's dtype
    for BHA_FMAP_RELU_PROJ, else None."""
    n, hkv, T, d = K.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().bha_state_prefill_fm(_ptr(K), _ptr(V), n, hkv, T, d, _dtype(K), int(fmap),
                                      _ptr(W), _ptr(S), _ptr(z), _ptr(workspace), ws_bytes,
                                      _stream(stream)), "bha_state_prefill_fm")


def bha_state_commit_fm(Kb, Vb, S, z=None, fmap=BHA_FMAP_RELU, W=None, stream=None):
    """bha_state_commit with feature map ``fmap`` (W as for bha_state_prefill_fm)."""
    n, hkv, b, d = Kb.shape
    _check(lib().bha_state_commit_fm(_ptr(Kb), _ptr(Vb), n, hkv, b, d, _dtype(Kb), int(fmap),
                                     _ptr(W), _ptr(S), _ptr(z), _stream(stream)),
           "bha_state_commit_fm")


def bha_hybrid_step_fm(Q, K, V, S, Y, z=None, scale=0.0, flags=0, fmap=BHA_FMAP_RELU, W=None,
                       stream=None):
    """bha_hybrid_step with feature map ``fmap`` (W as for bha_state_prefill_fm)."""
    n, hq, b, d = Q.shape
    hkv = K.shape[1]
    _check(lib().bha_hybrid_step_fm(_ptr(Q), _ptr(K), _ptr(V), _ptr(S), _ptr(z), _ptr(Y), n,
                                    hq, hkv, b, d, float(scale), int(flags), _dtype(Q),
                                    int(fmap), _ptr(W), _stream(stream)), "bha_hybrid_step_fm")


def bha_hybrid_step_commit_fm(Q, K, V, S, Y, z=None, scale=0.0, flags=0, fmap=BHA_FMAP_RELU,
                              W=None, stream=None):
    """bha_hybrid_step_commit with feature map ``fmap``."""
    n, hq, b, d = Q.shape
    hkv = K.shape[1]
    _check(lib().bha_hybrid_step_commit_fm(_ptr(Q), _ptr(K), _ptr(V), _ptr(S), _ptr(z),
                                           _ptr(Y), n, hq, hkv, b, d, float(scale), int(flags),
                                           _dtype(Q), int(fmap), _ptr(W), _stream(stream)),
           "bha_hybrid_step_commit_fm")


def bha_prefix_softmax_workspace_size(n, hq, hkv, b, d, P, dtype=BHA_BF16):
    return lib().bha_prefix_softmax_workspace_size(n, hq, hkv, b, d, P, dtype)


def bha_prefix_softmax(Q, Kc, Vc, P, K, V, Y, scale=0.0, workspace=None, stream=None):
    """Exact softmax over [Kc[:, :, :P] || K].  Kc, Vc: [n, hkv, cap, d]."""
    n, hq, b, d = Q.shape
    hkv, cap = Kc.shape[1], Kc.shape[2]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().bha_prefix_softmax(_ptr(Q), _ptr(Kc), _ptr(Vc), int(P), cap, _ptr(K),
                                    _ptr(V), _ptr(Y), n, hq, hkv, b, d, float(scale),
                                    _dtype(Q), _ptr(workspace), ws_bytes, _stream(stream)),
           "bha_prefix_softmax")


def bha_prefix_softmax_reuse_workspace_size(n, hq, hkv, b, d, P, k, dtype=BHA_BF16):
    return lib().bha_prefix_softmax_reuse_workspace_size(n, hq, hkv, b, d, P, k, dtype)


def bha_prefix_softmax_reuse(Q, Qprev, Kc, Vc, P, K, V, Y, O_pre, L_pre, k, active=None,
                             scale=0.0, workspace=None, stream=None):
    """One denoising step of the exact path with reuse for stable tokens.

    Qprev: the previous step's queries, or None for the block's first step
    (every token active).  O_pre [n, hq, b, d] / L_pre [n, hq, b] fp32: the
    reuse cache (read for stable tokens, written for active ones).  active:
    optional [n, k] int32 output of the selected tokens."""
    n, hq, b, d = Q.shape
    hkv, cap = Kc.shape[1], Kc.shape[2]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().bha_prefix_softmax_reuse(_ptr(Q), _ptr(Qprev), _ptr(Kc), _ptr(Vc), int(P), cap,
                                          _ptr(K), _ptr(V), _ptr(Y), _ptr(O_pre), _ptr(L_pre),
                                          _ptr(active), int(k), n, hq, hkv, b, d, float(scale),
                                          _dtype(Q), _ptr(workspace), ws_bytes,
                                          _stream(stream)), "bha_prefix_softmax_reuse")


def bha_prefix_softmax_paged_workspace_size(n, hq, hkv, b, d, max_pages, page_size,
                                            dtype=BHA_BF16):
    return lib().bha_prefix_softmax_paged_workspace_size(n, hq, hkv, b, d, max_pages, page_size,
                                                         dtype)


def bha_prefix_softmax_paged(Q, Kpool, Vpool, block_table, P_lens, K, V, Y, scale=0.0,
                             workspace=None, stream=None):
    """Exact softmax of each request over its own paged cache, then its block.

    Kpool, Vpool: [num_pages, hkv, page_size, d]; block_table: [n, max_pages]
    int32 (device); P_lens: [n] int32 (device)."""
    n, hq, b, d = Q.shape
    num_pages, hkv, page_size, _ = Kpool.shape
    max_pages = block_table.shape[1]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().bha_prefix_softmax_paged(_ptr(Q), _ptr(Kpool), _ptr(Vpool), num_pages,
                                          page_size, _ptr(block_table), max_pages, _ptr(P_lens),
                                          _ptr(K), _ptr(V), _ptr(Y), n, hq, hkv, b, d,
                                          float(scale), _dtype(Q), _ptr(workspace), ws_bytes,
                                          _stream(stream)), "bha_prefix_softmax_paged")


def bha_state_prefill_ragged(K, V, T_lens, S, z=None, fmap=BHA_FMAP_RELU, W=None, workspace=None,
                             stream=None):
    """Prefill of prompts of different lengths: K, V [n, hkv, Tmax, d]; T_lens
    [n] int32 (device)."""
    n, hkv, T, d = K.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().bha_state_prefill_ragged(_ptr(K), _ptr(V), _ptr(T_lens), n, hkv, T, d,
                                          _dtype(K), int(fmap), _ptr(W), _ptr(S), _ptr(z),
                                          _ptr(workspace), ws_bytes, _stream(stream)),
           "bha_state_prefill_ragged")
