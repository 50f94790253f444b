"""block_hybrid_linear_b200 -- block-hybrid attention for blockwise
semi-autoregressive diffusion-LM decoding, on NVIDIA B200 (sm_100a).

Exact softmax inside the active denoising block plus ReLU-feature linear
attention over all previous blocks through a per-KV-head fp32 prefix state
("Retrofitting Linear Attention into Diffusion Language Models").  The
compute lives in ``libbha.so`` (C ABI, ``include/bha.h``); this package is
its binding (``_lib``) plus the seeded input generators (``inputs``).
"""
from ._lib import (  # noqa: F401
    BHA_BF16, BHA_ERR_CUDA, BHA_ERR_DEVICE, BHA_ERR_INVALID_ARG,
    BHA_ERR_MISALIGNED, BHA_ERR_TIMEOUT, BHA_ERR_UNSUPPORTED, BHA_ERR_WORKSPACE,
    BHA_F32, BHA_FLAG_SHARED_DENOM, BHA_FMAP_ELU1, BHA_FMAP_RELU, BHA_FMAP_RELU_PROJ, BHA_OK,
    BhaError, EXPORTED, LIB_PATH,
    bha_block_partition, bha_device_error, bha_hybrid_step, bha_hybrid_step_commit,
    bha_hybrid_step_commit_fm, bha_hybrid_step_fm, bha_state_commit_fm, bha_state_prefill_fm,
    bha_prefix_softmax, bha_prefix_softmax_paged, bha_prefix_softmax_paged_workspace_size,
    bha_prefix_softmax_workspace_size, bha_prefix_softmax_reuse,
    bha_prefix_softmax_reuse_workspace_size, bha_state_prefill_ragged, bha_selftest_timeout, bha_state_commit,
    bha_state_prefill,
    bha_state_prefill_noalloc, bha_state_prefill_workspace_size, bha_version, lib,
    status_string,
)
