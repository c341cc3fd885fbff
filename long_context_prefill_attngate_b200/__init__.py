"""B200-native SeerAttention prefill hot path.

AttnGate soft scores -> threshold / per-row TopK block mask -> block-sparse
causal FlashAttention prefill (GQA), plus the Figure-8 pass returning O and
the max-pooled attention map A, and the decode step (gate without query
pooling, mask row, sparse attention of the new token over its KV cache).  The work runs in libseer.so (hand-written
CUDA for sm_100a, C ABI in include/seer.h); this package only marshals
arguments.  Importing it does not load the library; the first call does, and
fails loudly if it has not been built.
"""
from ._binding import (  # noqa: F401
    BLOCK, EXPORTS, SEER_CALL_ATTN_POOLED_MAP, SEER_CALL_BLOCK_SPARSE_DECODE, SEER_CALL_BLOCK_SPARSE_PREFILL,
    SEER_CALL_DECODE_GATE_CACHED, SEER_CALL_DECODE_GATE_SCORES, SEER_CALL_GATE_KEY_CACHE, SEER_CALL_GATE_SCORES, SEER_ERR_CUDA, SEER_ERR_DEVICE, SEER_ERR_INVALID_ARG,
    SEER_ERR_TIMEOUT, SEER_ERR_UNSUPPORTED, SEER_ERR_WORKSPACE, SEER_KPOOL_AVG, SEER_KPOOL_MAXMIN,
    SEER_MASK_THRESHOLD, SEER_MASK_TOPK, SEER_OK, SeerError, lib, seer_attn_pooled_map, seer_block_mask,
    seer_block_sparse_decode, seer_block_sparse_prefill, seer_check_status, seer_compact_mask,
    seer_decode_block_mask, seer_decode_gate_scores, seer_decode_gate_scores_cached, seer_distill_loss,
    seer_gate_key_cache, seer_gate_params, seer_gate_scores,
    seer_gate_scores_noalloc, seer_last_error, seer_mask_params, seer_set_wait_timeout_ns, seer_shape,
    seer_topk_from_density, seer_version, seer_workspace_bytes, shape_of,
)

from .pipeline import HostPrefill  # noqa: F401,E402

__version__ = "0.1.0"
