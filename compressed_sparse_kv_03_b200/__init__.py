"""B200-native (sm_100a) CSA / HCA hot path: block compression, lightning
indexer + top-k, and sparse / dense shared-KV attention with a sliding window.

The computation runs in the CUDA library ``_csa_b200.so`` (C ABI:
include/csa.h); this package is its thin Python binding.
"""
from ._lib import (CsaError, KERNEL_ATTENTION, KERNEL_COMPRESS, KERNEL_INDEXER_SCORE,  # noqa: F401
                   KERNEL_MERGE, KERNEL_QUANTIZE, KERNEL_TOPK_SAMPLE, KERNEL_TOPK_SELECT,
                   load)
from .api import (AppendState, Cache, QRope, Workspace, cache_append, compress_kv, hca_attn,  # noqa: F401
                  indexer_topk, indexer_topk_mxfp4, launch_count, norm_rope, quantize_entries_fp8,
                  quantize_mxfp4, set_attention_kernel, set_batch_invariant, set_timing_events,
                  sparse_attn_decode, sparse_attn_decode_fp8, sparse_attn_prefill,
                  test_attention_timeout)

__all__ = ["Cache", "QRope", "Workspace", "CsaError", "compress_kv", "cache_append", "AppendState", "norm_rope",
           "indexer_topk", "quantize_mxfp4", "indexer_topk_mxfp4", "quantize_entries_fp8",
           "sparse_attn_decode_fp8", "sparse_attn_prefill", "sparse_attn_decode", "hca_attn", "launch_count",
           "set_attention_kernel", "set_batch_invariant", "set_timing_events", "test_attention_timeout",
           "load"]
