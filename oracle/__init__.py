"""Plain fp64 CPU oracle for the CSA / HCA hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the package
``compressed_sparse_kv_03_b200``) imports, calls or links this package.  Only
``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may use it.  It shares no code, table or helper with the CUDA
path; both sides only receive the same seeded inputs from ``synth``.

Every function is written from the DeepSeek-V4 book pages (slop-6tp.pages.dev,
"papers-html-argon/dsv4") and cites the chapter and section it follows.
"""
from .csa_oracle import (  # noqa: F401
    bf16_round,
    page_rows,
    unpage,
    pool_block,
    pool_overlap,
    DecodeCacheState,
    rmsnorm,
    rope_rotate,
    eligible_entries,
    indexer_scores,
    topk_select,
    attend_shared_kv,
    prefill_window_rows,
    csa_prefill,
    csa_prefill_attention,
    csa_prefill_topk,
    csa_decode,
    hca_decode,
    hca_prefill,
)
from . import cost_model  # noqa: F401
from . import mxfp4  # noqa: F401
from . import fp8_entry  # noqa: F401
