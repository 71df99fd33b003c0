"""Paged sparse-KV attention for B200 (sm_100a).

The computation lives in ``libsa.so`` (C ABI, ``include/sa.h``); this package
is its thin Python binding plus the seeded workload generators the tests and
benchmark share.  Build the library with ``python -m paged_sparse_kv_sa_b200.build``.
"""
from ._lib import (EXPORTED, LIB_PATH, SAError, bind, load, page_budget, sa_block_union,  # noqa: F401
                   sa_build_page_summaries, sa_combine, sa_select_pages,
                   sa_select_pages_no_alloc, sa_select_pages_tiered,
                   sa_select_workspace_size, sa_update_page_summaries,
                   sa_sparse_decode, sa_sparse_decode_fp8, sa_build_page_summaries_fp8,
                   sa_sparse_attention, sa_sparse_attention_fp8, attention_workspace,
                   sa_sparse_step, sa_sparse_step_workspace_size, sa_append_kv,
                   sa_sparse_step_fp8,
                   sa_select_ambient_heads, sa_sparse_decode_at, sa_sparse_attention_at,
                   sa_build_page_summaries_dir, sa_sparse_step_dir, sa_append_kv_dir,
                   dir_capacity)
from .pipeline import SparseDecodeStep, default_splits  # noqa: F401
