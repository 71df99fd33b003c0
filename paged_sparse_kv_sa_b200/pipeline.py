"""One sparse-attention decode step (select -> decode -> combine; or select ->
attend, which is decode + combine in one call) over preallocated buffers, so
that a timed or graph-captured step allocates nothing.

Every stage is a call through the C ABI; this module only sizes buffers and
chooses the split count.
"""
from __future__ import annotations

import math

import torch

from . import _lib


def default_splits(n_units: int, max_list: int, sm_count: int = None, warps_per_sm: int = 12,
                   max_entries: int = 128) -> int:
    """Split count for ``n_units`` (sequence, list) pairs of up to ``max_list`` pages.

    The decode kernel runs one split per warp and keeps one wave of warps
    resident (twelve per SM: three CTAs of four), striding over the flattened
    (split, pair, sequence) items; take as many splits as fill that wave, and at
    least enough that no split holds more than ``max_entries`` pages."""
    if n_units <= 0 or max_list <= 0:
        return 1
    if sm_count is None:
        sm_count = (torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
                    if torch.cuda.is_available() else 148)
    n = max(1, (warps_per_sm * sm_count) // n_units)
    n = min(n, max(1, max_list))
    while -(-max_list // n) > max_entries:
        n += 1
    return max(1, min(n, 64))


class SparseDecodeStep:
    """GQA sparse decode: per (sequence, kv head) page selection, then attention of
    every head over its group's list, then the split merge.

    Inputs live on the GPU (q, caches, page table, seq_lens, summaries); outputs are
    ``self.o`` [B,T,Hq,D] float32 and ``self.lse`` [B,T,Hq].
    """

    def __init__(self, B: int, T: int, Hq: int, Hkv: int, D: int, page_size: int, max_pages: int,
                 sink_tokens: int, local_tokens: int, budget_tokens: int, scale: float = None,
                 n_splits: int = None, device="cuda", out_bf16: bool = False):
        self.B, self.T, self.Hq, self.Hkv, self.D = B, T, Hq, Hkv, D
        self.P = page_size
        self.sink, self.local, self.budget = sink_tokens, local_tokens, budget_tokens
        _, _, self.budget_pages, _ = _lib.page_budget(sink_tokens, local_tokens, budget_tokens,
                                                      page_size)
        self.scale = 1.0 / math.sqrt(D) if scale is None else scale
        self.n_splits = (default_splits(B * Hkv, self.budget_pages) if n_splits is None
                         else n_splits)
        self.head_to_list = [h // (Hq // Hkv) for h in range(Hq)]
        dev = torch.device(device)
        self.pages = torch.empty((B, Hkv, self.budget_pages), dtype=torch.int32, device=dev)
        self.counts = torch.empty((B, Hkv), dtype=torch.int32, device=dev)
        self.o_part = torch.empty((self.n_splits, B, T, Hq, D), dtype=torch.float32, device=dev)
        self.lse_part = torch.empty((self.n_splits, B, T, Hq), dtype=torch.float32, device=dev)
        self.o = torch.empty((B, T, Hq, D), dtype=torch.float32, device=dev)
        self.o_bf16 = (torch.empty((B, T, Hq, D), dtype=torch.bfloat16, device=dev)
                       if out_bf16 else None)
        self.lse = torch.empty((B, T, Hq), dtype=torch.float32, device=dev)
        self.dev_error = torch.zeros((1,), dtype=torch.int32, device=dev)
        self.sel_ws = torch.empty(max(_lib.sa_select_workspace_size(B, Hkv, max_pages), 16),
                                  dtype=torch.uint8, device=dev)
        # the split partials of sa_sparse_attention
        self.attn_ws = _lib.attention_workspace(B, T, Hq, D, self.n_splits, dev)
        # score bounds + split partials of the one-call step (sa_sparse_step)
        self.step_ws = torch.empty(max(_lib.sa_sparse_step_workspace_size(
            B, T, Hq, Hkv, D, page_size, max_pages, budget_tokens, self.n_splits), 16),
            dtype=torch.uint8, device=dev)

    def select(self, q, summaries, page_table, seq_lens, stream=None):
        _lib.sa_select_pages(q, summaries, page_table, seq_lens, self.P, self.sink, self.local,
                             self.budget, out_pages=self.pages, out_counts=self.counts,
                             workspace=self.sel_ws, dev_error=self.dev_error, stream=stream)

    def decode(self, q, k_cache, v_cache, page_table, seq_lens, stream=None):
        _lib.sa_sparse_decode(q, k_cache, v_cache, page_table, seq_lens, self.pages, self.counts,
                              self.head_to_list, self.scale, self.n_splits,
                              o_partial=self.o_part, lse_partial=self.lse_part,
                              dev_error=self.dev_error, stream=stream)

    def decode_fp8(self, q, k_codes, v_codes, k_scale, v_scale, page_table, seq_lens,
                   stream=None):
        """decode over FP8 E4M3 pages with per-(page, kv head) scales (D == 128)."""
        _lib.sa_sparse_decode_fp8(q, k_codes, v_codes, k_scale, v_scale, page_table, seq_lens,
                                  self.pages, self.counts, self.head_to_list, self.scale,
                                  self.n_splits, o_partial=self.o_part, lse_partial=self.lse_part,
                                  dev_error=self.dev_error, stream=stream)

    def attend(self, q, k_cache, v_cache, page_table, seq_lens, stream=None):
        """decode + combine in one call (sa_sparse_attention) into self.o / self.lse."""
        _lib.sa_sparse_attention(q, k_cache, v_cache, page_table, seq_lens, self.pages,
                                 self.counts, self.head_to_list, self.scale, self.n_splits,
                                 o_out=self.o, o_out_bf16=self.o_bf16, lse_out=self.lse,
                                 workspace=self.attn_ws, dev_error=self.dev_error, stream=stream)

    def attend_fp8(self, q, k_codes, v_codes, k_scale, v_scale, page_table, seq_lens,
                   stream=None):
        """attend over FP8 E4M3 pages (sa_sparse_attention_fp8)."""
        _lib.sa_sparse_attention_fp8(q, k_codes, v_codes, k_scale, v_scale, page_table, seq_lens,
                                     self.pages, self.counts, self.head_to_list, self.scale,
                                     self.n_splits, o_out=self.o, o_out_bf16=self.o_bf16,
                                     lse_out=self.lse, workspace=self.attn_ws,
                                     dev_error=self.dev_error, stream=stream)

    def combine(self, stream=None):
        _lib.sa_combine(self.o_part, self.lse_part, o_out=self.o, o_out_bf16=self.o_bf16,
                        lse_out=self.lse, stream=stream)

    def run(self, q, k_cache, v_cache, summaries, page_table, seq_lens, stream=None):
        """select + decode + merge as one C call (sa_sparse_step) into self.pages,
        self.counts, self.o / self.o_bf16 and self.lse."""
        _lib.sa_sparse_step(q, summaries, k_cache, v_cache, page_table, seq_lens, self.P,
                            self.sink, self.local, self.budget, self.scale, self.n_splits,
                            out_pages=self.pages, out_counts=self.counts, o_out=self.o,
                            o_out_bf16=self.o_bf16, lse_out=self.lse, workspace=self.step_ws,
                            dev_error=self.dev_error, stream=stream)

    def run_fp8(self, q, k_codes, v_codes, k_scale, v_scale, summaries, page_table, seq_lens,
                stream=None):
        """run over FP8 E4M3 pages with per-(page, kv head) scales, as one C call
        (sa_sparse_step_fp8)."""
        _lib.sa_sparse_step_fp8(q, summaries, k_codes, v_codes, k_scale, v_scale, page_table,
                                seq_lens, self.P, self.sink, self.local, self.budget, self.scale,
                                self.n_splits, out_pages=self.pages, out_counts=self.counts,
                                o_out=self.o, o_out_bf16=self.o_bf16, lse_out=self.lse,
                                workspace=self.step_ws, dev_error=self.dev_error, stream=stream)

    def bind(self, q, k_cache, v_cache, summaries, page_table, seq_lens, stream=None):
        """A zero-argument callable that runs `run` on these tensors: the arguments
        are checked and marshalled once (_lib.bind; the tensors must stay where
        they are)."""
        return _lib.bind(lambda: self.run(q, k_cache, v_cache, summaries, page_table, seq_lens,
                                          stream))

    def __call__(self, q, k_cache, v_cache, summaries, page_table, seq_lens, stream=None):
        self.run(q, k_cache, v_cache, summaries, page_table, seq_lens, stream)
        return self.o, self.lse
