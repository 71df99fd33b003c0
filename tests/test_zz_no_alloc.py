"""sa_select_pages_no_alloc against the oracle and against sa_select_pages
(marked gpu).

The no-allocation entry point exists for callers that cannot allocate device
memory where they select pages (inside a CUDA-graph capture, behind a sealed
memory pool, or in a host framework that only passes raw pointers).  It keeps
its score bounds in the library's own static device array instead of a
caller-provided workspace.  Selections are integers: they must equal the
oracle's bit for bit (a ragged case generated on the CPU, summaries from the
oracle), and both entry points must agree exactly at larger shapes; two calls
in a row check that the shared array left over from the first call does not
leak into the second.  This file sorts last so that a
run stopping at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import paged_sparse_kv_sa_b200 as sa
from paged_sparse_kv_sa_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _case(cfg, seed):
    inp = W.gqa_decode_inputs(cfg, seed=seed, device="cuda")
    sig = sa.sa_build_page_summaries(inp["k"], inp["page_table"], inp["seq_lens"])
    return inp, sig


def _no_alloc_via_abi(inp, sig, cfg, pages, counts):
    lib = sa.load()
    q = inp["q"]
    B, T, Hq, Dk = q.shape
    st = lib.sa_select_pages_no_alloc(
        ctypes.c_void_p(q.data_ptr()), (ctypes.c_int64 * 4)(*q.stride()),
        ctypes.c_void_p(sig.data_ptr()), ctypes.c_void_p(inp["page_table"].data_ptr()),
        ctypes.c_void_p(inp["seq_lens"].data_ptr()), B, T, Hq, cfg.Hkv, Dk, cfg.page_size,
        inp["page_table"].shape[1], sig.shape[0], cfg.sink_tokens, cfg.local_tokens,
        cfg.budget_tokens, ctypes.c_void_p(pages.data_ptr()), ctypes.c_void_p(counts.data_ptr()),
        None, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, lib.sa_status_string(st)


def test_no_alloc_selection_matches_workspace_selection_twice():
    cfgs = [W.scaled(W.LLAMA8B_DECODE, B=4), W.scaled(W.LLAMA70B_LONG, B=2, seq_len_lo=40000,
                                                       seq_len_hi=70000)]
    for i, cfg in enumerate(cfgs):            # two calls in a row, different shapes and data
        inp, sig = _case(cfg, seed=11 + i)
        bp = cfg.budget_tokens // cfg.page_size
        pages = torch.full((cfg.B, cfg.Hkv, bp), -7, dtype=torch.int32, device="cuda")
        counts = torch.full((cfg.B, cfg.Hkv), -7, dtype=torch.int32, device="cuda")
        _no_alloc_via_abi(inp, sig, cfg, pages, counts)
        ref_p, ref_c = sa.sa_select_pages(inp["q"], sig, inp["page_table"], inp["seq_lens"],
                                          cfg.page_size, cfg.sink_tokens, cfg.local_tokens,
                                          cfg.budget_tokens)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(counts.cpu().numpy(), ref_c.cpu().numpy())
        np.testing.assert_array_equal(pages.cpu().numpy(), ref_p.cpu().numpy())


def test_no_alloc_selection_matches_oracle():
    cfg = W.scaled(W.LLAMA8B_DECODE, B=4, Hq=16, Hkv=4, seq_len_lo=0, seq_len_hi=0)
    lens = [5000, 1100, 17, 2048]
    inp = W.gqa_decode_inputs(cfg, seed=21, device="cpu", seq_lens=lens)
    kb = W.bf16_bits(inp["k"])
    pt, sl = inp["page_table"].numpy(), inp["seq_lens"].numpy()
    sig_b = O.page_summaries(kb, pt, sl, cfg.page_size)
    g = {k: (v.to("cuda") if torch.is_tensor(v) else v) for k, v in inp.items()}
    g["k"] = None
    sig = torch.from_numpy(sig_b.view(np.int16)).view(torch.bfloat16).to("cuda")
    bp = cfg.budget_tokens // cfg.page_size
    pages = torch.full((cfg.B, cfg.Hkv, bp), -7, dtype=torch.int32, device="cuda")
    counts = torch.full((cfg.B, cfg.Hkv), -7, dtype=torch.int32, device="cuda")
    _no_alloc_via_abi(g, sig, cfg, pages, counts)
    torch.cuda.synchronize()
    rp, rc = O.select_pages(W.bf16_bits(inp["q"]), sig_b, pt, sl, cfg.page_size, cfg.sink_tokens,
                            cfg.local_tokens, cfg.budget_tokens)
    np.testing.assert_array_equal(counts.cpu().numpy(), rc)
    np.testing.assert_array_equal(pages.cpu().numpy(), rp)


def test_no_alloc_rejects_sizes_beyond_the_static_array():
    lib = sa.load()
    fake = ctypes.c_void_p(0x1000)
    s = (ctypes.c_int64 * 4)(1024, 1024, 128, 1)
    # 64 x 8 x 16384 pages > 2,097,152 entries: refused before any launch
    assert lib.sa_select_pages_no_alloc(fake, s, fake, fake, fake, 64, 1, 32, 8, 128, 16, 16384,
                                        16384, 32, 512, 1024, fake, fake, None, None) == 2
