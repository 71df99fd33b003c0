"""Explicit query positions (sa_sparse_decode_at / sa_sparse_attention_at)
against the oracle (marked gpu).

A prompt chunk computed while the cache already holds tokens past it: query
token t of sequence b sits at q_pos[b] + t, not at the end of the sequence.
Every decode kernel takes the positions: the per-split warp-MMA kernel (through
sa_sparse_decode_at, and merged through sa_sparse_attention_at), the tcgen05
many-row kernel (sa_sparse_attention_at with T x heads rows of 96 x 4) and the
MLA kernel.  Positions inside the sequence, past its end (every key
visible) and before its start (no key visible: O = 0, LSE = -inf).
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import paged_sparse_kv_sa_b200 as sa
from paged_sparse_kv_sa_b200 import workloads as W
from test_gpu_parity import (DEV, assert_attn_close, bits, gqa_case, mla_lists_from_oracle,
                             np_i32, oracle_lists, oracle_summaries)

pytestmark = pytest.mark.gpu


def _positions(lens, T):
    # inside, inside near the start, past the end, and partly before the start
    pick = [lens[0] // 2, 40, lens[2] + 3, -(T // 2)]
    return np.array(pick[:len(lens)], dtype=np.int32)


@pytest.mark.parametrize("T,path", [(2, "split"), (2, "merged"), (96, "many_rows")])
def test_positions_gqa(T, path):
    P = 16
    cfg = W.GQADecode("case", B=4, Hq=8, Hkv=2, D=128, page_size=P, seq_len_lo=0, seq_len_hi=0,
                      sink_tokens=P, local_tokens=4 * P, budget_tokens=24 * P, T=T)
    lens = [1500, 900, 700, 1200]
    inp, g = gqa_case(cfg, seed=90 + T, seq_lens=lens)
    sig = oracle_summaries(inp, cfg)
    lists, counts = oracle_lists(inp, cfg, sig)
    qp = _positions(lens, T)
    h2l = [h // cfg.G for h in range(cfg.Hq)]
    scale = 1.0 / math.sqrt(cfg.D)
    lt, ct = torch.from_numpy(lists).to(DEV), torch.from_numpy(counts).to(DEV)
    qpd = torch.from_numpy(qp).to(DEV)
    if path == "split":
        o_p, l_p = sa.sa_sparse_decode_at(g["q"], g["k"], g["v"], g["page_table"], g["seq_lens"],
                                          qpd, lt, ct, h2l, scale, 3)
        o, _, lse = sa.sa_combine(o_p, l_p)
    else:
        o, _, lse = sa.sa_sparse_attention_at(g["q"], g["k"], g["v"], g["page_table"],
                                              g["seq_lens"], qpd, lt, ct, h2l, scale, 2)
    torch.cuda.synchronize()
    ro, rl = O.sparse_attention(bits(inp["q"]), bits(inp["k"]), bits(inp["v"]),
                                np_i32(inp["page_table"]), np_i32(inp["seq_lens"]), lists, counts,
                                np.array(h2l), scale, P, q_pos=qp)
    assert np.isneginf(rl[3, 0]).all()            # token 0 of sequence 3 sees no key
    assert_attn_close(o, lse, ro, rl)


def test_positions_mla():
    cfg = W.MLADecode("case", B=3, T=2, Hq=16, Dk=576, Dv=512, page_size=64, seq_len=2500,
                      alpha=3, beta=6, h_ambient=4)
    inp = W.mla_decode_inputs(cfg, seed=95, device="cpu")
    sig = O.page_summaries(bits(inp["kv"]), np_i32(inp["page_table"]), np_i32(inp["seq_lens"]), 64)
    lists, counts = mla_lists_from_oracle(inp, sig, cfg)
    g = {k: (v.to(DEV) if torch.is_tensor(v) else v) for k, v in inp.items()}
    amb = set(int(h) for h in inp["ambient_heads"].tolist())
    h2l = [1 if h in amb else 0 for h in range(cfg.Hq)]
    qp = np.array([1200, 2600, -1], dtype=np.int32)
    kv = g["kv"]
    scale = 1.0 / math.sqrt(cfg.Dk)
    o, _, lse = sa.sa_sparse_attention_at(g["q"], kv, kv[..., :cfg.Dv], g["page_table"],
                                          g["seq_lens"], torch.from_numpy(qp).to(DEV),
                                          torch.from_numpy(lists).to(DEV),
                                          torch.from_numpy(counts).to(DEV), h2l, scale, 3)
    torch.cuda.synchronize()
    kvb = bits(inp["kv"])
    ro, rl = O.sparse_attention(bits(inp["q"]), kvb, kvb[..., :cfg.Dv], np_i32(inp["page_table"]),
                                np_i32(inp["seq_lens"]), lists, counts, np.array(h2l), scale, 64,
                                q_pos=qp)
    assert_attn_close(o, lse, ro, rl)


def test_positions_are_required():
    cfg = W.scaled(W.TINY_GQA, B=1)
    inp, g = gqa_case(cfg, seed=96)
    lt = torch.zeros((1, 2, 4), dtype=torch.int32, device=DEV)
    ct = torch.zeros((1, 2), dtype=torch.int32, device=DEV)
    lib = sa.load()
    import ctypes
    h = (ctypes.c_int32 * 8)(*[x // 4 for x in range(8)])
    q = g["q"]
    st = lib.sa_sparse_decode_at(q.data_ptr(), (ctypes.c_int64 * 4)(*q.stride()), g["k"].data_ptr(),
                                 (ctypes.c_int64 * 4)(*g["k"].stride()), g["v"].data_ptr(),
                                 (ctypes.c_int64 * 4)(*g["v"].stride()),
                                 g["page_table"].data_ptr(), g["page_table"].shape[1],
                                 g["seq_lens"].data_ptr(), None, lt.data_ptr(), ct.data_ptr(), 2,
                                 4, ctypes.cast(h, ctypes.c_void_p), 1, 1, 8, 2, 64, 64, 16,
                                 g["k"].shape[0], 0.125, 1, None, None, None, None)
    assert st == 1
