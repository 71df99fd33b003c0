"""sa_sparse_attention(_fp8): the decode and the split merge in one call (marked gpu).

Every decode path (warp-MMA GQA, FP8, tcgen05 MLA and many-row) is checked
against the float64 oracle with the parity bar of the decode tests, and the bf16
output against the float32 one (it is its round-to-nearest-even).
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import paged_sparse_kv_sa_b200 as sa
from oracle import sa_oracle as O
from paged_sparse_kv_sa_b200 import workloads as W
from test_gpu_parity import (DEV, assert_attn_close, bits, fp8_case, gqa_case, mla_lists_from_oracle,
                             np_i32, oracle_fp8, oracle_lists, oracle_summaries, to_bf16_dev)

pytestmark = pytest.mark.gpu


def attend(g, lists, counts, cfg, n_splits, h2l=None, ws=None, **kw):
    Hq, Hkv = cfg.Hq, cfg.Hkv
    h2l = [h // (Hq // Hkv) for h in range(Hq)] if h2l is None else h2l
    o, ob, lse = sa.sa_sparse_attention(g["q"], g["k"], g["v"], g["page_table"], g["seq_lens"],
                                        torch.from_numpy(lists).to(DEV),
                                        torch.from_numpy(counts).to(DEV), h2l,
                                        1.0 / math.sqrt(cfg.D), n_splits, workspace=ws, **kw)
    torch.cuda.synchronize()
    return o, ob, lse


@pytest.mark.parametrize("D,P,T,n_splits", [(128, 16, 1, 13), (128, 16, 2, 3), (64, 32, 2, 5),
                                            (256, 16, 1, 4), (128, 64, 1, 1), (128, 16, 1, 40)])
def test_attention_vs_oracle(D, P, T, n_splits):
    cfg = W.GQADecode("case", B=3, Hq=8, Hkv=2, D=D, page_size=P, seq_len_lo=0, seq_len_hi=0,
                      sink_tokens=P, local_tokens=2 * P, budget_tokens=12 * P, T=T)
    lens = [50 * P + 7, 9 * P, 3 * P + 1]
    inp, g = gqa_case(cfg, seed=41, seq_lens=lens)
    sig = oracle_summaries(inp, cfg)
    lists, counts = oracle_lists(inp, cfg, sig)
    ws = sa.attention_workspace(cfg.B, T, cfg.Hq, D, n_splits, DEV)
    o, ob, lse = attend(g, lists, counts, cfg, n_splits, ws=ws, want_bf16=True)
    ro, rl = O.sparse_attention(bits(inp["q"]), bits(inp["k"]), bits(inp["v"]),
                                np_i32(inp["page_table"]), np_i32(inp["seq_lens"]), lists, counts,
                                np.arange(cfg.Hq) // cfg.G, 1.0 / math.sqrt(D), P)
    assert_attn_close(o, lse, ro, rl)
    assert torch.equal(ob, o.to(torch.bfloat16)), "bf16 output is not the rounded float32 one"


def test_attention_per_head_lists_and_empty_list():
    # heads of one kv group read different lists, one list empty (its rows: O = 0, lse = -inf)
    cfg = W.GQADecode("case", B=2, Hq=8, Hkv=2, D=128, page_size=16, seq_len_lo=0, seq_len_hi=0,
                      sink_tokens=16, local_tokens=16, budget_tokens=160)
    inp, g = gqa_case(cfg, seed=42, seq_lens=[700, 333])
    rng = np.random.default_rng(42)
    n_lists, cap = 3, 9
    lists = np.full((2, n_lists, cap), -1, dtype=np.int32)
    counts = np.zeros((2, n_lists), dtype=np.int32)
    for b, L in enumerate([700, 333]):
        nb = -(-L // 16)
        for li in range(n_lists - 1):
            c = int(rng.integers(1, cap + 1))
            lists[b, li, :c] = np.sort(rng.choice(nb, c, replace=False))
            counts[b, li] = c
    h2l = [0, 1, 2, 0, 1, 1, 2, 0]
    ws = sa.attention_workspace(2, 1, 8, 128, 3, DEV)
    o, _, lse = attend(g, lists, counts, cfg, 3, h2l=h2l, ws=ws)
    ro, rl = O.sparse_attention(bits(inp["q"]), bits(inp["k"]), bits(inp["v"]),
                                np_i32(inp["page_table"]), np_i32(inp["seq_lens"]), lists, counts,
                                np.array(h2l), 1.0 / math.sqrt(128), 16)
    assert_attn_close(o, lse, ro, rl)


def test_attention_workspace_reused_across_calls():
    # one workspace, three calls with different data and lengths: nothing a call
    # leaves in it may leak into the next
    cfg = W.scaled(W.LLAMA8B_DECODE, B=2, Hq=8, Hkv=2, seq_len_lo=0, seq_len_hi=0)
    n_splits = 7
    ws = sa.attention_workspace(cfg.B, cfg.T, cfg.Hq, cfg.D, n_splits, DEV)
    for i, lens in enumerate([[4000, 1500], [300, 2600], [5000, 17]]):
        inp, g = gqa_case(cfg, seed=50 + i, seq_lens=lens)
        sig = oracle_summaries(inp, cfg)
        lists, counts = oracle_lists(inp, cfg, sig)
        o, _, lse = attend(g, lists, counts, cfg, n_splits, ws=ws)
        ro, rl = O.sparse_attention(bits(inp["q"]), bits(inp["k"]), bits(inp["v"]),
                                    np_i32(inp["page_table"]), np_i32(inp["seq_lens"]), lists,
                                    counts, np.arange(cfg.Hq) // cfg.G, 1.0 / math.sqrt(cfg.D),
                                    cfg.page_size)
        assert_attn_close(o, lse, ro, rl)


def test_attention_lse_only():
    cfg = W.scaled(W.TINY_GQA, B=2)
    inp, g = gqa_case(cfg, seed=43)
    sig = oracle_summaries(inp, cfg)
    lists, counts = oracle_lists(inp, cfg, sig)
    o, ob, lse = attend(g, lists, counts, cfg, 3, want_f32=False)
    assert o is None and ob is None
    _, rl = O.sparse_attention(bits(inp["q"]), bits(inp["k"]), bits(inp["v"]),
                               np_i32(inp["page_table"]), np_i32(inp["seq_lens"]), lists, counts,
                               np.arange(cfg.Hq) // cfg.G, 1.0 / math.sqrt(cfg.D), cfg.page_size)
    got = lse.cpu().double().numpy()
    fin = np.isfinite(rl)
    assert np.array_equal(np.isfinite(got), fin)
    assert np.abs(got[fin] - rl[fin]).max() <= 1e-3


@pytest.mark.parametrize("n_splits", [1, 3, 13])
def test_attention_fp8_vs_oracle(n_splits):
    cfg = W.scaled(W.TINY_GQA, D=128, B=3)
    inp, g, f8, f8d = fp8_case(cfg, seed=44, seq_lens=[2048, 1000 + 3, 37])
    sig = O.page_summaries_fp8(f8["kc"].numpy(), f8["ks"].numpy(), np_i32(inp["page_table"]),
                               np_i32(inp["seq_lens"]), cfg.page_size)
    lists, counts = oracle_lists(inp, cfg, sig)
    h2l = [h // cfg.G for h in range(cfg.Hq)]
    ws = sa.attention_workspace(cfg.B, cfg.T, cfg.Hq, 128, n_splits, DEV)
    o, _, lse = sa.sa_sparse_attention_fp8(g["q"], f8d["kc"], f8d["vc"], f8d["ks"], f8d["vs"],
                                           g["page_table"], g["seq_lens"],
                                           torch.from_numpy(lists).to(DEV),
                                           torch.from_numpy(counts).to(DEV), h2l,
                                           1.0 / math.sqrt(cfg.D), n_splits, workspace=ws)
    torch.cuda.synchronize()
    ro, rl = oracle_fp8(inp, f8, lists, counts, cfg)
    assert_attn_close(o, lse, ro, rl)


def test_attention_mla_path():
    cfg = W.MLADecode("case", B=2, T=2, Hq=16, Dk=576, Dv=512, page_size=64, seq_len=2500,
                      alpha=3, beta=6, h_ambient=4)
    inp = W.mla_decode_inputs(cfg, seed=45, device="cpu")
    sig = O.page_summaries(bits(inp["kv"]), np_i32(inp["page_table"]), np_i32(inp["seq_lens"]), 64)
    lists, counts = mla_lists_from_oracle(inp, sig, cfg)
    g = {k: (v.to(DEV) if torch.is_tensor(v) else v) for k, v in inp.items()}
    amb = set(int(h) for h in inp["ambient_heads"].tolist())
    h2l = [1 if h in amb else 0 for h in range(cfg.Hq)]
    kv = g["kv"]
    o, _, lse = sa.sa_sparse_attention(g["q"], kv, kv[..., :cfg.Dv], g["page_table"],
                                       g["seq_lens"], torch.from_numpy(lists).to(DEV),
                                       torch.from_numpy(counts).to(DEV), h2l,
                                       1.0 / math.sqrt(cfg.Dk), 3)
    torch.cuda.synchronize()
    kvb = bits(inp["kv"])
    ro, rl = O.sparse_attention(bits(inp["q"]), kvb, kvb[..., :cfg.Dv], np_i32(inp["page_table"]),
                                np_i32(inp["seq_lens"]), lists, counts, np.array(h2l),
                                1.0 / math.sqrt(cfg.Dk), 64)
    assert_attn_close(o, lse, ro, rl)


def test_attention_tensor_core_path():
    # 32 query rows per pair (T = 4, 8 heads per kv head): the tcgen05 kernel
    cfg = W.GQADecode("case", B=2, Hq=16, Hkv=2, D=128, page_size=16, seq_len_lo=0, seq_len_hi=0,
                      sink_tokens=16, local_tokens=64, budget_tokens=256, T=4)
    inp, g = gqa_case(cfg, seed=46, seq_lens=[3000, 777])
    sig = oracle_summaries(inp, cfg)
    lists, counts = oracle_lists(inp, cfg, sig)
    o, _, lse = attend(g, lists, counts, cfg, 2)
    ro, rl = O.sparse_attention(bits(inp["q"]), bits(inp["k"]), bits(inp["v"]),
                                np_i32(inp["page_table"]), np_i32(inp["seq_lens"]), lists, counts,
                                np.arange(cfg.Hq) // cfg.G, 1.0 / math.sqrt(cfg.D), cfg.page_size)
    assert_attn_close(o, lse, ro, rl)


def test_attention_argument_errors():
    cfg = W.scaled(W.TINY_GQA, B=2)
    inp, g = gqa_case(cfg, seed=47)
    sig = oracle_summaries(inp, cfg)
    lists, counts = oracle_lists(inp, cfg, sig)
    h2l = [h // cfg.G for h in range(cfg.Hq)]
    args = (g["q"], g["k"], g["v"], g["page_table"], g["seq_lens"], torch.from_numpy(lists).to(DEV),
            torch.from_numpy(counts).to(DEV), h2l, 1.0 / math.sqrt(cfg.D), 3)
    short = torch.zeros(64, dtype=torch.uint8, device=DEV)
    with pytest.raises(sa.SAError, match="WORKSPACE"):
        sa.sa_sparse_attention(*args, workspace=short)
    with pytest.raises(sa.SAError, match="INVALID_ARG"):   # no output at all
        lib = sa.load()
        q = g["q"]
        ws = sa.attention_workspace(cfg.B, cfg.T, cfg.Hq, cfg.D, 3, DEV)
        h = (ctypes.c_int32 * cfg.Hq)(*h2l)
        st = lib.sa_sparse_attention(q.data_ptr(), (ctypes.c_int64 * 4)(*q.stride()),
                                     g["k"].data_ptr(), (ctypes.c_int64 * 4)(*g["k"].stride()),
                                     g["v"].data_ptr(), (ctypes.c_int64 * 4)(*g["v"].stride()),
                                     g["page_table"].data_ptr(), g["page_table"].shape[1],
                                     g["seq_lens"].data_ptr(), args[5].data_ptr(),
                                     args[6].data_ptr(), cfg.Hkv, lists.shape[2],
                                     ctypes.cast(h, ctypes.c_void_p), cfg.B, cfg.T, cfg.Hq,
                                     cfg.Hkv, cfg.D, cfg.D, cfg.page_size, g["k"].shape[0],
                                     1.0 / math.sqrt(cfg.D), 3, None, None, None, ws.data_ptr(),
                                     ws.numel(), None, None)
        sa._lib._check(st, "sa_sparse_attention")


def _scaled_case(path, scale_mult, seed):
    """(o, lse, o_ref, lse_ref) of one call with scale = scale_mult / sqrt(Dk)."""
    if path == "mla":
        cfg = W.MLADecode("case", B=2, T=2, Hq=16, Dk=576, Dv=512, page_size=64, seq_len=1500,
                          alpha=3, beta=6, h_ambient=4)
        inp = W.mla_decode_inputs(cfg, seed=seed, device="cpu")
        scale = scale_mult / math.sqrt(cfg.Dk)
        sig = O.page_summaries(bits(inp["kv"]), np_i32(inp["page_table"]),
                               np_i32(inp["seq_lens"]), 64)
        lists, counts = mla_lists_from_oracle(inp, sig, cfg)
        g = {k: (v.to(DEV) if torch.is_tensor(v) else v) for k, v in inp.items()}
        amb = set(int(h) for h in inp["ambient_heads"].tolist())
        h2l = [1 if h in amb else 0 for h in range(cfg.Hq)]
        kv = g["kv"]
        o, _, lse = sa.sa_sparse_attention(g["q"], kv, kv[..., :cfg.Dv], g["page_table"],
                                           g["seq_lens"], torch.from_numpy(lists).to(DEV),
                                           torch.from_numpy(counts).to(DEV), h2l, scale, 2)
        torch.cuda.synchronize()
        kvb = bits(inp["kv"])
        ro, rl = O.sparse_attention(bits(inp["q"]), kvb, kvb[..., :cfg.Dv],
                                    np_i32(inp["page_table"]), np_i32(inp["seq_lens"]), lists,
                                    counts, np.array(h2l), scale, 64)
    else:
        T, Hq = (1, 8) if path == "gqa" else (4, 16)
        cfg = W.GQADecode("case", B=2, Hq=Hq, Hkv=2, D=128, page_size=16, seq_len_lo=0,
                          seq_len_hi=0, sink_tokens=16, local_tokens=64, budget_tokens=256, T=T)
        inp, g = gqa_case(cfg, seed=seed, seq_lens=[3000, 777 if T > 1 else 35])
        scale = scale_mult / math.sqrt(cfg.D)
        sig = oracle_summaries(inp, cfg)
        lists, counts = oracle_lists(inp, cfg, sig)
        h2l = [h // cfg.G for h in range(cfg.Hq)]
        o, _, lse = sa.sa_sparse_attention(g["q"], g["k"], g["v"], g["page_table"],
                                           g["seq_lens"], torch.from_numpy(lists).to(DEV),
                                           torch.from_numpy(counts).to(DEV), h2l, scale, 3)
        torch.cuda.synchronize()
        ro, rl = O.sparse_attention(bits(inp["q"]), bits(inp["k"]), bits(inp["v"]),
                                    np_i32(inp["page_table"]), np_i32(inp["seq_lens"]), lists,
                                    counts, np.arange(cfg.Hq) // cfg.G, scale, cfg.page_size)
    return o, lse, ro, rl


@pytest.mark.parametrize("path", ["gqa", "tensor_core", "mla"])
def test_attention_negative_scale(path):
    # the scale may be any finite number: with s < 0 the row max of the scaled scores
    # is s times the smallest raw score, and masked keys must still weigh nothing
    assert_attn_close(*_scaled_case(path, -1.0, 48))


@pytest.mark.parametrize("mult", [3.0, 8.0])
@pytest.mark.parametrize("path", ["gqa", "tensor_core", "mla"])
def test_attention_sharp_softmax(path, mult):
    # three and eight times the usual 1/sqrt(D): a few keys dominate each row, so
    # the probabilities' rounding before the PV product shows directly in O.
    # Every kernel multiplies by P as a bf16 pair hi + lo (~2^-17 relative; a
    # single bf16 P, 2^-9, missed the bar at three times the scale)
    assert_attn_close(*_scaled_case(path, mult, 49))


@pytest.mark.parametrize("D,P,T,n_splits", [(128, 16, 1, 0), (64, 32, 2, 3), (256, 16, 1, 0),
                                            (128, 64, 1, 5)])
def test_step_vs_oracle(D, P, T, n_splits):
    # sa_sparse_step: selection + attention + merge in one C call (n_splits 0 = the
    # library's default), against the oracle's selection and attention
    cfg = W.GQADecode("case", B=3, Hq=8, Hkv=2, D=D, page_size=P, seq_len_lo=0, seq_len_hi=0,
                      sink_tokens=P, local_tokens=2 * P, budget_tokens=12 * P, T=T)
    lens = [50 * P + 7, 9 * P, 3 * P + 1]
    inp, g = gqa_case(cfg, seed=60, seq_lens=lens)
    sig = oracle_summaries(inp, cfg)
    scale = 1.0 / math.sqrt(D)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    pages, counts, o, _, lse = sa.sa_sparse_step(g["q"], to_bf16_dev(sig), g["k"], g["v"],
                                                 g["page_table"], g["seq_lens"], P,
                                                 cfg.sink_tokens, cfg.local_tokens,
                                                 cfg.budget_tokens, scale, n_splits,
                                                 dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rp, rc = O.select_pages(bits(inp["q"]), sig, np_i32(inp["page_table"]),
                            np_i32(inp["seq_lens"]), P, cfg.sink_tokens, cfg.local_tokens,
                            cfg.budget_tokens)
    assert np.array_equal(np_i32(counts), rc) and np.array_equal(np_i32(pages), rp)
    ro, rl = O.sparse_attention(bits(inp["q"]), bits(inp["k"]), bits(inp["v"]),
                                np_i32(inp["page_table"]), np_i32(inp["seq_lens"]), rp, rc,
                                np.arange(cfg.Hq) // cfg.G, scale, P)
    assert_attn_close(o, lse, ro, rl)


@pytest.mark.parametrize("P,T,n_splits", [(16, 1, 0), (32, 2, 3)])
def test_step_fp8_vs_oracle(P, T, n_splits):
    # sa_sparse_step_fp8: selection on the FP8 pages' summaries, attention over the
    # FP8 pages and the merge in one C call, against the oracle; and the same bits
    # as the selection and the FP8 attention called one after the other
    cfg = W.GQADecode("case", B=3, Hq=8, Hkv=2, D=128, page_size=P, seq_len_lo=0, seq_len_hi=0,
                      sink_tokens=P, local_tokens=2 * P, budget_tokens=12 * P, T=T)
    lens = [50 * P + 7, 9 * P, 3 * P + 1]
    inp, g, f8, f8d = fp8_case(cfg, seed=64, seq_lens=lens)
    sig = O.page_summaries_fp8(f8["kc"].numpy(), f8["ks"].numpy(), np_i32(inp["page_table"]),
                               np_i32(inp["seq_lens"]), P)
    sig_d = to_bf16_dev(sig)
    scale = 1.0 / math.sqrt(cfg.D)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    pages, counts, o, _, lse = sa.sa_sparse_step_fp8(
        g["q"], sig_d, f8d["kc"], f8d["vc"], f8d["ks"], f8d["vs"], g["page_table"],
        g["seq_lens"], P, cfg.sink_tokens, cfg.local_tokens, cfg.budget_tokens, scale, n_splits,
        dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rp, rc = O.select_pages(bits(inp["q"]), sig, np_i32(inp["page_table"]),
                            np_i32(inp["seq_lens"]), P, cfg.sink_tokens, cfg.local_tokens,
                            cfg.budget_tokens)
    assert np.array_equal(np_i32(counts), rc) and np.array_equal(np_i32(pages), rp)
    ro, rl = oracle_fp8(inp, f8, rp, rc, cfg)
    assert_attn_close(o, lse, ro, rl)
    # the two-call path gives the same bits
    p2, c2 = sa.sa_select_pages(g["q"], sig_d, g["page_table"], g["seq_lens"], P,
                                cfg.sink_tokens, cfg.local_tokens, cfg.budget_tokens)
    ns = n_splits or sa.default_splits(cfg.B * cfg.Hkv, cfg.budget_tokens // P)
    o2, _, l2 = sa.sa_sparse_attention_fp8(g["q"], f8d["kc"], f8d["vc"], f8d["ks"], f8d["vs"],
                                           g["page_table"], g["seq_lens"], p2, c2,
                                           [h // cfg.G for h in range(cfg.Hq)], scale, ns)
    torch.cuda.synchronize()
    assert torch.equal(p2, pages) and torch.equal(o2, o) and torch.equal(l2, lse)


def test_bound_calls_replay_on_new_contents():
    # sa.bind records the C calls of a step once; replaying them after the input
    # tensors' contents change (same storage) must give what fresh calls give
    cfg = W.GQADecode("case", B=2, Hq=8, Hkv=2, D=128, page_size=16, seq_len_lo=0, seq_len_hi=0,
                      sink_tokens=16, local_tokens=64, budget_tokens=256)
    inp, g = gqa_case(cfg, seed=61, seq_lens=[3000, 1111])
    sig = to_bf16_dev(oracle_summaries(inp, cfg))
    step = sa.SparseDecodeStep(cfg.B, cfg.T, cfg.Hq, cfg.Hkv, cfg.D, cfg.page_size,
                               g["page_table"].shape[1], cfg.sink_tokens, cfg.local_tokens,
                               cfg.budget_tokens, device=DEV)
    q = g["q"].clone()
    run = step.bind(q, g["k"], g["v"], sig, g["page_table"], g["seq_lens"])
    assert run.n_calls == 1
    for seed in (62, 63):
        q.copy_(torch.randn(q.shape, generator=torch.Generator().manual_seed(seed))
                .to(torch.bfloat16).to(DEV))
        run()
        torch.cuda.synchronize()
        got = (step.pages.clone(), step.o.clone(), step.lse.clone())
        ref = sa.sa_sparse_step(q, sig, g["k"], g["v"], g["page_table"], g["seq_lens"],
                                cfg.page_size, cfg.sink_tokens, cfg.local_tokens,
                                cfg.budget_tokens, step.scale, step.n_splits)
        torch.cuda.synchronize()
        assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[2])
        assert torch.equal(got[2], ref[4])
