"""The two-level page map (sa_build_page_summaries_dir, sa_sparse_step_dir,
sa_append_kv_dir) against the oracle and against the flat-table calls (marked
gpu).

The oracle sees only the flat table its own page_table_from_dir makes of the
directory and blocks (reading R19); the GPU reads the directory and blocks.
Summaries and selected pages must equal the oracle's bit for bit, O and LSE
hold the attention tolerance.  The flat-table calls on the table the map
stands for must give the same bits as the *_dir calls (same kernels, another
lookup).  Block sizes of 1, 4 and 16 pages; a directory hole inside a
sequence is flagged as a page outside the pool, like a bad flat-table entry.
At full size: 8 sequences of 64K-1M tokens in 64-token pages (million-token
page tables), the whole batch on the GPU, the oracle on sampled units.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import paged_sparse_kv_sa_b200 as sa
from paged_sparse_kv_sa_b200 import workloads as W
from test_gpu_parity import DEV, assert_attn_close, bits, gqa_case, np_i32

pytestmark = pytest.mark.gpu

ERR_POOL = 2      # SA_DEVERR_POOL_RANGE


def _small_cfg():
    return W.scaled(W.LLAMA8B_DECODE, B=4, Hq=16, Hkv=4, D=128, page_size=16, seq_len_lo=0,
                    seq_len_hi=0, sink_tokens=32, local_tokens=128, budget_tokens=512,
                    lift_frac=0.05, lift_sigma=3.0)


def _dir_case(cfg, lens, shift, seed):
    inp, g = gqa_case(cfg, seed=seed, seq_lens=lens)
    page_dir, blocks = W.page_directory(inp["page_table"], inp["seq_lens"], cfg.page_size, shift,
                                        seed=seed + 1)
    flat = O.page_table_from_dir(page_dir.numpy(), blocks.numpy(), shift)
    return inp, g, page_dir.to(DEV), blocks.to(DEV), flat


@pytest.mark.parametrize("shift", [0, 2, 4])
def test_dir_summaries_and_step_match_oracle(shift):
    cfg = _small_cfg()
    lens = [3000, 1, 777, 0]
    inp, g, page_dir, blocks, flat = _dir_case(cfg, lens, shift, seed=60 + shift)
    sl = np_i32(inp["seq_lens"])
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    sig = sa.sa_build_page_summaries_dir(g["k"], page_dir, blocks, shift, g["seq_lens"],
                                         dev_error=err)
    ref_sig = O.page_summaries(bits(inp["k"]), flat, sl, cfg.page_size)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(bits(sig), ref_sig)
    scale = 1.0 / math.sqrt(cfg.D)
    pages, counts, o, _, lse = sa.sa_sparse_step_dir(
        g["q"], sig, g["k"], g["v"], page_dir, blocks, shift, g["seq_lens"], cfg.page_size,
        cfg.sink_tokens, cfg.local_tokens, cfg.budget_tokens, scale, n_splits=3, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rp, rc = O.select_pages(bits(inp["q"]), ref_sig, flat, sl, cfg.page_size, cfg.sink_tokens,
                            cfg.local_tokens, cfg.budget_tokens)
    assert np.array_equal(np_i32(counts), rc)
    assert np.array_equal(np_i32(pages), rp)
    h2l = np.array([h // cfg.G for h in range(cfg.Hq)])
    ro, rl = O.sparse_attention(bits(inp["q"]), bits(inp["k"]), bits(inp["v"]), flat, sl, rp, rc,
                                h2l, scale, cfg.page_size)
    assert_attn_close(o, lse, ro, rl)
    # the flat-table call on the table the map stands for: the same bits
    pt_flat = torch.from_numpy(flat).to(DEV)
    sig_f = sa.sa_build_page_summaries(g["k"], pt_flat, g["seq_lens"])
    pf, cf, of, _, lf = sa.sa_sparse_step(g["q"], sig_f, g["k"], g["v"], pt_flat, g["seq_lens"],
                                          cfg.page_size, cfg.sink_tokens, cfg.local_tokens,
                                          cfg.budget_tokens, scale, n_splits=3)
    torch.cuda.synchronize()
    assert torch.equal(sig_f, sig)
    assert torch.equal(pf, pages) and torch.equal(cf, counts)
    assert torch.equal(of, o) and torch.equal(lf, lse)


def test_dir_hole_is_flagged_like_a_bad_flat_entry():
    cfg = _small_cfg()
    lens = [3000, 900, 777, 400]
    shift = 2
    inp, g, page_dir, blocks, flat = _dir_case(cfg, lens, shift, seed=70)
    holed = page_dir.clone()
    holed[1, 3] = -1                          # pages 12..15 of sequence 1 (of 57)
    flat_holed = flat.copy()
    flat_holed[1, 12:16] = -1
    scale = 1.0 / math.sqrt(cfg.D)
    outs = []
    for use_dir in (True, False):
        err = torch.zeros(1, dtype=torch.int32, device=DEV)
        if use_dir:
            sig = sa.sa_build_page_summaries_dir(g["k"], holed, blocks, shift, g["seq_lens"],
                                                 dev_error=err)
            r = sa.sa_sparse_step_dir(g["q"], sig, g["k"], g["v"], holed, blocks, shift,
                                      g["seq_lens"], cfg.page_size, cfg.sink_tokens,
                                      cfg.local_tokens, cfg.budget_tokens, scale, n_splits=2,
                                      dev_error=err)
        else:
            pt = torch.from_numpy(flat_holed).to(DEV)
            sig = sa.sa_build_page_summaries(g["k"], pt, g["seq_lens"], dev_error=err)
            r = sa.sa_sparse_step(g["q"], sig, g["k"], g["v"], pt, g["seq_lens"], cfg.page_size,
                                  cfg.sink_tokens, cfg.local_tokens, cfg.budget_tokens, scale,
                                  n_splits=2, dev_error=err)
        torch.cuda.synchronize()
        assert int(err.item()) & ERR_POOL
        outs.append((sig, r[0], r[1], r[2], r[4]))
    for a, b in zip(*outs):
        assert torch.equal(a, b)
    # the other sequences are untouched by the hole: their rows match the oracle
    sl = np_i32(inp["seq_lens"])
    ref_sig = O.page_summaries(bits(inp["k"]), flat, sl, cfg.page_size)
    sig, pages, counts, o, lse = outs[0]
    keep = [0, 2, 3]
    rp, rc = O.select_pages(bits(inp["q"][keep]), ref_sig, flat[keep], sl[keep], cfg.page_size,
                            cfg.sink_tokens, cfg.local_tokens, cfg.budget_tokens)
    assert np.array_equal(np_i32(pages[keep]), rp) and np.array_equal(np_i32(counts[keep]), rc)


@pytest.mark.parametrize("shift", [0, 3])
def test_dir_append_matches_oracle(shift):
    P, Hkv, D, max_new = 16, 4, 64, 40
    lens = [0, 15, 200, 333]
    g = torch.Generator().manual_seed(80 + shift)
    B = len(lens)
    npg = [-(-(L + max_new) // P) for L in lens]
    pool = sum(npg) + 5
    perm = torch.randperm(pool, generator=g).numpy()
    pt = np.full((B, max(npg)), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(npg):
        pt[b, :n] = perm[off:off + n]
        off += n
    cap_lens = torch.tensor([n * P for n in npg], dtype=torch.int32)   # every allocated page
    page_dir, blocks = W.page_directory(torch.from_numpy(pt), cap_lens, P, shift, seed=5)
    flat = O.page_table_from_dir(page_dir.numpy(), blocks.numpy(), shift)
    k = bits(torch.randn((pool, Hkv, P, D), generator=g).to(torch.bfloat16))
    v = bits(torch.randn((pool, Hkv, P, D), generator=g).to(torch.bfloat16))
    sl = np.array(lens, dtype=np.int32)
    sig = O.page_summaries(k, flat, sl, P)
    kn = bits(torch.randn((B, max_new, Hkv, D), generator=g).to(torch.bfloat16))
    vn = bits(torch.randn((B, max_new, Hkv, D), generator=g).to(torch.bfloat16))
    nn = np.array([40, 1, 17, 0], dtype=np.int32)
    rk, rv, rs, rl = O.append_kv(k, v, sig, flat, sl, kn, vn, nn, P)

    def dev(x):
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).to(DEV)
    kd, vd, sd = dev(k), dev(v), dev(sig)
    out_len = torch.full((B,), -1, dtype=torch.int32, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    sa.sa_append_kv_dir(dev(kn), dev(vn), torch.from_numpy(nn).to(DEV), kd, vd, page_dir.to(DEV),
                        blocks.to(DEV), shift, torch.from_numpy(sl).to(DEV), sd,
                        out_seq_lens=out_len, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(bits(kd), rk) and np.array_equal(bits(vd), rv)
    assert np.array_equal(bits(sd), rs)
    assert np.array_equal(out_len.cpu().numpy(), rl)


# ----------------------------------------------------------------------------
# full size: million-token page tables
# ----------------------------------------------------------------------------
def _local_unit(inp, flat, cfg, b, kvh):
    """Unit (b, kv head) as a local problem over the pages the oracle's flat
    table gives it (identity page table over those pages)."""
    L = int(inp["seq_lens"][b].item())
    N = -(-L // cfg.page_size)
    phys = torch.from_numpy(flat[b, :N].astype(np.int64)).to(inp["k"].device)
    G = cfg.G
    k = bits(inp["k"][phys, kvh].unsqueeze(1))
    v = bits(inp["v"][phys, kvh].unsqueeze(1))
    q = bits(inp["q"][b:b + 1, :, kvh * G:(kvh + 1) * G])
    return q, k, v, np.arange(N, dtype=np.int32).reshape(1, N), np.array([L], np.int32), phys


@pytest.mark.slow
def test_dir_million_token_workload():
    cfg = W.LLAMA8B_DIR_1M
    shift = W.DIR_BLOCK_SHIFT
    inp = W.gqa_decode_inputs(cfg, seed=0, device=DEV)
    page_dir, blocks = W.page_directory(inp["page_table"], inp["seq_lens"], cfg.page_size, shift)
    flat = O.page_table_from_dir(np_i32(page_dir), np_i32(blocks), shift)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    sig = sa.sa_build_page_summaries_dir(inp["k"], page_dir, blocks, shift, inp["seq_lens"],
                                         dev_error=err)
    scale = 1.0 / math.sqrt(cfg.D)
    pages, counts, o, _, lse = sa.sa_sparse_step_dir(
        inp["q"], sig, inp["k"], inp["v"], page_dir, blocks, shift, inp["seq_lens"],
        cfg.page_size, cfg.sink_tokens, cfg.local_tokens, cfg.budget_tokens, scale, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    # the flat call on the (million-token) table the map stands for: same bits
    pt = torch.from_numpy(flat[:, :inp["page_table"].shape[1]]).to(DEV)
    sig_f = sa.sa_build_page_summaries(inp["k"], pt, inp["seq_lens"])
    pf, cf, of, _, lf = sa.sa_sparse_step(inp["q"], sig_f, inp["k"], inp["v"], pt,
                                          inp["seq_lens"], cfg.page_size, cfg.sink_tokens,
                                          cfg.local_tokens, cfg.budget_tokens, scale)
    torch.cuda.synchronize()
    assert torch.equal(sig_f, sig)
    assert torch.equal(pf, pages) and torch.equal(cf, counts)
    assert torch.equal(of, o) and torch.equal(lf, lse)
    # the oracle on sampled units: the longest sequence's and two others
    lens = np_i32(inp["seq_lens"])
    rng = np.random.default_rng(7)
    units = {(int(np.argmax(lens)), int(rng.integers(cfg.Hkv)))}
    while len(units) < 3:
        units.add((int(rng.integers(cfg.B)), int(rng.integers(cfg.Hkv))))
    for b, kvh in sorted(units):
        q, k, v, lpt, lsl, phys = _local_unit(inp, flat, cfg, b, kvh)
        ref_sig = O.page_summaries(k, lpt, lsl, cfg.page_size)
        assert np.array_equal(bits(sig[phys, kvh]), ref_sig[:, 0]), (b, kvh)
        rp, rc = O.select_pages(q, ref_sig, lpt, lsl, cfg.page_size, cfg.sink_tokens,
                                cfg.local_tokens, cfg.budget_tokens)
        assert int(counts[b, kvh]) == int(rc[0, 0]), (b, kvh)
        assert np.array_equal(np_i32(pages[b, kvh]), rp[0, 0]), (b, kvh)
        ro, rl = O.sparse_attention(q, k, v, lpt, lsl, rp, rc, np.zeros(cfg.G, np.int64), scale,
                                    cfg.page_size)
        G = cfg.G
        assert_attn_close(o[b:b + 1, :, kvh * G:(kvh + 1) * G],
                          lse[b:b + 1, :, kvh * G:(kvh + 1) * G], ro, rl)
