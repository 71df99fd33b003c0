"""sa_select_ambient_heads against the oracle (marked gpu).

The head set is an index result decided by float64 scores (reading R16): the
GPU sums its float64 dot products and masses in another order than the oracle,
so the scores agree to ~1e-12 relative, not bit for bit.  The chosen heads must
equal the oracle's; the only tolerated difference is a swap at the boundary
between two heads whose oracle scores are within 1e-9 of each other (then both
sets are valid), which the test accepts explicitly.  Cases: an MLA-shaped call
with 2 sequences, the full MLA + MTP workload (8 sequences of 65536 tokens, 128
heads, 32 chosen), both from the tiered selection's lists, and the chosen heads
fed to the decode end to end.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import paged_sparse_kv_sa_b200 as sa
from paged_sparse_kv_sa_b200 import workloads as W
from test_gpu_parity import DEV, assert_attn_close, bits, np_i32, to_bf16_dev

pytestmark = pytest.mark.gpu


def _check_heads(got_heads, got_scores, want_heads, want_scores, h):
    got_heads = sorted(int(x) for x in got_heads)
    want_heads = sorted(int(x) for x in want_heads)
    assert np.allclose(got_scores, want_scores, rtol=1e-9, atol=1e-12)
    if got_heads != want_heads:
        # only a boundary swap between heads of (nearly) equal score is valid
        kth = np.sort(want_scores)[::-1][h - 1]
        for x in set(got_heads) ^ set(want_heads):
            assert abs(want_scores[x] - kth) <= 1e-9 * max(1.0, abs(kth)), (x, want_scores[x], kth)


def _case(cfg, seed, device):
    inp = W.mla_decode_inputs(cfg, seed=seed, device=device)
    g = {k: (v.to(DEV) if torch.is_tensor(v) else v) for k, v in inp.items()}
    sig = sa.sa_build_page_summaries(g["kv"], g["page_table"], g["seq_lens"])
    lists, counts = sa.sa_select_pages_tiered(g["q"], sig, g["page_table"], g["seq_lens"],
                                              cfg.page_size, cfg.alpha, cfg.beta)
    torch.cuda.synchronize()
    return inp, g, sig, lists, counts


def _oracle(inp, g, sig, lists, counts, cfg, scale, h):
    ls, cs = np_i32(lists), np_i32(counts)
    crit = [ls[b, 0, :cs[b, 0]] for b in range(cfg.B)]
    both = [ls[b, 1, :cs[b, 1]] for b in range(cfg.B)]
    return O.select_ambient_heads(bits(g["q"]), bits(sig), np_i32(g["page_table"]),
                                  np_i32(g["seq_lens"]), crit, cs[:, 0], both, cs[:, 1], scale,
                                  cfg.page_size, h)


@pytest.mark.parametrize("h", [1, 4, 12])
def test_heads_small(h):
    cfg = W.MLADecode("case", B=2, T=2, Hq=16, Dk=576, Dv=512, page_size=64, seq_len=2500,
                      alpha=3, beta=6, h_ambient=h)
    inp, g, sig, lists, counts = _case(cfg, 80 + h, "cpu")
    scale = float(np.float32(1.0 / math.sqrt(cfg.Dk)))   # the float32 the C call takes
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    heads, scores = sa.sa_select_ambient_heads(g["q"], sig, g["page_table"], g["seq_lens"], lists,
                                               counts, cfg.page_size, scale, h, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    wh, ws = _oracle(inp, g, sig, lists, counts, cfg, scale, h)
    got = heads.cpu().numpy()
    assert list(got) == sorted(got)
    _check_heads(got, scores.cpu().numpy(), wh, ws, h)


@pytest.mark.slow
def test_heads_mla_workload_and_decode_with_them():
    cfg = W.MLA_MTP
    inp, g, sig, lists, counts = _case(cfg, 0, "cuda")
    scale = float(np.float32(1.0 / math.sqrt(cfg.Dk)))   # the float32 the C call takes
    heads, scores = sa.sa_select_ambient_heads(g["q"], sig, g["page_table"], g["seq_lens"], lists,
                                               counts, cfg.page_size, scale, cfg.h_ambient)
    torch.cuda.synchronize()
    wh, ws = _oracle(inp, g, sig, lists, counts, cfg, scale, cfg.h_ambient)
    _check_heads(heads.cpu().numpy(), scores.cpu().numpy(), wh, ws, cfg.h_ambient)
    # the chosen heads attend critical + ambient pages, the others critical only
    chosen = set(int(x) for x in heads.cpu().numpy())
    h2l = [1 if h in chosen else 0 for h in range(cfg.Hq)]
    kv = g["kv"]
    o, _, lse = sa.sa_sparse_attention(g["q"], kv, kv[..., :cfg.Dv], g["page_table"],
                                       g["seq_lens"], lists, counts, h2l, scale, 8)
    torch.cuda.synchronize()
    rng = np.random.default_rng(3)
    rows = [(b, t, int(hh)) for b in range(cfg.B) for t in range(cfg.T)
            for hh in rng.choice(cfg.Hq, 3, replace=False)]
    ls, cs = np_i32(lists), np_i32(counts)
    L = int(inp["seq_lens"][0])
    for b, t, hh in rows:
        lst = ls[b, h2l[hh], :cs[b, h2l[hh]]]
        phys = np_i32(g["page_table"])[b, lst]
        kvb = bits(kv[torch.from_numpy(phys.astype(np.int64)).to(DEV)])
        loc_pt = np.full((1, np_i32(g["page_table"]).shape[1]), -1, np.int32)
        loc_pt[0, lst] = np.arange(len(lst))
        ro, rl = O.sparse_attention(bits(g["q"][b:b + 1]), kvb, kvb[..., :cfg.Dv], loc_pt,
                                    np.array([L], np.int32), lst.reshape(1, 1, -1),
                                    np.array([[len(lst)]]), np.zeros(cfg.Hq, np.int64), scale,
                                    cfg.page_size, rows=[(0, t, hh)])
        assert_attn_close(o[b:b + 1, t:t + 1, hh:hh + 1], lse[b:b + 1, t:t + 1, hh:hh + 1],
                          ro[:, t:t + 1, hh:hh + 1], rl[:, t:t + 1, hh:hh + 1])
