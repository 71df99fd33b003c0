"""Randomised shapes through the one-call paths, against the oracle (marked gpu).

Each case draws its shape from a seeded generator: batch, kv heads, group size,
query tokens, head dim, page size, sequence lengths (empty, one token, exact
page multiples, ragged), sink / local / budget tokens, split count (0 = the
library's default), a flat or a two-level page map, and a scale between -2 and
+3 times 1/sqrt(D).  The selection must equal the oracle's bit for bit, O and
LSE hold the 2e-3 / 1e-3 bar.  A second set appends a random number of tokens
to random sequences through the two-level map and checks pools and summaries
bit for bit.  A third draws MLA + MTP shapes (1-3 query tokens, 8-128 heads,
pages of 16-128 tokens, tier depths, ambient head counts, splits, scales)
through the tiered selection and the MLA decode, and a fourth many-row shapes
(17-159 query tokens, the tcgen05 kernel) over random page lists with the
queries at explicit positions.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import paged_sparse_kv_sa_b200 as sa
from paged_sparse_kv_sa_b200 import workloads as W
from test_gpu_parity import DEV, assert_attn_close, bits, gqa_case, np_i32, to_bf16_dev

pytestmark = pytest.mark.gpu


def _draw(rng):
    D = int(rng.choice([64, 128, 256]))
    P = int(rng.choice([16, 32, 64]))
    Hkv = int(rng.choice([1, 2, 4]))
    T = int(rng.choice([1, 2]))
    G = int(rng.choice([g for g in (1, 2, 4, 8) if T * g <= 16]))
    B = int(rng.integers(1, 5))
    lens = []
    for _ in range(B):
        kind = rng.integers(5)
        lens.append(0 if kind == 0 else 1 if kind == 1 else int(rng.integers(1, 60)) * P
                    if kind == 2 else int(rng.integers(2, 4000)))
    sink = int(rng.choice([0, 1, P, 2 * P]))
    local = int(rng.choice([0, P // 2, P, 4 * P]))
    n_sink, n_local = -(-sink // P), -(-local // P)
    budget_pages = n_sink + n_local + int(rng.integers(1, 40))
    budget = budget_pages * P + int(rng.integers(0, P))        # floor(budget / P) pages
    splits = int(rng.choice([0, 1, 2, 5]))
    if splits and -(-budget_pages // splits) > 128:
        splits = 0
    shift = int(rng.choice([-1, 0, 2, 4]))                      # -1: flat page table
    mult = float(rng.choice([-2.0, 1.0, 3.0]))
    return dict(D=D, P=P, Hkv=Hkv, G=G, T=T, B=B, lens=lens, sink=sink, local=local,
                budget=budget, splits=splits, shift=shift, mult=mult)


@pytest.mark.parametrize("seed", range(40))
def test_fuzz_step_vs_oracle(seed):
    rng = np.random.default_rng(1000 + seed)
    c = _draw(rng)
    cfg = W.GQADecode("fuzz", B=c["B"], Hq=c["Hkv"] * c["G"], Hkv=c["Hkv"], D=c["D"],
                      page_size=c["P"], seq_len_lo=0, seq_len_hi=0, sink_tokens=c["sink"],
                      local_tokens=c["local"], budget_tokens=c["budget"], T=c["T"])
    inp, g = gqa_case(cfg, seed=2000 + seed, seq_lens=c["lens"])
    pt, sl = np_i32(inp["page_table"]), np_i32(inp["seq_lens"])
    scale = c["mult"] / math.sqrt(c["D"])
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    if c["shift"] < 0:
        sig_b = O.page_summaries(bits(inp["k"]), pt, sl, c["P"])
        sig = to_bf16_dev(sig_b)
        pages, counts, o, _, lse = sa.sa_sparse_step(
            g["q"], sig, g["k"], g["v"], g["page_table"], g["seq_lens"], c["P"], c["sink"],
            c["local"], c["budget"], scale, c["splits"], dev_error=err)
        flat = pt
    else:
        page_dir, blocks = W.page_directory(inp["page_table"], inp["seq_lens"], c["P"], c["shift"],
                                            seed=seed)
        flat = O.page_table_from_dir(page_dir.numpy(), blocks.numpy(), c["shift"])
        sig_b = O.page_summaries(bits(inp["k"]), flat, sl, c["P"])
        sig = sa.sa_build_page_summaries_dir(g["k"], page_dir.to(DEV), blocks.to(DEV), c["shift"],
                                             g["seq_lens"], dev_error=err)
        torch.cuda.synchronize()
        for b, L in enumerate(c["lens"]):        # the rows the sequences reference
            used = flat[b, :-(-L // c["P"])]
            assert np.array_equal(bits(sig)[used], sig_b[used]), (c, b)
        pages, counts, o, _, lse = sa.sa_sparse_step_dir(
            g["q"], sig, g["k"], g["v"], page_dir.to(DEV), blocks.to(DEV), c["shift"],
            g["seq_lens"], c["P"], c["sink"], c["local"], c["budget"], scale, c["splits"],
            dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0, c
    rp, rc = O.select_pages(bits(inp["q"]), sig_b, flat, sl, c["P"], c["sink"], c["local"],
                            c["budget"])
    assert np.array_equal(np_i32(counts), rc), c
    assert np.array_equal(np_i32(pages), rp), c
    ro, rl = O.sparse_attention(bits(inp["q"]), bits(inp["k"]), bits(inp["v"]), flat, sl, rp, rc,
                                np.arange(cfg.Hq) // c["G"], scale, c["P"])
    assert_attn_close(o, lse, ro, rl)


@pytest.mark.parametrize("seed", range(16))
def test_fuzz_append_dir_vs_oracle(seed):
    rng = np.random.default_rng(3000 + seed)
    P = int(rng.choice([16, 32, 64]))
    D = int(rng.choice([64, 128]))
    Hkv = int(rng.choice([1, 2, 4]))
    B = int(rng.integers(1, 5))
    max_new = int(rng.integers(1, 70))
    shift = int(rng.choice([0, 1, 3]))
    lens = [int(rng.integers(0, 500)) for _ in range(B)]
    n_new = np.array([int(rng.integers(0, max_new + 1)) for _ in range(B)], dtype=np.int32)
    g = torch.Generator().manual_seed(4000 + seed)
    npg = [-(-(L + max_new) // P) for L in lens]
    pool = sum(npg) + 2
    perm = torch.randperm(pool, generator=g).numpy()
    pt = np.full((B, max(max(npg), 1)), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(npg):
        pt[b, :n] = perm[off:off + n]
        off += n
    cap = torch.tensor([n * P for n in npg], dtype=torch.int32)
    page_dir, blocks = W.page_directory(torch.from_numpy(pt), cap, P, shift, seed=seed)
    flat = O.page_table_from_dir(page_dir.numpy(), blocks.numpy(), shift)
    k = bits(torch.randn((pool, Hkv, P, D), generator=g).to(torch.bfloat16))
    v = bits(torch.randn((pool, Hkv, P, D), generator=g).to(torch.bfloat16))
    sl = np.array(lens, dtype=np.int32)
    sig = O.page_summaries(k, flat, sl, P)
    kn = bits(torch.randn((B, max_new, Hkv, D), generator=g).to(torch.bfloat16))
    vn = bits(torch.randn((B, max_new, Hkv, D), generator=g).to(torch.bfloat16))
    rk, rv, rs, rl = O.append_kv(k, v, sig, flat, sl, kn, vn, n_new, P)

    def dev(x):
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).to(DEV)
    kd, vd, sd = dev(k), dev(v), dev(sig)
    out_len = torch.full((B,), -1, dtype=torch.int32, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    sa.sa_append_kv_dir(dev(kn), dev(vn), torch.from_numpy(n_new).to(DEV), kd, vd,
                        page_dir.to(DEV), blocks.to(DEV), shift, torch.from_numpy(sl).to(DEV), sd,
                        out_seq_lens=out_len, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(bits(kd), rk) and np.array_equal(bits(vd), rv)
    assert np.array_equal(bits(sd), rs)
    assert np.array_equal(out_len.cpu().numpy(), rl)


@pytest.mark.parametrize("seed", range(16))
def test_fuzz_mla_tiers_and_decode_vs_oracle(seed):
    # MLA + MTP: tiered selection bit-exact, then the decode over the oracle's
    # tiers (critical heads: list 0; ambient heads: critical + ambient, list 1)
    rng = np.random.default_rng(5000 + seed)
    T = int(rng.choice([1, 2, 3]))
    Hq = int(rng.choice([8, 16, 32, 64, 128]))
    P = int(rng.choice([16, 32, 64, 128]))
    B = int(rng.integers(1, 4))
    L = int(rng.integers(1, 3000))
    alpha, beta = int(rng.integers(0, 9)), int(rng.integers(1, 25))
    h = int(rng.integers(1, Hq + 1))
    n_splits = int(rng.integers(1, 5))
    mult = float(rng.choice([-1.0, 1.0, 2.0]))
    cfg = W.MLADecode("fuzz", B=B, T=T, Hq=Hq, Dk=576, Dv=512, page_size=P, seq_len=L,
                      alpha=alpha, beta=beta, h_ambient=h)
    inp = W.mla_decode_inputs(cfg, seed=6000 + seed, device="cpu")
    pt, sl = np_i32(inp["page_table"]), np_i32(inp["seq_lens"])
    sig = O.page_summaries(bits(inp["kv"]), pt, sl, P)
    g = {k: (v.to(DEV) if torch.is_tensor(v) else v) for k, v in inp.items()}
    lists, counts = sa.sa_select_pages_tiered(g["q"], to_bf16_dev(sig), g["page_table"],
                                              g["seq_lens"], P, alpha, beta)
    torch.cuda.synchronize()
    lists, counts = np_i32(lists), np_i32(counts)
    crit, cc, amb, ac = O.select_pages_mla(bits(inp["q"]), sig, pt, sl, P, alpha, beta)
    cap = alpha + beta
    want = np.full((B, 2, cap), -1, dtype=np.int32)
    wc = np.zeros((B, 2), dtype=np.int32)
    for b in range(B):
        c0 = list(crit[b, :cc[b]])
        c1 = sorted(c0 + list(amb[b, :ac[b]]))
        want[b, 0, :len(c0)], want[b, 1, :len(c1)] = c0, c1
        wc[b] = len(c0), len(c1)
    assert np.array_equal(counts, wc) and np.array_equal(lists, want), (seed, L, alpha, beta)
    ambs = set(int(x) for x in inp["ambient_heads"].tolist())
    h2l = [1 if hh in ambs else 0 for hh in range(Hq)]
    scale = mult / math.sqrt(576)
    kv = g["kv"]
    o, _, lse = sa.sa_sparse_attention(g["q"], kv, kv[..., :512], g["page_table"], g["seq_lens"],
                                       torch.from_numpy(want).to(DEV), torch.from_numpy(wc).to(DEV),
                                       h2l, scale, n_splits)
    torch.cuda.synchronize()
    kvb = bits(inp["kv"])
    ro, rl = O.sparse_attention(bits(inp["q"]), kvb, kvb[..., :512], pt, sl, want, wc,
                                np.array(h2l), scale, P)
    assert_attn_close(o, lse, ro, rl)


@pytest.mark.parametrize("seed", range(8))
def test_fuzz_many_rows_at_positions_vs_oracle(seed):
    # more than 16 query rows per (list, kv head) pair -- the tcgen05 kernel --
    # over random per-group page lists, with queries at explicit positions
    rng = np.random.default_rng(7000 + seed)
    D = int(rng.choice([64, 128]))
    P = int(rng.choice([16, 32, 48, 64, 128]))   # 48: a tile of 128 keys cuts a page
    Hkv = int(rng.choice([1, 2]))
    G = int(rng.choice([1, 2, 4]))
    T = int(rng.integers(17, 160))
    B = int(rng.integers(1, 3))
    lens = [int(rng.integers(P, 2500)) for _ in range(B)]
    cfg = W.GQADecode("fuzz", B=B, Hq=Hkv * G, Hkv=Hkv, D=D, page_size=P, seq_len_lo=0,
                      seq_len_hi=0, sink_tokens=P, local_tokens=P, budget_tokens=4 * P, T=T)
    inp, g = gqa_case(cfg, seed=8000 + seed, seq_lens=lens)
    cap = int(rng.integers(1, 40))
    lists = np.full((B, Hkv, cap), -1, dtype=np.int32)
    counts = np.zeros((B, Hkv), dtype=np.int32)
    for b, L in enumerate(lens):
        n_pg = -(-L // P)
        for kvh in range(Hkv):
            k = int(rng.integers(0, min(cap, n_pg) + 1))
            sel = np.sort(rng.choice(n_pg, size=k, replace=False)).astype(np.int32)
            lists[b, kvh, :k] = sel
            counts[b, kvh] = k
    q_pos = np.array([int(rng.integers(-T // 2, L + 50)) for L in lens], dtype=np.int32)
    scale = float(rng.choice([-1.0, 1.0, 3.0])) / math.sqrt(D)
    n_splits = int(rng.integers(1, 4))
    h2l = [hh // G for hh in range(cfg.Hq)]
    o, _, lse = sa.sa_sparse_attention_at(g["q"], g["k"], g["v"], g["page_table"], g["seq_lens"],
                                          torch.from_numpy(q_pos).to(DEV),
                                          torch.from_numpy(lists).to(DEV),
                                          torch.from_numpy(counts).to(DEV), h2l, scale, n_splits)
    torch.cuda.synchronize()
    ro, rl = O.sparse_attention(bits(inp["q"]), bits(inp["k"]), bits(inp["v"]),
                                np_i32(inp["page_table"]), np_i32(inp["seq_lens"]), lists, counts,
                                np.array(h2l), scale, P, q_pos=q_pos)
    assert_attn_close(o, lse, ro, rl)
