"""CUDA path vs the float64 oracle, through the C ABI (marked gpu).

Tolerances: page selections and block tables bit-exact; summaries bit-exact;
float32 outputs max-abs 2e-3 and LSE max-abs 1e-3 against the float64 oracle
(bf16 inputs, float32 accumulation); the optional bf16 output within one bf16
ulp of RNE_bf16(oracle) plus the float32 tolerance.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import paged_sparse_kv_sa_b200 as sa
from paged_sparse_kv_sa_b200 import workloads as W

pytestmark = pytest.mark.gpu

O_TOL = 2e-3
LSE_TOL = 1e-3
DEV = "cuda"


def bits(t):
    return W.bf16_bits(t)


def np_i32(t):
    return t.detach().cpu().numpy().astype(np.int32)


def assert_attn_close(o_gpu, lse_gpu, o_ref, lse_ref):
    o_gpu = o_gpu.detach().cpu().double().numpy()
    lse_gpu = lse_gpu.detach().cpu().double().numpy()
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse_gpu), fin), "empty-row pattern differs"
    err_o = np.abs(o_gpu - o_ref).max() if o_ref.size else 0.0
    err_l = np.abs(lse_gpu[fin] - lse_ref[fin]).max() if fin.any() else 0.0
    assert err_o <= O_TOL, f"max |O - O_ref| = {err_o}"
    assert err_l <= LSE_TOL, f"max |lse - lse_ref| = {err_l}"
    assert np.all(o_gpu[~fin] == 0)


def gqa_case(cfg, seed=0, seq_lens=None):
    inp = W.gqa_decode_inputs(cfg, seed=seed, device="cpu", seq_lens=seq_lens)
    return inp, {k: (v.to(DEV) if torch.is_tensor(v) else v) for k, v in inp.items()}


def oracle_summaries(inp, cfg):
    return O.page_summaries(bits(inp["k"]), np_i32(inp["page_table"]), np_i32(inp["seq_lens"]),
                            cfg.page_size)


def to_bf16_dev(bits_np):
    return torch.from_numpy(bits_np.view(np.int16)).view(torch.bfloat16).to(DEV)


# ----------------------------------------------------------------------------
# summaries
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("lens", [None, [2048 - 5]])
def test_summaries_bitexact_tiny(lens):
    cfg = W.TINY_GQA
    inp, g = gqa_case(cfg, seed=1, seq_lens=lens)
    ref = oracle_summaries(inp, cfg)
    sig = sa.sa_build_page_summaries(g["k"], g["page_table"], g["seq_lens"])
    torch.cuda.synchronize()
    got = bits(sig)
    used = np.unique(np_i32(inp["page_table"])[np_i32(inp["page_table"]) >= 0])
    np.testing.assert_array_equal(got[used], ref[used])


def test_summaries_exact_fallback_values():
    # columns whose values span more than float64 can add exactly
    P, Hkv, D = 16, 1, 64
    k = torch.randn((3, Hkv, P, D)).to(torch.bfloat16)
    kb = bits(k).copy()
    kb[0, 0, :4, 0] = [0x7180, 0x3F80, 0xF180, 0x0001]   # 2^100, 1, -2^100, 2^-133
    kb[1, 0, :, 1] = 0x0001                              # subnormals only
    kb[2, 0, 0, 2] = 0x7F7F                              # near the top of the range
    kb[2, 0, 1:, 2] = 0x0003
    pt = np.array([[0, 1, 2]], dtype=np.int32)
    sl = np.array([3 * P - 3], dtype=np.int32)
    ref = O.page_summaries(kb, pt, sl, P)
    sig = sa.sa_build_page_summaries(to_bf16_dev(kb), torch.from_numpy(pt).to(DEV),
                                     torch.from_numpy(sl).to(DEV))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bits(sig), ref)


@pytest.mark.parametrize("n_new", [1, 3, 40])
def test_summaries_update_after_append(n_new):
    # summaries built for the shorter sequences, then updated for the pages an
    # append of n_new tokens touched: every referenced row must equal the oracle
    # for the new lengths (rows before the append are unchanged by it)
    cfg = W.scaled(W.TINY_GQA, B=3)
    lens_new = [2048 - 5, 1000, 17 + n_new]
    inp, g = gqa_case(cfg, seed=12, seq_lens=lens_new)
    sl_old = torch.tensor([max(x - n_new, 0) for x in lens_new], dtype=torch.int32, device=DEV)
    sig = sa.sa_build_page_summaries(g["k"], g["page_table"], sl_old)
    sa.sa_update_page_summaries(g["k"], g["page_table"], g["seq_lens"], sig, n_new)
    torch.cuda.synchronize()
    ref = oracle_summaries(inp, cfg)
    got = bits(sig)
    pt = np_i32(inp["page_table"])
    for b, L in enumerate(lens_new):
        used = pt[b, :-(-L // cfg.page_size)]
        np.testing.assert_array_equal(got[used], ref[used])


# ----------------------------------------------------------------------------
# selection
# ----------------------------------------------------------------------------
def run_select(g, sig_bits, cfg):
    sig = to_bf16_dev(sig_bits)
    pages, counts = sa.sa_select_pages(g["q"], sig, g["page_table"], g["seq_lens"], cfg.page_size,
                                       cfg.sink_tokens, cfg.local_tokens, cfg.budget_tokens)
    torch.cuda.synchronize()
    return np_i32(pages), np_i32(counts)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_select_bitexact_tiny(seed):
    cfg = W.TINY_GQA
    inp, g = gqa_case(cfg, seed=seed)
    sig = oracle_summaries(inp, cfg)
    pages, counts = run_select(g, sig, cfg)
    rp, rc = O.select_pages(bits(inp["q"]), sig, np_i32(inp["page_table"]), np_i32(inp["seq_lens"]),
                            cfg.page_size, cfg.sink_tokens, cfg.local_tokens, cfg.budget_tokens)
    np.testing.assert_array_equal(counts, rc)
    np.testing.assert_array_equal(pages, rp)


def test_select_ragged_mtp_and_short_sequences():
    cfg = W.scaled(W.LLAMA8B_DECODE, B=5, T=2, Hq=16, Hkv=2, seq_len_lo=0, seq_len_hi=0,
                   lift_frac=0.05, lift_sigma=3.0)
    lens = [4000, 1023, 1025, 17, 0]
    inp, g = gqa_case(cfg, seed=3, seq_lens=lens)
    sig = oracle_summaries(inp, cfg)
    pages, counts = run_select(g, sig, cfg)
    rp, rc = O.select_pages(bits(inp["q"]), sig, np_i32(inp["page_table"]), np_i32(inp["seq_lens"]),
                            cfg.page_size, cfg.sink_tokens, cfg.local_tokens, cfg.budget_tokens)
    np.testing.assert_array_equal(counts, rc)
    np.testing.assert_array_equal(pages, rp)


def test_select_ties_and_cancellation():
    cfg = W.scaled(W.TINY_GQA, B=3)
    inp, g = gqa_case(cfg, seed=4)
    sig = oracle_summaries(inp, cfg).copy()
    pt = np_i32(inp["page_table"])
    qb = bits(inp["q"]).copy()
    qb[0] = 0                                        # sequence 0: every score is 0
    sig[pt[1, 40]] = sig[pt[1, 41]]                  # sequence 1: duplicated summaries
    sig[pt[1, 42]] = sig[pt[1, 41]]
    # sequence 2: a page whose exact score needs cancellation-free summation
    sig[pt[2, 50], :, :] = 0
    sig[pt[2, 50], :, 0] = 0x7180
    sig[pt[2, 50], :, 1] = 0x7180
    qb[2, 0, :, 0] = 0x3F80
    qb[2, 0, :, 1] = 0xBF80
    qb[2, 0, :, 2] = 0x4000
    sig[pt[2, 50], :, 2] = 0x4480                    # 2 * 1024 = 2048 exactly
    g["q"] = to_bf16_dev(qb)
    pages, counts = run_select(g, sig, cfg)
    rp, rc = O.select_pages(qb, sig, pt, np_i32(inp["seq_lens"]), cfg.page_size, cfg.sink_tokens,
                            cfg.local_tokens, cfg.budget_tokens)
    np.testing.assert_array_equal(counts, rc)
    np.testing.assert_array_equal(pages, rp)
    assert list(rp[0, 0, :12]) == list(range(12))   # ties -> lowest pages after the 2 sinks


def test_select_long_all_ties():
    # one long sequence whose scores all tie (q = 0): more equal candidates than
    # the selector's threshold filter keeps, so its radix path decides; the
    # winners are the lowest candidate pages
    cfg = W.scaled(W.TINY_GQA, B=2, seq_len_lo=40000, seq_len_hi=40000)
    inp, g = gqa_case(cfg, seed=6)
    sig = oracle_summaries(inp, cfg)
    qb = bits(inp["q"]).copy()
    qb[1] = 0
    g["q"] = to_bf16_dev(qb)
    pages, counts = run_select(g, sig, cfg)
    rp, rc = O.select_pages(qb, sig, np_i32(inp["page_table"]), np_i32(inp["seq_lens"]),
                            cfg.page_size, cfg.sink_tokens, cfg.local_tokens, cfg.budget_tokens)
    np.testing.assert_array_equal(counts, rc)
    np.testing.assert_array_equal(pages, rp)
    n_sink, _, _, k = O.page_budget(cfg.sink_tokens, cfg.local_tokens, cfg.budget_tokens,
                                    cfg.page_size)
    assert list(rp[1, 0, :n_sink + k]) == list(range(n_sink + k))


def test_select_deep_budget():
    # 403 top-k slots over 966 candidate pages: deeper than the threshold pruning
    # covers, so every candidate is classified by counting
    cfg = W.scaled(W.LLAMA8B_DECODE, B=2, Hq=8, Hkv=2, seq_len_lo=16000, seq_len_hi=16000,
                   budget_tokens=7000)
    inp, g = gqa_case(cfg, seed=8)
    sig = oracle_summaries(inp, cfg)
    pages, counts = run_select(g, sig, cfg)
    rp, rc = O.select_pages(bits(inp["q"]), sig, np_i32(inp["page_table"]), np_i32(inp["seq_lens"]),
                            cfg.page_size, cfg.sink_tokens, cfg.local_tokens, cfg.budget_tokens)
    np.testing.assert_array_equal(counts, rc)
    np.testing.assert_array_equal(pages, rp)


def test_select_workspace_contents_do_not_matter():
    # The selection workspace has no initial contents to rely on: a workspace
    # full of random bytes, reused over several calls, gives the oracle's
    # selection every time.
    cfg = W.scaled(W.LLAMA8B_DECODE, B=3, seq_len_lo=8192, seq_len_hi=8192)
    inp, g = gqa_case(cfg, seed=21)
    sig = oracle_summaries(inp, cfg)
    rp, rc = O.select_pages(bits(inp["q"]), sig, np_i32(inp["page_table"]), np_i32(inp["seq_lens"]),
                            cfg.page_size, cfg.sink_tokens, cfg.local_tokens, cfg.budget_tokens)
    max_pages = g["page_table"].shape[1]
    n = sa.sa_select_workspace_size(cfg.B, cfg.Hkv, max_pages)
    gen = torch.Generator(device=DEV)
    gen.manual_seed(5)
    ws = torch.randint(0, 256, (n,), dtype=torch.uint8, device=DEV, generator=gen)
    sigd = to_bf16_dev(sig)
    for _ in range(3):
        pages, counts = sa.sa_select_pages(g["q"], sigd, g["page_table"], g["seq_lens"],
                                           cfg.page_size, cfg.sink_tokens, cfg.local_tokens,
                                           cfg.budget_tokens, workspace=ws)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(np_i32(counts), rc)
        np.testing.assert_array_equal(np_i32(pages), rp)


@pytest.mark.parametrize("D,T", [(128, 1), (64, 2)])
def test_select_eight_kv_heads_ragged(D, T):
    # Hkv = 8 (one scoring CTA covers all kv heads of a page): a long sequence
    # (16 scoring chunks), one of a single chunk, one shorter than the budget
    # (nothing to rank) and a ragged one, in the same call.
    cfg = W.scaled(W.LLAMA8B_DECODE, B=4, Hq=16 if T == 2 else 32, Hkv=8, D=D, T=T,
                   seq_len_lo=0, seq_len_hi=0)
    lens = [32768 - 7, 1100, 700, 9000 + 5]
    inp, g = gqa_case(cfg, seed=40 + D, seq_lens=lens)
    sig = oracle_summaries(inp, cfg)
    pages, counts = run_select(g, sig, cfg)
    rp, rc = O.select_pages(bits(inp["q"]), sig, np_i32(inp["page_table"]), np_i32(inp["seq_lens"]),
                            cfg.page_size, cfg.sink_tokens, cfg.local_tokens, cfg.budget_tokens)
    np.testing.assert_array_equal(counts, rc)
    np.testing.assert_array_equal(pages, rp)


def test_select_eight_kv_heads_ties():
    # Hkv = 8 and all scores of one sequence tie (q = 0): resolved by the
    # lowest logical pages
    cfg = W.scaled(W.LLAMA8B_DECODE, B=2, seq_len_lo=8192, seq_len_hi=8192)
    inp, g = gqa_case(cfg, seed=44)
    sig = oracle_summaries(inp, cfg)
    qb = bits(inp["q"]).copy()
    qb[1] = 0
    g["q"] = to_bf16_dev(qb)
    pages, counts = run_select(g, sig, cfg)
    rp, rc = O.select_pages(qb, sig, np_i32(inp["page_table"]), np_i32(inp["seq_lens"]),
                            cfg.page_size, cfg.sink_tokens, cfg.local_tokens, cfg.budget_tokens)
    np.testing.assert_array_equal(counts, rc)
    np.testing.assert_array_equal(pages, rp)


def _random_bf16_bits(rng, shape, e_lo, e_hi, p_sub=0.03, p_zero=0.03):
    """bf16 bit patterns: random sign and fraction, exponent field uniform in
    [e_lo, e_hi]; a share of subnormals and zeros."""
    sign = rng.integers(0, 2, shape, dtype=np.uint16) << 15
    frac = rng.integers(0, 128, shape, dtype=np.uint16)
    expo = rng.integers(e_lo, e_hi + 1, shape, dtype=np.uint16)
    out = sign | (expo << 7) | frac
    u = rng.random(shape)
    out = np.where(u < p_sub, sign | np.maximum(frac, 1).astype(np.uint16), out)
    out = np.where((u >= p_sub) & (u < p_sub + p_zero), sign, out)
    return out.astype(np.uint16)


@pytest.mark.parametrize("T,Hq,Hkv", [(1, 8, 2), (2, 16, 2)])
def test_select_score_brackets_hold(T, Hq, Hkv):
    # The selector's per-page score brackets (its workspace) must contain the
    # exact row-max score for every candidate page, on inputs with a wide
    # exponent range, subnormals and zeros; the selection must equal the oracle's.
    cfg = W.scaled(W.TINY_GQA, B=2, T=T, Hq=Hq, Hkv=Hkv, D=128)
    inp, g = gqa_case(cfg, seed=11)
    rng = np.random.default_rng(11)
    pt = np_i32(inp["page_table"])
    sl = np_i32(inp["seq_lens"])
    qb = _random_bf16_bits(rng, tuple(inp["q"].shape), 112, 136)
    sig = _random_bf16_bits(rng, (int(pt.max()) + 1, Hkv, cfg.D), 100, 146)
    g["q"] = to_bf16_dev(qb)
    max_pages = pt.shape[1]
    ws = torch.zeros(sa.sa_select_workspace_size(cfg.B, Hkv, max_pages), dtype=torch.uint8,
                     device=DEV)
    pages, counts = sa.sa_select_pages(g["q"], to_bf16_dev(sig), g["page_table"], g["seq_lens"],
                                       cfg.page_size, cfg.sink_tokens, cfg.local_tokens,
                                       cfg.budget_tokens, workspace=ws)
    torch.cuda.synchronize()
    n_bounds = cfg.B * Hkv * max_pages * 2
    lohi = (ws.view(torch.float32)[:n_bounds].cpu().numpy()
            .reshape(cfg.B, Hkv, max_pages, 2).astype(np.float64))
    n_sink, n_local, budget_pages, _ = O.page_budget(cfg.sink_tokens, cfg.local_tokens,
                                                     cfg.budget_tokens, cfg.page_size)
    q = O.bf16_to_f64(qb)
    G = Hq // Hkv
    checked = 0
    for b in range(cfg.B):
        nb = -(-int(sl[b]) // cfg.page_size)
        cand = np.arange(n_sink, nb - n_local)
        for kvh in range(Hkv):
            rows = q[b, :, kvh * G:(kvh + 1) * G, :].reshape(T * G, cfg.D)
            ex = O.page_scores(rows, O.bf16_to_f64(sig[pt[b, cand], kvh, :]))
            lo, hi = lohi[b, kvh, cand, 0], lohi[b, kvh, cand, 1]
            assert np.all(lo <= ex) and np.all(ex <= hi), "score bracket misses the exact score"
            checked += len(cand)
    assert checked > 0
    rp, rc = O.select_pages(qb, sig, pt, sl, cfg.page_size, cfg.sink_tokens, cfg.local_tokens,
                            cfg.budget_tokens)
    np.testing.assert_array_equal(np_i32(counts), rc)
    np.testing.assert_array_equal(np_i32(pages), rp)


def test_select_streaming_k0():
    cfg = W.scaled(W.TINY_GQA, budget_tokens=96)    # 2 sink + 4 local, no top-k
    inp, g = gqa_case(cfg, seed=5)
    sig = oracle_summaries(inp, cfg)
    pages, counts = run_select(g, sig, cfg)
    assert list(pages[0, 0, :counts[0, 0]]) == [0, 1, 124, 125, 126, 127]


# ----------------------------------------------------------------------------
# decode + combine
# ----------------------------------------------------------------------------
def oracle_lists(inp, cfg, sig):
    return O.select_pages(bits(inp["q"]), sig, np_i32(inp["page_table"]), np_i32(inp["seq_lens"]),
                          cfg.page_size, cfg.sink_tokens, cfg.local_tokens, cfg.budget_tokens)


def run_decode(g, lists, counts, cfg, n_splits, k=None, v=None, h2l=None):
    Hq, Hkv = cfg.Hq, cfg.Hkv
    h2l = [h // (Hq // Hkv) for h in range(Hq)] if h2l is None else h2l
    o_p, l_p = sa.sa_sparse_decode(g["q"], g["k"] if k is None else k, g["v"] if v is None else v,
                                   g["page_table"], g["seq_lens"],
                                   torch.from_numpy(lists).to(DEV), torch.from_numpy(counts).to(DEV),
                                   h2l, 1.0 / math.sqrt(cfg.D), n_splits)
    o, ob, lse = sa.sa_combine(o_p, l_p)
    torch.cuda.synchronize()
    return o, lse


@pytest.mark.parametrize("n_splits", [1, 3])
def test_decode_tiny_vs_oracle(n_splits):
    cfg = W.TINY_GQA
    inp, g = gqa_case(cfg, seed=0)
    sig = oracle_summaries(inp, cfg)
    lists, counts = oracle_lists(inp, cfg, sig)
    o, lse = run_decode(g, lists, counts, cfg, n_splits)
    h2l = np.arange(cfg.Hq) // cfg.G
    ro, rl = O.sparse_attention(bits(inp["q"]), bits(inp["k"]), bits(inp["v"]),
                                np_i32(inp["page_table"]), np_i32(inp["seq_lens"]), lists, counts,
                                h2l, 1.0 / math.sqrt(cfg.D), cfg.page_size)
    assert_attn_close(o, lse, ro, rl)


@pytest.mark.parametrize("D,P,T", [(128, 16, 1), (128, 16, 2), (64, 32, 2), (256, 16, 1),
                                   (128, 64, 1)])
def test_decode_shapes_ragged_vs_oracle(D, P, T):
    cfg = W.GQADecode("case", B=3, Hq=8, Hkv=2, D=D, page_size=P, seq_len_lo=0, seq_len_hi=0,
                      sink_tokens=P, local_tokens=2 * P, budget_tokens=12 * P, T=T)
    lens = [50 * P + 7, 9 * P, 3 * P + 1]
    inp, g = gqa_case(cfg, seed=6, seq_lens=lens)
    sig = oracle_summaries(inp, cfg)
    lists, counts = oracle_lists(inp, cfg, sig)
    o, lse = run_decode(g, lists, counts, cfg, 2)
    ro, rl = O.sparse_attention(bits(inp["q"]), bits(inp["k"]), bits(inp["v"]),
                                np_i32(inp["page_table"]), np_i32(inp["seq_lens"]), lists, counts,
                                np.arange(cfg.Hq) // cfg.G, 1.0 / math.sqrt(D), P)
    assert_attn_close(o, lse, ro, rl)


def test_decode_per_head_lists_and_empty():
    # QK 2D sparsity: heads of one kv group read different lists; one list empty
    cfg = W.GQADecode("case", B=2, Hq=8, Hkv=2, D=128, page_size=16, seq_len_lo=0, seq_len_hi=0,
                      sink_tokens=16, local_tokens=16, budget_tokens=160)
    inp, g = gqa_case(cfg, seed=7, seq_lens=[700, 333])
    rng = np.random.default_rng(7)
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
    o, lse = run_decode(g, lists, counts, cfg, 2, h2l=h2l)
    ro, rl = O.sparse_attention(bits(inp["q"]), bits(inp["k"]), bits(inp["v"]),
                                np_i32(inp["page_table"]), np_i32(inp["seq_lens"]), lists, counts,
                                np.array(h2l), 1.0 / math.sqrt(128), 16)
    assert_attn_close(o, lse, ro, rl)


def test_decode_strided_cache_layout():
    # the pool stored as [P_pool, P, Hkv, D] (vLLM order) and viewed through strides
    cfg = W.scaled(W.TINY_GQA, B=2, seq_len_lo=1500, seq_len_hi=1500)
    inp, g = gqa_case(cfg, seed=8)
    sig = oracle_summaries(inp, cfg)
    lists, counts = oracle_lists(inp, cfg, sig)
    k_alt = g["k"].permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
    v_alt = g["v"].permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
    assert k_alt.stride() != g["k"].stride()
    o, lse = run_decode(g, lists, counts, cfg, 2, k=k_alt, v=v_alt)
    ro, rl = O.sparse_attention(bits(inp["q"]), bits(inp["k"]), bits(inp["v"]),
                                np_i32(inp["page_table"]), np_i32(inp["seq_lens"]), lists, counts,
                                np.arange(cfg.Hq) // cfg.G, 1.0 / math.sqrt(cfg.D), cfg.page_size)
    assert_attn_close(o, lse, ro, rl)


def test_decode_bad_pages_flagged_not_trapped():
    cfg = W.scaled(W.TINY_GQA, B=1)
    inp, g = gqa_case(cfg, seed=9)
    lists = np.array([[[0, 1, 5000, -3], [2, 3, 4, 5]]], dtype=np.int32)
    counts = np.array([[4, 4]], dtype=np.int32)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    o_p, l_p = sa.sa_sparse_decode(g["q"], g["k"], g["v"], g["page_table"], g["seq_lens"],
                                   torch.from_numpy(lists).to(DEV), torch.from_numpy(counts).to(DEV),
                                   [0, 0, 0, 0, 1, 1, 1, 1], 0.125, 1, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) & 1          # SA_DEVERR_PAGE_RANGE
    ok = np.array([[[0, 1, -1, -1], [2, 3, 4, 5]]], dtype=np.int32)
    ro, rl = O.sparse_attention(bits(inp["q"]), bits(inp["k"]), bits(inp["v"]),
                                np_i32(inp["page_table"]), np_i32(inp["seq_lens"]), ok,
                                np.array([[2, 4]]), [0, 0, 0, 0, 1, 1, 1, 1], 0.125, 16)
    assert_attn_close(o_p[0], l_p[0], ro, rl)


def test_combine_vs_oracle():
    rng = np.random.default_rng(11)
    S, rows, Dv = 5, 37, 128
    o = rng.standard_normal((S, rows, Dv)).astype(np.float32)
    lse = (rng.standard_normal((S, rows)) * 3).astype(np.float32)
    lse[1, :10] = -np.inf
    lse[:, 20] = -np.inf                       # a row with every split empty
    o[:, 20] = 0
    ob = torch.empty((rows, Dv), dtype=torch.bfloat16, device=DEV)
    go, _, gl = sa.sa_combine(torch.from_numpy(o).to(DEV), torch.from_numpy(lse).to(DEV),
                              o_out_bf16=ob)
    torch.cuda.synchronize()
    ro, rl = O.combine(o.astype(np.float64), lse.astype(np.float64))
    assert_attn_close(go, gl, ro, rl)
    rb = O.bf16_to_f64(O.f64_to_bf16_rne(ro))
    err = np.abs(ob.float().cpu().numpy() - rb)
    assert np.all(err <= np.abs(rb) * 2.0 ** -7 + O_TOL)


# ----------------------------------------------------------------------------
# block union
# ----------------------------------------------------------------------------
def test_block_union_small_bitexact():
    Hq, Hkv, NQB, off, top_k = 8, 2, 6, 40, 5
    s = torch.randn((Hq, NQB, off + NQB), generator=torch.Generator().manual_seed(3))
    s[0, 2, 10] = s[0, 2, 11]
    tables, counts = sa.sa_block_union(s.to(DEV), Hkv, off, top_k)
    torch.cuda.synchronize()
    rt, rc = O.block_union(s.numpy(), Hkv, off, top_k)
    np.testing.assert_array_equal(np_i32(counts), rc)
    np.testing.assert_array_equal(np_i32(tables), rt)


@pytest.mark.slow
def test_block_union_full_size_sampled():
    cfg = W.UNION_PREFILL
    s = W.block_union_scores(cfg, seed=0, device="cpu")
    off = cfg.q_offset // cfg.block
    tables, counts = sa.sa_block_union(s.to(DEV), cfg.Hkv, off, cfg.top_k)
    torch.cuda.synchronize()
    t, c = np_i32(tables), np_i32(counts)
    G = cfg.Hq // cfg.Hkv
    rng = np.random.default_rng(0)
    for g in range(cfg.Hkv):
        row = t[g, :c[g]]
        assert np.all(np.diff(row) > 0) and np.all(t[g, c[g]:] == -1)
    # every sampled (head, Q-block) mask lies inside its group's table
    sn = s.numpy()
    for _ in range(24):
        h, j = int(rng.integers(cfg.Hq)), int(rng.integers(cfg.n_q_blocks))
        d = off + j
        cand = np.arange(1, d)
        win = O.rank_select(sn[h, j, cand].astype(np.float64), cand, cfg.top_k)
        mask = {0, d} | set(cand[win].tolist())
        assert mask <= set(t[h // G, :c[h // G]].tolist())
    # exact equality on two full groups, recomputed by the oracle
    rt, rc = O.block_union(sn[:2 * G], 2, off, cfg.top_k)
    np.testing.assert_array_equal(c[:2], rc)
    np.testing.assert_array_equal(t[:2], rt)


# ----------------------------------------------------------------------------
# many query rows per pair: the tcgen05 path (chunked prefill, long MTP)
# ----------------------------------------------------------------------------
def prefill_case(seed, T, q_off, P, Hq=8, Hkv=2, D=128, top_k=3, n_sink=1, ragged=0):
    """Chunk of T queries at q_off over a KV of q_off + T - ragged tokens, block-union
    tables (64-token blocks) from random block scores, expressed as lists of P-token
    pages (a block of 64 tokens = 64 / P pages)."""
    g = torch.Generator().manual_seed(seed)
    L = q_off + T - ragged
    nkb = -(-L // 64)
    nqb = -(-T // 64)
    qb_off = q_off // 64
    scores = torch.randn((Hq, nqb, nkb), generator=g)
    tables, counts = O.block_union(scores.numpy(), Hkv, qb_off, top_k, n_sink)
    per = 64 // P if P <= 64 else 1
    npg = -(-L // P)
    lists = np.full((1, Hkv, nkb * per), -1, dtype=np.int32)
    cnt = np.zeros((1, Hkv), dtype=np.int32)
    for h in range(Hkv):
        pages = []
        for blk in tables[h, :counts[h]]:
            if P <= 64:
                pages += [p for p in range(blk * per, blk * per + per) if p < npg]
            else:
                if blk * 64 // P not in pages:
                    pages.append(blk * 64 // P)
        lists[0, h, :len(pages)] = pages
        cnt[0, h] = len(pages)
    q = torch.randn((1, T, Hq, D), generator=g).to(torch.bfloat16)
    perm = torch.randperm(npg, generator=g)
    k = torch.randn((npg, Hkv, P, D), generator=g).to(torch.bfloat16)
    v = torch.randn((npg, Hkv, P, D), generator=g).to(torch.bfloat16)
    pt = perm.to(torch.int32).reshape(1, npg)
    sl = torch.tensor([L], dtype=torch.int32)
    return q, k, v, pt, sl, lists, cnt


@pytest.mark.parametrize("T,q_off,P,n_splits,ragged", [(64, 640, 64, 1, 0), (96, 448, 64, 2, 0),
                                                       (8, 700, 16, 1, 5), (40, 1000, 32, 3, 17)])
def test_prefill_tcgen05_vs_oracle(T, q_off, P, n_splits, ragged):
    q, k, v, pt, sl, lists, cnt = prefill_case(1, T, q_off, P, ragged=ragged)
    Hq, Hkv, D = q.shape[2], k.shape[1], q.shape[3]
    h2l = [h // (Hq // Hkv) for h in range(Hq)]
    o_p, l_p = sa.sa_sparse_decode(q.to(DEV), k.to(DEV), v.to(DEV), pt.to(DEV), sl.to(DEV),
                                   torch.from_numpy(lists).to(DEV), torch.from_numpy(cnt).to(DEV),
                                   h2l, 1.0 / math.sqrt(D), n_splits)
    o, _, lse = sa.sa_combine(o_p, l_p)
    torch.cuda.synchronize()
    ro, rl = O.sparse_attention(bits(q), bits(k), bits(v), np_i32(pt), np_i32(sl), lists, cnt,
                                np.array(h2l), 1.0 / math.sqrt(D), P)
    assert_attn_close(o, lse, ro, rl)


@pytest.mark.parametrize("mult", [3.0, 8.0, -3.0])
@pytest.mark.parametrize("T,q_off,P,n_splits,ragged", [(96, 448, 64, 2, 0), (40, 1000, 32, 3, 17)])
def test_prefill_tcgen05_sharp_scales(T, q_off, P, n_splits, ragged, mult):
    # a few keys dominate every row: P's rounding before the PV product shows in O
    # directly (P enters as a bf16 pair hi + lo); a negative scale flips the row max
    q, k, v, pt, sl, lists, cnt = prefill_case(2, T, q_off, P, ragged=ragged)
    Hq, Hkv, D = q.shape[2], k.shape[1], q.shape[3]
    h2l = [h // (Hq // Hkv) for h in range(Hq)]
    scale = mult / math.sqrt(D)
    o_p, l_p = sa.sa_sparse_decode(q.to(DEV), k.to(DEV), v.to(DEV), pt.to(DEV), sl.to(DEV),
                                   torch.from_numpy(lists).to(DEV), torch.from_numpy(cnt).to(DEV),
                                   h2l, scale, n_splits)
    o, _, lse = sa.sa_combine(o_p, l_p)
    torch.cuda.synchronize()
    ro, rl = O.sparse_attention(bits(q), bits(k), bits(v), np_i32(pt), np_i32(sl), lists, cnt,
                                np.array(h2l), scale, P)
    assert_attn_close(o, lse, ro, rl)


@pytest.mark.slow
@pytest.mark.parametrize("mult", [1.0, 3.0])
def test_prefill_full_size_sampled_rows(mult):
    cfg = W.UNION_PREFILL
    s = W.block_union_scores(cfg, seed=0, device=DEV)
    inp = W.prefill_inputs(cfg, seed=0, device=DEV)
    off = cfg.q_offset // cfg.block
    tables, counts = sa.sa_block_union(s, cfg.Hkv, off, cfg.top_k)
    h2l = [h // (cfg.Hq // cfg.Hkv) for h in range(cfg.Hq)]
    o_p, l_p = sa.sa_sparse_decode(inp["q"], inp["k"], inp["v"], inp["page_table"],
                                   inp["seq_lens"], tables.view(1, cfg.Hkv, -1).contiguous(),
                                   counts.view(1, cfg.Hkv).contiguous(), h2l,
                                   mult / math.sqrt(cfg.D), 2)
    o, _, lse = sa.sa_combine(o_p, l_p)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    ts = sorted(set(rng.integers(0, cfg.chunk, 12).tolist()) | {0, cfg.chunk - 1})
    rows = [(0, t, int(h)) for t in ts for h in rng.integers(0, cfg.Hq, 3)]
    tb = np_i32(tables).reshape(1, cfg.Hkv, -1)
    cb = np_i32(counts).reshape(1, cfg.Hkv)
    ro, rl = O.sparse_attention(bits(inp["q"]), bits(inp["k"]), bits(inp["v"]),
                                np_i32(inp["page_table"]), np_i32(inp["seq_lens"]), tb, cb,
                                np.array(h2l), mult / math.sqrt(cfg.D), cfg.block, rows=rows)
    og = o.cpu().double().numpy()
    lg = lse.cpu().double().numpy()
    for (b, t, h) in rows:
        assert np.abs(og[b, t, h] - ro[b, t, h]).max() <= O_TOL, (t, h)
        assert abs(lg[b, t, h] - rl[b, t, h]) <= LSE_TOL, (t, h)


# ----------------------------------------------------------------------------
# tiered (critical / ambient) selection for one latent head
# ----------------------------------------------------------------------------
def tiered_case(seed, B, T, Hq, Dk, P, L, alpha, beta):
    cfg = W.MLADecode("case", B=B, T=T, Hq=Hq, Dk=Dk, Dv=Dk - 64, page_size=P, seq_len=L,
                      alpha=alpha, beta=beta, h_ambient=max(1, Hq // 4))
    inp = W.mla_decode_inputs(cfg, seed=seed, device="cpu")
    sig = O.page_summaries(bits(inp["kv"]), np_i32(inp["page_table"]), np_i32(inp["seq_lens"]), P)
    return cfg, inp, sig


def check_tiered(cfg, inp, sig, units=None):
    g = {k: (v.to(DEV) if torch.is_tensor(v) else v) for k, v in inp.items()}
    lists, counts = sa.sa_select_pages_tiered(g["q"], to_bf16_dev(sig), g["page_table"],
                                              g["seq_lens"], cfg.page_size, cfg.alpha, cfg.beta)
    torch.cuda.synchronize()
    lists, counts = np_i32(lists), np_i32(counts)
    crit, cc, amb, ac = O.select_pages_mla(bits(inp["q"]), sig, np_i32(inp["page_table"]),
                                           np_i32(inp["seq_lens"]), cfg.page_size, cfg.alpha,
                                           cfg.beta, units=units)
    for b in (range(cfg.B) if units is None else units):
        want0 = list(crit[b, :cc[b]])
        want1 = sorted(want0 + list(amb[b, :ac[b]]))
        assert counts[b, 0] == len(want0) and counts[b, 1] == len(want1)
        assert list(lists[b, 0, :counts[b, 0]]) == want0
        assert list(lists[b, 1, :counts[b, 1]]) == want1
        assert np.all(lists[b, 0, counts[b, 0]:] == -1) and np.all(lists[b, 1, counts[b, 1]:] == -1)


@pytest.mark.parametrize("seed,L", [(0, 40 * 16 - 3), (1, 9 * 16), (2, 5 * 16)])
def test_select_tiered_small(seed, L):
    cfg, inp, sig = tiered_case(seed, B=2, T=2, Hq=16, Dk=576, P=16, L=L, alpha=3, beta=5)
    check_tiered(cfg, inp, sig)


@pytest.mark.parametrize("alpha,beta,n_pages,Dk", [(0, 12, 200, 576), (100, 200, 400, 128),
                                                   (5, 35, 3000, 128)])
def test_select_tiered_depths(alpha, beta, n_pages, Dk):
    """No critical tier; a boundary deeper than the threshold pruning covers (every page
    classified by counting); several thousand pages (several pages per thread)."""
    cfg, inp, sig = tiered_case(11, B=2, T=2, Hq=16, Dk=Dk, P=16, L=n_pages * 16 - 7,
                                alpha=alpha, beta=beta)
    check_tiered(cfg, inp, sig)


def test_select_tiered_max_pages_limit():
    """The widest page table the tiered selection takes (8192 pages: its choose pass keeps
    21 bytes per page in shared memory) runs and matches; one page wider is refused."""
    cfg, inp, sig = tiered_case(5, B=1, T=1, Hq=8, Dk=64, P=16, L=8192 * 16, alpha=4, beta=28)
    assert inp["page_table"].shape[1] == 8192
    check_tiered(cfg, inp, sig)
    g = {k: (v.to(DEV) if torch.is_tensor(v) else v) for k, v in inp.items()}
    wide = torch.cat([g["page_table"], torch.full((1, 1), -1, dtype=torch.int32, device=DEV)], 1)
    with pytest.raises(sa.SAError, match="UNSUPPORTED"):
        sa.sa_select_pages_tiered(g["q"], to_bf16_dev(sig), wide, g["seq_lens"], cfg.page_size,
                                  cfg.alpha, cfg.beta)


def test_select_tiered_ties():
    cfg, inp, sig = tiered_case(3, B=2, T=1, Hq=8, Dk=128, P=16, L=30 * 16, alpha=2, beta=4)
    inp["q"][0] = 0                                     # all scores tie: lowest pages
    sig = sig.copy()
    pt = np_i32(inp["page_table"])
    sig[pt[1, 7]] = sig[pt[1, 9]]                       # duplicated summaries
    check_tiered(cfg, inp, sig)


@pytest.mark.parametrize("Dk", [576, 136])
def test_select_tiered_brackets_and_row_masks(Dk):
    # The tiered scorer's workspace: per (sequence, 32-row group, page) a float32
    # bracket that must contain the exact row-group maximum, and a row mask that
    # must flag every row attaining it; wide exponents, subnormals and zeros.
    # Dk = 136 exercises the zero-padded last 16-feature step.
    cfg, inp, _ = tiered_case(7, B=2, T=2, Hq=64, Dk=Dk, P=16, L=70 * 16 - 5, alpha=3, beta=6)
    rng = np.random.default_rng(7)
    pt = np_i32(inp["page_table"])
    sl = np_i32(inp["seq_lens"])
    qb = _random_bf16_bits(rng, tuple(inp["q"].shape), 114, 136)
    sig = _random_bf16_bits(rng, (int(pt.max()) + 1, 1, Dk), 104, 144)
    max_pages = pt.shape[1]
    nbytes = sa.load().sa_select_tiered_workspace_size(cfg.B, cfg.T, cfg.Hq, max_pages)
    ws = torch.zeros(int(nbytes), dtype=torch.uint8, device=DEV)
    lists, counts = sa.sa_select_pages_tiered(to_bf16_dev(qb), to_bf16_dev(sig),
                                              inp["page_table"].to(DEV), inp["seq_lens"].to(DEV),
                                              cfg.page_size, cfg.alpha, cfg.beta, workspace=ws)
    torch.cuda.synchronize()
    R = cfg.T * cfg.Hq
    RG = 32                                   # query rows per scoring group
    n_rg = -(-R // RG)
    raw = ws.cpu().numpy()
    nl = cfg.B * n_rg * max_pages
    lohi = raw[:nl * 8].view(np.float32).reshape(cfg.B, n_rg, max_pages, 2).astype(np.float64)
    masks = raw[nl * 8:nl * 16].view(np.uint64).reshape(cfg.B, n_rg, max_pages)
    q = O.bf16_to_f64(qb)
    for b in range(cfg.B):
        nb = -(-int(sl[b]) // cfg.page_size)
        rows = q[b].reshape(R, Dk)
        ex = O.exact_dots(rows, O.bf16_to_f64(sig[pt[b, :nb], 0, :]))   # [R, nb]
        for g in range(n_rg):
            eg = ex[g * RG:(g + 1) * RG]
            gmax = eg.max(axis=0)
            lo, hi = lohi[b, g, :nb, 0], lohi[b, g, :nb, 1]
            assert np.all(lo <= gmax) and np.all(gmax <= hi), "bracket misses the group maximum"
            for p in range(nb):
                arg = np.flatnonzero(eg[:, p] == gmax[p])
                m = int(masks[b, g, p])
                assert all((m >> int(r)) & 1 for r in arg), "a maximising row is not flagged"
    # and the selection itself
    crit, cc, amb, ac = O.select_pages_mla(qb, sig, pt, sl, cfg.page_size, cfg.alpha, cfg.beta)
    lists, counts = np_i32(lists), np_i32(counts)
    for b in range(cfg.B):
        want0 = list(crit[b, :cc[b]])
        assert list(lists[b, 0, :counts[b, 0]]) == want0
        assert list(lists[b, 1, :counts[b, 1]]) == sorted(want0 + list(amb[b, :ac[b]]))


@pytest.mark.slow
def test_select_tiered_mla_workload_sampled():
    cfg = W.MLA_MTP
    inp = W.mla_decode_inputs(cfg, seed=0, device="cpu")
    n = cfg.seq_len // cfg.page_size
    units = [(b, p) for b in (0, 5) for p in range(n)]
    sig = O.page_summaries(bits(inp["kv"]), np_i32(inp["page_table"]), np_i32(inp["seq_lens"]),
                           cfg.page_size, units=units)
    check_tiered(cfg, inp, sig, units=[0, 5])


# ----------------------------------------------------------------------------
# MLA + MTP tiered decode (tcgen05, V = first 512 key columns)
# ----------------------------------------------------------------------------
def mla_lists_from_oracle(inp, sig, cfg, units=None):
    crit, cc, amb, ac = O.select_pages_mla(bits(inp["q"]), sig, np_i32(inp["page_table"]),
                                           np_i32(inp["seq_lens"]), cfg.page_size, cfg.alpha,
                                           cfg.beta, units=units)
    cap = cfg.alpha + cfg.beta
    lists = np.full((cfg.B, 2, cap), -1, dtype=np.int32)
    counts = np.zeros((cfg.B, 2), dtype=np.int32)
    for b in range(cfg.B):
        c0 = list(crit[b, :cc[b]])
        c1 = sorted(c0 + list(amb[b, :ac[b]]))
        lists[b, 0, :len(c0)] = c0
        lists[b, 1, :len(c1)] = c1
        counts[b] = (len(c0), len(c1))
    return lists, counts


def run_mla(inp, cfg, lists, counts, n_splits):
    g = {k: (v.to(DEV) if torch.is_tensor(v) else v) for k, v in inp.items()}
    amb = set(int(h) for h in inp["ambient_heads"].tolist())
    h2l = [1 if h in amb else 0 for h in range(cfg.Hq)]
    kv = g["kv"]
    o_p, l_p = sa.sa_sparse_decode(g["q"], kv, kv[..., :cfg.Dv], g["page_table"], g["seq_lens"],
                                   torch.from_numpy(lists).to(DEV),
                                   torch.from_numpy(counts).to(DEV), h2l,
                                   1.0 / math.sqrt(cfg.Dk), n_splits)
    o, _, lse = sa.sa_combine(o_p, l_p)
    torch.cuda.synchronize()
    return o, lse, h2l


@pytest.mark.parametrize("seed,L,n_splits", [(0, 2500, 1), (1, 2500, 3), (2, 700, 2)])
def test_mla_decode_vs_oracle(seed, L, n_splits):
    cfg = W.MLADecode("case", B=2, T=2, Hq=16, Dk=576, Dv=512, page_size=64, seq_len=L,
                      alpha=3, beta=6, h_ambient=4)
    inp = W.mla_decode_inputs(cfg, seed=seed, device="cpu")
    sig = O.page_summaries(bits(inp["kv"]), np_i32(inp["page_table"]), np_i32(inp["seq_lens"]), 64)
    lists, counts = mla_lists_from_oracle(inp, sig, cfg)
    o, lse, h2l = run_mla(inp, cfg, lists, counts, n_splits)
    kvb = bits(inp["kv"])
    ro, rl = O.sparse_attention(bits(inp["q"]), kvb, kvb[..., :cfg.Dv], np_i32(inp["page_table"]),
                                np_i32(inp["seq_lens"]), lists, counts, np.array(h2l),
                                1.0 / math.sqrt(cfg.Dk), 64)
    assert_attn_close(o, lse, ro, rl)


@pytest.mark.parametrize("page_size,L,Hq,n_splits", [(32, 1000, 48, 2), (48, 1100, 40, 3),
                                                     (128, 2300, 48, 2), (16, 777, 36, 1)])
def test_mla_decode_page_sizes(page_size, L, Hq, n_splits):
    """64-key tiles over pages of 16-48 tokens (a tile spans pages: 16-row groups), of 128
    tokens (two tiles per page: boxes start at row 0 or 64) and ragged row tiles (T x Hq
    rows not a multiple of 64)."""
    cfg = W.MLADecode("case", B=2, T=2, Hq=Hq, Dk=576, Dv=512, page_size=page_size, seq_len=L,
                      alpha=3, beta=6, h_ambient=8)
    inp = W.mla_decode_inputs(cfg, seed=7, device="cpu")
    sig = O.page_summaries(bits(inp["kv"]), np_i32(inp["page_table"]), np_i32(inp["seq_lens"]),
                           page_size)
    lists, counts = mla_lists_from_oracle(inp, sig, cfg)
    o, lse, h2l = run_mla(inp, cfg, lists, counts, n_splits)
    kvb = bits(inp["kv"])
    ro, rl = O.sparse_attention(bits(inp["q"]), kvb, kvb[..., :cfg.Dv], np_i32(inp["page_table"]),
                                np_i32(inp["seq_lens"]), lists, counts, np.array(h2l),
                                1.0 / math.sqrt(cfg.Dk), page_size)
    assert_attn_close(o, lse, ro, rl)


@pytest.mark.slow
def test_mla_decode_full_size_sampled():
    cfg = W.MLA_MTP
    inp = W.mla_decode_inputs(cfg, seed=0, device="cpu")
    n = cfg.seq_len // cfg.page_size
    units = [(b, p) for b in (0, 3) for p in range(n)]
    sig = O.page_summaries(bits(inp["kv"]), np_i32(inp["page_table"]), np_i32(inp["seq_lens"]),
                           cfg.page_size, units=units)
    lists, counts = mla_lists_from_oracle(inp, sig, cfg, units=[0, 3])
    o, lse, h2l = run_mla(inp, cfg, lists, counts, 4)
    rng = np.random.default_rng(1)
    rows = [(b, t, int(h)) for b in (0, 3) for t in range(cfg.T) for h in rng.integers(0, cfg.Hq, 6)]
    rows += [(0, 1, int(h)) for h in inp["ambient_heads"][:3].tolist()]
    kvb = bits(inp["kv"])
    ro, rl = O.sparse_attention(bits(inp["q"]), kvb, kvb[..., :cfg.Dv], np_i32(inp["page_table"]),
                                np_i32(inp["seq_lens"]), lists, counts, np.array(h2l),
                                1.0 / math.sqrt(cfg.Dk), cfg.page_size, rows=rows)
    og, lg = o.cpu().double().numpy(), lse.cpu().double().numpy()
    for (b, t, h) in rows:
        assert np.abs(og[b, t, h] - ro[b, t, h]).max() <= O_TOL, (b, t, h)
        assert abs(lg[b, t, h] - rl[b, t, h]) <= LSE_TOL, (b, t, h)


# ----------------------------------------------------------------------------
# FP8 E4M3 pages with per-(page, kv head) scales
# ----------------------------------------------------------------------------
def fp8_case(cfg, seed, seq_lens=None):
    inp, g = gqa_case(cfg, seed=seed, seq_lens=seq_lens)
    kc, ks = W.fp8_pages(inp["k"])
    vc, vs = W.fp8_pages(inp["v"])
    f8 = dict(kc=kc, ks=ks, vc=vc, vs=vs)
    return inp, g, f8, {k: v.to(DEV) for k, v in f8.items()}


def run_decode_fp8(g, f8d, lists, counts, cfg, n_splits, h2l=None):
    h2l = [h // (cfg.Hq // cfg.Hkv) for h in range(cfg.Hq)] if h2l is None else h2l
    o_p, l_p = sa.sa_sparse_decode_fp8(g["q"], f8d["kc"], f8d["vc"], f8d["ks"], f8d["vs"],
                                       g["page_table"], g["seq_lens"],
                                       torch.from_numpy(lists).to(DEV),
                                       torch.from_numpy(counts).to(DEV), h2l,
                                       1.0 / math.sqrt(cfg.D), n_splits)
    o, ob, lse = sa.sa_combine(o_p, l_p)
    torch.cuda.synchronize()
    return o, lse


def oracle_fp8(inp, f8, lists, counts, cfg, h2l=None, rows=None):
    h2l = np.arange(cfg.Hq) // (cfg.Hq // cfg.Hkv) if h2l is None else np.asarray(h2l)
    return O.sparse_attention_fp8(bits(inp["q"]), f8["kc"].numpy(), f8["ks"].numpy(),
                                  f8["vc"].numpy(), f8["vs"].numpy(), np_i32(inp["page_table"]),
                                  np_i32(inp["seq_lens"]), lists, counts, h2l,
                                  1.0 / math.sqrt(cfg.D), cfg.page_size, rows=rows)


def test_summaries_fp8_bitexact():
    cfg = W.scaled(W.TINY_GQA, D=128, B=3)
    inp, g, f8, f8d = fp8_case(cfg, seed=30, seq_lens=[2048, 1000 + 3, 17])
    ref = O.page_summaries_fp8(f8["kc"].numpy(), f8["ks"].numpy(), np_i32(inp["page_table"]),
                               np_i32(inp["seq_lens"]), cfg.page_size)
    sig = sa.sa_build_page_summaries_fp8(f8d["kc"], f8d["ks"], g["page_table"], g["seq_lens"])
    torch.cuda.synchronize()
    pt = np_i32(inp["page_table"])
    for b, L in enumerate([2048, 1003, 17]):
        used = pt[b, :-(-L // cfg.page_size)]
        np.testing.assert_array_equal(bits(sig)[used], ref[used])


@pytest.mark.parametrize("n_splits", [1, 3])
def test_decode_fp8_vs_oracle(n_splits):
    # selection on the FP8 pages' summaries, then decode over the FP8 pages
    cfg = W.scaled(W.TINY_GQA, D=128, B=3)
    inp, g, f8, f8d = fp8_case(cfg, seed=31, seq_lens=[2048, 1000 + 3, 37])
    sig = O.page_summaries_fp8(f8["kc"].numpy(), f8["ks"].numpy(), np_i32(inp["page_table"]),
                               np_i32(inp["seq_lens"]), cfg.page_size)
    lists, counts = oracle_lists(inp, cfg, sig)
    o, lse = run_decode_fp8(g, f8d, lists, counts, cfg, n_splits)
    ro, rl = oracle_fp8(inp, f8, lists, counts, cfg)
    assert_attn_close(o, lse, ro, rl)


def test_decode_fp8_mtp_per_head_lists_and_empty():
    # T = 2 and 8 heads per kv head (16 rows per pair); the heads of a group
    # read different lists, one of them empty
    cfg = W.GQADecode("case", B=2, Hq=16, Hkv=2, D=128, page_size=16, seq_len_lo=0,
                      seq_len_hi=0, sink_tokens=16, local_tokens=16, budget_tokens=160, T=2)
    lens = [700, 333]
    inp, g, f8, f8d = fp8_case(cfg, seed=32, seq_lens=lens)
    rng = np.random.default_rng(32)
    n_lists, cap = 3, 9
    lists = np.full((2, n_lists, cap), -1, dtype=np.int32)
    counts = np.zeros((2, n_lists), dtype=np.int32)
    for b, L in enumerate(lens):
        nb = -(-L // 16)
        for li in range(n_lists - 1):
            pick = np.sort(rng.choice(nb, size=min(cap, nb), replace=False))
            lists[b, li, :len(pick)] = pick
            counts[b, li] = len(pick)
    h2l = [h % n_lists for h in range(cfg.Hq)]
    o, lse = run_decode_fp8(g, f8d, lists, counts, cfg, 2, h2l=h2l)
    ro, rl = oracle_fp8(inp, f8, lists, counts, cfg, h2l=h2l)
    assert_attn_close(o, lse, ro, rl)


def test_decode_fp8_llama8b_length_sampled():
    # Llama-8B-shaped sequences at full length (32768 tokens, 2048 pages) with
    # seeded page lists of the workload's budget, 13 splits; sampled rows
    cfg = W.scaled(W.LLAMA8B_DECODE, B=4)
    inp, g, f8, f8d = fp8_case(cfg, seed=33)
    rng = np.random.default_rng(33)
    nb = cfg.seq_len_hi // cfg.page_size
    lists = np.stack([np.stack([np.sort(rng.choice(nb, size=64, replace=False))
                                for _ in range(cfg.Hkv)]) for _ in range(cfg.B)]).astype(np.int32)
    counts = np.full((cfg.B, cfg.Hkv), 64, dtype=np.int32)
    o, lse = run_decode_fp8(g, f8d, lists, counts, cfg, 13)
    rows = [(b, 0, int(h)) for b in range(cfg.B) for h in rng.integers(0, cfg.Hq, 5)]
    ro, rl = oracle_fp8(inp, f8, lists, counts, cfg, rows=rows)
    og, lg = o.cpu().double().numpy(), lse.cpu().double().numpy()
    for (b, t, h) in rows:
        assert np.abs(og[b, t, h] - ro[b, t, h]).max() <= O_TOL, (b, t, h)
        assert abs(lg[b, t, h] - rl[b, t, h]) <= LSE_TOL, (b, t, h)


def test_decode_fp8_rejects_unsupported_shapes():
    cfg = W.TINY_GQA                                      # D = 64
    inp, g, f8, f8d = fp8_case(cfg, seed=34)
    lists = np.zeros((cfg.B, cfg.Hkv, 4), dtype=np.int32)
    counts = np.zeros((cfg.B, cfg.Hkv), dtype=np.int32)
    with pytest.raises(sa.SAError, match="UNSUPPORTED"):
        run_decode_fp8(g, f8d, lists, counts, cfg, 1)
