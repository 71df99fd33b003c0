"""Pins for the float64 oracle: each test ties it to something other than itself
(exact rational arithmetic, brute-force enumeration, closed forms, library
routines, the workload statements), so that a dropped term, a wrong sign or
index, or a transposed operand in the oracle fails one of them.  CPU only.
"""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch

import oracle as O

GOLDEN = __import__("os").path.join(__import__("os").path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------
# helpers (independent of the oracle's own arithmetic)
# ----------------------------------------------------------------------------
def rand_bf16(rng, shape, scale=1.0):
    x = (rng.standard_normal(shape) * scale).astype(np.float32)
    return (torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))


def bf16_fraction(bits):
    """Exact value of one bf16 pattern from its fields (sign, exponent, fraction)."""
    bits = int(bits)
    s = -1 if bits >> 15 else 1
    e = (bits >> 7) & 0xFF
    f = bits & 0x7F
    if e == 0:
        return s * Fraction(f, 1) * Fraction(2) ** (-133)
    return s * Fraction(128 + f, 1) * Fraction(2) ** (e - 134)


def nearest_bf16_bruteforce(x: Fraction, cands):
    best = min(abs(v - x) for _, v in cands)
    ties = [b for b, v in cands if abs(v - x) == best]
    if len(ties) == 1:
        return ties[0]
    even = [b for b in ties if (b & 1) == 0]
    assert len(even) >= 1
    # +0 / -0 both even for x == 0: take the sign of x
    return even[0] if len(even) == 1 else (even[1] if x < 0 else even[0])


def exact_dot_fraction(a_bits, b_bits):
    return sum((bf16_fraction(x) * bf16_fraction(y) for x, y in zip(a_bits, b_bits)), Fraction(0))


# ----------------------------------------------------------------------------
# bf16 conversions
# ----------------------------------------------------------------------------
def test_bf16_decode_against_field_definition():
    rng = np.random.default_rng(1)
    bits = np.concatenate([np.array([0x3F80, 0xC000, 0x0001, 0x7F7F, 0x8000, 0x0080, 0x007F],
                                    dtype=np.uint16),
                           rng.integers(0, 0x7F80, 500).astype(np.uint16)])
    vals = O.bf16_to_f64(bits)
    for b, v in zip(bits, vals):
        assert Fraction(float(v)) == bf16_fraction(b)
    assert vals[0] == 1.0 and vals[1] == -2.0 and vals[2] == 2.0 ** -133
    assert vals[3] == (2 - 2 ** -7) * 2.0 ** 127


def test_bf16_rne_against_bruteforce():
    rng = np.random.default_rng(2)
    xs = [1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -30, -(1 + 2 ** -8), 1.5 * 2.0 ** -133,
          2.5 * 2.0 ** -133, 2.0 ** -126 * (1 - 2 ** -9), 0.0, 255.5, 256.5 * 2 ** -7]
    xs += list(rng.standard_normal(20) * 10.0 ** rng.integers(-30, 30, 20))
    got = O.f64_to_bf16_rne(np.array(xs))
    for x, g in zip(xs, got):
        fx = Fraction(x)
        # candidates: the two bf16 neighbours of x found from float32 truncation
        t = int(np.array([x], dtype=np.float32).view(np.uint32)[0] >> 16)
        cands = [(c, bf16_fraction(c)) for c in {t - 1, t, t + 1, t + 2} if 0 <= (c & 0x7FFF) < 0x7F80]
        assert int(g) == nearest_bf16_bruteforce(fx, cands), (x, hex(g))
    assert O.f64_to_bf16_rne(np.array([1 + 2 ** -8]))[0] == 0x3F80        # tie -> even
    assert O.f64_to_bf16_rne(np.array([1 + 3 * 2 ** -8]))[0] == 0x3F82    # tie -> even (up)
    assert O.f64_to_bf16_rne(np.array([1.5 * 2.0 ** -133]))[0] == 0x0002  # subnormal tie


# ----------------------------------------------------------------------------
# page budget (tests/golden/page_budget.txt: the tiny workload's stated counts,
# and reading R1's counts for the other two budgets worked out by hand)
# ----------------------------------------------------------------------------
def test_page_budget_matches_golden_counts():
    rows = []
    for line in open(f"{GOLDEN}/page_budget.txt"):
        line = line.split("#")[0].strip()
        if line:
            rows.append([int(x) for x in line.split()])
    assert len(rows) == 3
    for sink, local, budget, P, n_sink, n_local, pages, k_top in rows:
        assert O.page_budget(sink, local, budget, P) == (n_sink, n_local, pages, k_top)


# ----------------------------------------------------------------------------
# two-level page map (reading R19)
# ----------------------------------------------------------------------------
def _read_page_dir_golden():
    sections, cur, shift = {}, None, None
    for line in open(f"{GOLDEN}/page_dir.txt"):
        line = line.split("#")[0].strip()
        if not line:
            continue
        if line.startswith("shift"):
            shift = int(line.split()[1])
        elif line in ("dir", "blocks", "table"):
            cur = sections.setdefault(line, [])
        else:
            cur.append([int(x) for x in line.split()])
    return shift, {k: np.array(v, dtype=np.int32) for k, v in sections.items()}


def test_page_dir_golden_worked_example():
    shift, g = _read_page_dir_golden()
    got = O.page_table_from_dir(g["dir"], g["blocks"], shift)
    assert got.dtype == np.int32 and got.shape == g["table"].shape
    assert np.array_equal(got, g["table"])


def _pack_dir(table, shift, rng):
    """A two-level map holding a flat table: one block per run of 2^shift
    columns that has any page, blocks numbered in a shuffled order."""
    B, W = table.shape
    width = 1 << shift
    n_dir = -(-W // width)
    padded = np.full((B, n_dir * width), -1, dtype=np.int32)
    padded[:, :W] = table
    used = [(b, j) for b in range(B) for j in range(n_dir)
            if (padded[b, j * width:(j + 1) * width] >= 0).any()]
    order = rng.permutation(len(used))
    page_dir = np.full((B, n_dir), -1, dtype=np.int32)
    blocks = np.full((max(len(used), 1), width), -1, dtype=np.int32)
    for (b, j), bid in zip(used, order):
        page_dir[b, j] = bid
        blocks[bid] = padded[b, j * width:(j + 1) * width]
    return page_dir, blocks, padded


@pytest.mark.parametrize("shift", [0, 1, 3, 5])
def test_page_dir_holds_any_flat_table(shift):
    # a flat table packed into blocks by the inverse construction comes back
    # unchanged; the metadata is the directory plus the used blocks only
    rng = np.random.default_rng(40 + shift)
    lens = [0, 1, 37, 200, 64]
    W = max(lens)
    table = np.full((len(lens), W), -1, dtype=np.int32)
    ids = rng.permutation(sum(lens)).astype(np.int32)
    off = 0
    for b, n in enumerate(lens):
        table[b, :n] = ids[off:off + n]
        off += n
    page_dir, blocks, padded = _pack_dir(table, shift, rng)
    assert np.array_equal(O.page_table_from_dir(page_dir, blocks, shift), padded)
    width = 1 << shift
    assert blocks.shape[0] == sum(-(-n // width) for n in lens)


def test_page_dir_block_numbering_is_irrelevant():
    # renumbering the blocks (and the directory with them) changes nothing
    shift, g = _read_page_dir_golden()
    perm = np.array([2, 0, 1])                 # new id of old block i
    blocks = np.empty_like(g["blocks"])
    blocks[perm] = g["blocks"]
    d = g["dir"].copy()
    ok = (d >= 0) & (d < len(perm))
    d[ok] = perm[d[ok]]
    assert np.array_equal(O.page_table_from_dir(d, blocks, shift), g["table"])


# ----------------------------------------------------------------------------
# exact dot products
# ----------------------------------------------------------------------------
def test_exact_dots_correctly_rounded():
    rng = np.random.default_rng(3)
    A = rand_bf16(rng, (5, 64))
    Bm = rand_bf16(rng, (7, 64), scale=0.3)
    # adversarial rows: huge cancelling terms around a small one
    A[0, :3] = np.array([0x7180, 0x3F80, 0x7180], dtype=np.uint16)   # 2^100, 1, 2^100
    Bm[0, :3] = np.array([0x3F80, 0x3F80, 0xBF80], dtype=np.uint16)  # 1, 1, -1
    Bm[0, 3:] = 0
    A[1, :] = 0x0001                                                 # subnormal q
    got = O.exact_dots(O.bf16_to_f64(A), O.bf16_to_f64(Bm))
    for i in range(A.shape[0]):
        for j in range(Bm.shape[0]):
            assert got[i, j] == float(exact_dot_fraction(A[i], Bm[j])), (i, j)
    assert got[0, 0] == 1.0
    assert (2.0 ** 100 + 1.0) - 2.0 ** 100 == 0.0     # left-to-right float64 loses it


# ----------------------------------------------------------------------------
# selection
# ----------------------------------------------------------------------------
def _tiny_select_case(rng, B, T, Hq, Hkv, D, P, lens, pool_perm=True, sig_scale=1.0):
    q = rand_bf16(rng, (B, T, Hq, D))
    npages = [-(-L // P) for L in lens]
    pool = sum(npages)
    perm = rng.permutation(pool) if pool_perm else np.arange(pool)
    pt = np.full((B, max(npages)), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(npages):
        pt[b, :n] = perm[off:off + n]
        off += n
    sig = rand_bf16(rng, (pool, Hkv, D), scale=sig_scale)
    return q, sig, pt, np.array(lens, dtype=np.int32)


def _bruteforce_selection(q, sig, pt, lens, P, sink, local, budget, b, kvh, G):
    n_sink, n_local = -(-sink // P), -(-local // P)
    bp = budget // P
    nb = -(-int(lens[b]) // P)
    if nb <= bp:
        return list(range(nb))
    cand = list(range(n_sink, nb - n_local))
    k = bp - n_sink - n_local
    T = q.shape[1]
    score = {}
    for p in cand:
        vals = [float(exact_dot_fraction(q[b, t, h], sig[pt[b, p], kvh]))
                for t in range(T) for h in range(kvh * G, (kvh + 1) * G)]
        score[p] = max(vals)
    key = lambda p: (-score[p], p)  # noqa: E731
    winners = []
    for subset in itertools.combinations(cand, k):
        rest = [p for p in cand if p not in subset]
        if all(key(s) < key(r) for s in subset for r in rest):
            winners.append(subset)
    assert len(winners) == 1          # exactly one dominant subset
    return sorted(list(range(n_sink)) + list(winners[0]) + list(range(nb - n_local, nb)))


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_select_matches_bruteforce(seed):
    rng = np.random.default_rng(10 + seed)
    P, Hq, Hkv, D, T = 4, 4, 2, 16, (1 if seed % 2 == 0 else 2)
    lens = [45, 37]   # 12 and 10 pages, ragged last page
    sink, local, budget = 4, 8, 24   # 1 sink page, 2 local pages, 6-page budget -> k_top = 3
    q, sig, pt, sl = _tiny_select_case(rng, 2, T, Hq, Hkv, D, P, lens)
    pages, counts = O.select_pages(q, sig, pt, sl, P, sink, local, budget)
    for b in range(2):
        for kvh in range(Hkv):
            want = _bruteforce_selection(q, sig, pt, sl, P, sink, local, budget, b, kvh, Hq // Hkv)
            assert counts[b, kvh] == len(want)
            assert list(pages[b, kvh, :counts[b, kvh]]) == want
            assert all(pages[b, kvh, counts[b, kvh]:] == -1)


def test_select_ties_go_to_lowest_index():
    rng = np.random.default_rng(20)
    P, Hq, Hkv, D = 4, 2, 1, 8
    q, sig, pt, sl = _tiny_select_case(rng, 1, 1, Hq, Hkv, D, P, [48])
    q[:] = 0                                      # every score is exactly 0
    pages, counts = O.select_pages(q, sig, pt, sl, P, 4, 4, 20)   # 1 sink, 1 local, k_top 3
    assert list(pages[0, 0, :counts[0, 0]]) == [0, 1, 2, 3, 11]
    # duplicate summaries: the lower logical page wins the last slot
    q, sig, pt, sl = _tiny_select_case(rng, 1, 1, Hq, Hkv, D, P, [48], pool_perm=True)
    sig[pt[0, 7]] = sig[pt[0, 9]]
    sc = O.page_scores(O.bf16_to_f64(q[0, 0]), O.bf16_to_f64(sig[pt[0, 1:11], 0]))
    order = sorted(range(1, 11), key=lambda p: (-sc[p - 1], p))
    pos7, pos9 = order.index(7), order.index(9)
    assert pos7 + 1 == pos9                       # adjacent, 7 first
    k = pos9                                      # budget cutting between them
    pages, counts = O.select_pages(q, sig, pt, sl, P, 4, 4, 4 * (k + 2))
    sel = set(pages[0, 0, :counts[0, 0]])
    assert 7 in sel and 9 not in sel


def test_streaming_and_dense_special_cases():
    rng = np.random.default_rng(21)
    q, sig, pt, sl = _tiny_select_case(rng, 2, 1, 4, 2, 8, 4, [40, 9])
    # k_top = 0: StreamingLLM (sink + local only), [TS] "Configuration" streaming mode
    pages, counts = O.select_pages(q, sig, pt, sl, 4, 8, 8, 16)
    assert list(pages[0, 0, :counts[0, 0]]) == [0, 1, 8, 9]
    # N_b <= budget pages: everything
    assert list(pages[1, 1, :counts[1, 1]]) == [0, 1, 2]


def test_selection_invariant_to_physical_page_ids():
    rng = np.random.default_rng(22)
    q, sig, pt, sl = _tiny_select_case(rng, 2, 2, 8, 2, 16, 4, [80, 61])
    a, ca = O.select_pages(q, sig, pt, sl, 4, 4, 8, 36)
    perm = rng.permutation(sig.shape[0])
    sig2 = np.empty_like(sig)
    sig2[perm] = sig                         # physical page i moves to perm[i]
    pt2 = np.where(pt >= 0, perm[np.maximum(pt, 0)], -1).astype(np.int32)
    b2, cb = O.select_pages(q, sig2, pt2, sl, 4, 4, 8, 36)
    assert np.array_equal(a, b2) and np.array_equal(ca, cb)


def test_selection_refines_cancelling_scores():
    # page 1 scores exactly 1 but float64 BLAS gives 0; page 2 scores exactly 0.5
    P, D = 1, 3
    q = np.array([[[[0x3F80, 0x3F80, 0x3F80]]]], dtype=np.uint16)
    sig = np.zeros((4, 1, D), dtype=np.uint16)
    sig[1, 0] = [0x7180, 0x3F80, 0xF180]      # 2^100, 1, -2^100
    sig[2, 0] = [0x3F00, 0, 0]                # 0.5
    sig[3, 0] = [0x3E80, 0, 0]                # 0.25
    pt = np.array([[0, 1, 2, 3]], dtype=np.int32)
    pages, counts = O.select_pages(q, sig, pt, np.array([4], dtype=np.int32), P, 1, 1, 3)
    assert list(pages[0, 0, :counts[0, 0]]) == [0, 1, 3]


@pytest.mark.parametrize("alpha,beta", [(3, 4), (0, 7), (6, 6)])
def test_mla_tiers(alpha, beta):
    # (0, 7): no critical tier; (6, 6): the tiers ask for more pages than a
    # sequence holds (every page in, the critical ones first by rank)
    rng = np.random.default_rng(23)
    B, T, Hq, Dk, P = 2, 2, 8, 24, 4
    q = rand_bf16(rng, (B, T, Hq, Dk))
    pool = 2 * 10
    sig = rand_bf16(rng, (pool, 1, Dk))
    pt = rng.permutation(pool).astype(np.int32).reshape(2, 10)
    sl = np.array([40, 37], dtype=np.int32)
    crit, cc, amb, ac = O.select_pages_mla(q, sig, pt, sl, P, alpha, beta)
    for b in range(B):
        nb = -(-int(sl[b]) // P)
        exact = {p: max(float(exact_dot_fraction(q[b, t, h], sig[pt[b, p], 0]))
                        for t in range(T) for h in range(Hq)) for p in range(nb)}
        order = sorted(range(nb), key=lambda p: (-exact[p], p))
        assert list(crit[b, :cc[b]]) == sorted(order[:alpha])
        assert list(amb[b, :ac[b]]) == sorted(order[alpha:alpha + beta])
    # with every head ambient, crit u amb equals the untiered top-(alpha+beta)
    pages, counts = O.select_pages(q, sig, pt, sl, P, 0, 0, (alpha + beta) * P)
    for b in range(B):
        assert sorted(list(crit[b, :cc[b]]) + list(amb[b, :ac[b]])) == list(pages[b, 0, :counts[b, 0]])


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------
def _attn_case(rng, B=2, T=1, Hq=4, Hkv=2, D=16, Dv=16, P=4, lens=(23, 14)):
    q = rand_bf16(rng, (B, T, Hq, D))
    npages = [-(-L // P) for L in lens]
    pool = sum(npages)
    perm = rng.permutation(pool)
    pt = np.full((B, max(npages)), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(npages):
        pt[b, :n] = perm[off:off + n]
        off += n
    k = rand_bf16(rng, (pool, Hkv, P, D))
    v = rand_bf16(rng, (pool, Hkv, P, Dv))
    return q, k, v, pt, np.array(lens, dtype=np.int32), npages


@pytest.mark.parametrize("T,scale_mult", [(1, 1.0), (3, 1.0), (2, -1.0), (2, 3.0)])
def test_dense_budget_equals_sdpa(T, scale_mult):
    # also at a negative scale and a 3x sharper one (the GPU parity cases use both)
    rng = np.random.default_rng(30 + T)
    q, k, v, pt, sl, npages = _attn_case(rng, T=T)
    B, _, Hq, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    P = 4
    lists = np.full((B, Hkv, max(npages)), -1, dtype=np.int32)
    counts = np.zeros((B, Hkv), dtype=np.int32)
    for b in range(B):
        lists[b, :, :npages[b]] = np.arange(npages[b])
        counts[b] = npages[b]
    h2l = np.arange(Hq) // G
    scale = scale_mult / math.sqrt(D)
    o, lse = O.sparse_attention(q, k, v, pt, sl, lists, counts, h2l, scale, P)
    for b in range(B):
        L = int(sl[b])
        phys = pt[b, :npages[b]]
        K = torch.from_numpy(O.bf16_to_f64(k[phys]).transpose(1, 0, 2, 3).reshape(Hkv, -1, D)[:, :L])
        V = torch.from_numpy(O.bf16_to_f64(v[phys]).transpose(1, 0, 2, 3).reshape(Hkv, -1, D)[:, :L])
        Q = torch.from_numpy(O.bf16_to_f64(q[b]).transpose(1, 0, 2))       # [Hq, T, D]
        Kx = K.repeat_interleave(G, 0)
        Vx = V.repeat_interleave(G, 0)
        mask = torch.arange(L)[None, :] <= (L - T + torch.arange(T))[:, None]
        ref = torch.nn.functional.scaled_dot_product_attention(Q, Kx, Vx, attn_mask=mask, scale=scale)
        np.testing.assert_allclose(o[b].transpose(1, 0, 2), ref.numpy(), rtol=0, atol=1e-12)
        s = (scale * (Q @ Kx.transpose(1, 2))).numpy()
        s = np.where(mask.numpy()[None], s, -np.inf)
        np.testing.assert_allclose(lse[b].T, scipy.special.logsumexp(s, axis=-1), rtol=0, atol=1e-12)


def test_explicit_query_positions_equal_sdpa_with_their_mask():
    # query token t of sequence b at q_pos[b] + t (a prompt chunk inside the
    # cache, one past its end, one partly before its start): full budget against
    # the library's attention with the mask those positions define
    T = 3
    rng = np.random.default_rng(37)
    q, k, v, pt, sl, npages = _attn_case(rng, B=3, T=T, lens=(23, 14, 9))
    B, _, Hq, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    P = 4
    lists = np.full((B, Hkv, max(npages)), -1, dtype=np.int32)
    counts = np.zeros((B, Hkv), dtype=np.int32)
    for b in range(B):
        lists[b, :, :npages[b]] = np.arange(npages[b])
        counts[b] = npages[b]
    q_pos = np.array([int(sl[0]) // 2, int(sl[1]) + 5, -1][:B], dtype=np.int32)
    scale = 1.0 / math.sqrt(D)
    o, lse = O.sparse_attention(q, k, v, pt, sl, lists, counts, np.arange(Hq) // G, scale, P,
                                q_pos=q_pos)
    for b in range(B):
        L = int(sl[b])
        phys = pt[b, :npages[b]]
        K = torch.from_numpy(O.bf16_to_f64(k[phys]).transpose(1, 0, 2, 3).reshape(Hkv, -1, D)[:, :L])
        V = torch.from_numpy(O.bf16_to_f64(v[phys]).transpose(1, 0, 2, 3).reshape(Hkv, -1, D)[:, :L])
        Q = torch.from_numpy(O.bf16_to_f64(q[b]).transpose(1, 0, 2))
        mask = torch.arange(L)[None, :] <= (int(q_pos[b]) + torch.arange(T))[:, None]
        seen = mask.any(dim=1).numpy()
        ref = torch.nn.functional.scaled_dot_product_attention(
            Q, K.repeat_interleave(G, 0), V.repeat_interleave(G, 0), attn_mask=mask, scale=scale)
        got = o[b].transpose(1, 0, 2)
        np.testing.assert_allclose(got[:, seen], ref.numpy()[:, seen], rtol=0, atol=1e-12)
        assert np.all(got[:, ~seen] == 0) and np.all(np.isneginf(lse[b][~seen]))


@pytest.mark.parametrize("T", [1, 2])
def test_sparse_equals_masked_dense(T):
    rng = np.random.default_rng(40 + T)
    q, k, v, pt, sl, npages = _attn_case(rng, T=T, lens=(37, 29))
    B, _, Hq, D = q.shape
    Hkv = k.shape[1]
    n_lists = 3      # per-head lists, not tied to the kv head (QK 2D sparsity)
    lists = np.full((B, n_lists, 6), -1, dtype=np.int32)
    counts = np.zeros((B, n_lists), dtype=np.int32)
    for b in range(B):
        for li in range(n_lists):
            c = int(rng.integers(0, min(6, npages[b]) + 1))
            lists[b, li, :c] = np.sort(rng.choice(npages[b], c, replace=False))
            counts[b, li] = c
    h2l = rng.integers(0, n_lists, (B, Hq))
    a = O.sparse_attention(q, k, v, pt, sl, lists, counts, h2l, 0.3, 4)
    m = O.masked_dense_attention(q, k, v, pt, sl, lists, counts, h2l, 0.3, 4)
    np.testing.assert_allclose(a[0], m[0], rtol=0, atol=1e-12)
    np.testing.assert_array_equal(np.isinf(a[1]), np.isinf(m[1]))
    fin = np.isfinite(a[1])
    np.testing.assert_allclose(a[1][fin], m[1][fin], rtol=0, atol=1e-12)
    assert np.all(a[0][~fin] == 0)


def test_closed_forms():
    rng = np.random.default_rng(50)
    D, P = 8, 4
    q = rand_bf16(rng, (1, 1, 1, D))
    k = rand_bf16(rng, (1, 1, P, D))
    v = rand_bf16(rng, (1, 1, P, D))
    pt = np.array([[0]], dtype=np.int32)
    lists = np.array([[[0]]], dtype=np.int32)
    cnt = np.array([[1]], dtype=np.int32)
    # one key: O = v, lse = scale q.k
    o, lse = O.sparse_attention(q, k, v, pt, np.array([1]), lists, cnt, [0], 0.5, P)
    np.testing.assert_array_equal(o[0, 0, 0], O.bf16_to_f64(v[0, 0, 0]))
    qk = float(exact_dot_fraction(q[0, 0, 0], k[0, 0, 0]))
    assert abs(lse[0, 0, 0] - 0.5 * qk) < 1e-14
    # equal keys: O = mean(v), lse = s + log n
    k2 = np.repeat(k[:, :, :1], P, axis=2)
    o, lse = O.sparse_attention(q, k2, v, pt, np.array([P]), lists, cnt, [0], 0.5, P)
    np.testing.assert_allclose(o[0, 0, 0], O.bf16_to_f64(v[0, 0]).mean(0), atol=1e-14)
    assert abs(lse[0, 0, 0] - (0.5 * qk + math.log(P))) < 1e-13
    # two keys: weights are sigmoid(s0 - s1), 1 - that
    o, lse = O.sparse_attention(q, k, v, pt, np.array([2]), lists, cnt, [0], 0.5, P)
    s0 = 0.5 * float(exact_dot_fraction(q[0, 0, 0], k[0, 0, 0]))
    s1 = 0.5 * float(exact_dot_fraction(q[0, 0, 0], k[0, 0, 1]))
    w0 = 1 / (1 + math.exp(s1 - s0))
    want = w0 * O.bf16_to_f64(v[0, 0, 0]) + (1 - w0) * O.bf16_to_f64(v[0, 0, 1])
    np.testing.assert_allclose(o[0, 0, 0], want, atol=1e-14)
    assert abs(lse[0, 0, 0] - (max(s0, s1) + math.log1p(math.exp(-abs(s0 - s1))))) < 1e-14
    # empty list: O = 0, lse = -inf
    o, lse = O.sparse_attention(q, k, v, pt, np.array([P]), lists, np.array([[0]]), [0], 0.5, P)
    assert np.all(o == 0) and lse[0, 0, 0] == -np.inf


# ----------------------------------------------------------------------------
# combine
# ----------------------------------------------------------------------------
def test_combine_partition_invariance():
    rng = np.random.default_rng(60)
    q, k, v, pt, sl, npages = _attn_case(rng, T=2, lens=(44, 41))
    B, T, Hq, D = q.shape
    Hkv = k.shape[1]
    h2l = np.arange(Hq) // (Hq // Hkv)
    lists = np.tile(np.arange(11, dtype=np.int32), (B, Hkv, 1))
    counts = np.full((B, Hkv), 11, dtype=np.int32)
    full = O.sparse_attention(q, k, v, pt, sl, lists, counts, h2l, 0.25, 4)
    for bounds in ([0, 11], [0, 3, 11], [0, 5, 6, 11], [0, 0, 4, 4, 11]):
        parts = []
        for s0, s1 in zip(bounds[:-1], bounds[1:]):
            li = np.full_like(lists, -1)
            li[:, :, :s1 - s0] = lists[:, :, s0:s1]
            parts.append(O.sparse_attention(q, k, v, pt, sl, li, np.full_like(counts, s1 - s0),
                                            h2l, 0.25, 4))
        o_p = np.stack([p[0] for p in parts])
        l_p = np.stack([p[1] for p in parts])
        for perm in (None, np.arange(len(parts))[::-1]):
            op, lp = (o_p, l_p) if perm is None else (o_p[perm], l_p[perm])
            o, lse = O.combine(op, lp)
            np.testing.assert_allclose(o, full[0], atol=1e-12)
            np.testing.assert_allclose(lse, full[1], atol=1e-12)


def test_combine_special_cases():
    rng = np.random.default_rng(61)
    o = rng.standard_normal((1, 5, 4))
    lse = rng.standard_normal((1, 5))
    a, la = O.combine(o, lse)
    np.testing.assert_array_equal(a, o[0])
    np.testing.assert_array_equal(la, lse[0])
    o2 = np.concatenate([o, rng.standard_normal((1, 5, 4))])
    l2 = np.concatenate([lse, np.full((1, 5), -np.inf)])
    a, la = O.combine(o2, l2)
    np.testing.assert_allclose(a, o[0], atol=1e-15)
    np.testing.assert_allclose(la, lse[0], atol=1e-15)
    a, la = O.combine(o2, np.full((2, 5), -np.inf))
    assert np.all(a == 0) and np.all(la == -np.inf)
    # two splits: closed form with scipy
    l3 = rng.standard_normal((2, 5))
    a, la = O.combine(o2, l3)
    np.testing.assert_allclose(la, scipy.special.logsumexp(l3, axis=0), atol=1e-14)
    w = scipy.special.softmax(l3, axis=0)
    np.testing.assert_allclose(a, (w[..., None] * o2).sum(0), atol=1e-14)


# ----------------------------------------------------------------------------
# block union
# ----------------------------------------------------------------------------
def test_block_union_bruteforce():
    rng = np.random.default_rng(70)
    Hq, Hkv, NQB, off, top_k = 4, 2, 3, 6, 2
    NKB = off + NQB
    s = rng.standard_normal((Hq, NQB, NKB)).astype(np.float32)
    s[0, 1, 2] = s[0, 1, 3]        # an exact tie: the lower block wins
    tables, counts = O.block_union(s, Hkv, off, top_k)
    for g in range(Hkv):
        want = set()
        for h in range(g * 2, g * 2 + 2):
            for j in range(NQB):
                d = off + j
                cand = sorted(range(1, d), key=lambda c: (-float(s[h, j, c]), c))
                mask = {0, d} | set(cand[:top_k])
                assert mask <= set(tables[g, :counts[g]])
                want |= mask
        assert list(tables[g, :counts[g]]) == sorted(want)
        assert all(tables[g, counts[g]:] == -1)
    if s[0, 1, 2] >= np.sort(s[0, 1, 1:7])[-2]:
        assert 2 in set(tables[0, :counts[0]])


# ----------------------------------------------------------------------------
# page summaries
# ----------------------------------------------------------------------------
def test_page_summaries_exact_mean():
    rng = np.random.default_rng(80)
    P, Hkv, D = 4, 2, 6
    k = rand_bf16(rng, (3, Hkv, P, D))
    k[2, 0, :, 0] = [0x7180, 0x3F80, 0xF180, 0x0001]      # cancellation + subnormal
    pt = np.array([[2, 0, 1]], dtype=np.int32)
    sl = np.array([10], dtype=np.int32)                  # last page has 2 valid keys
    sig = O.page_summaries(k, pt, sl, P)
    for p, nval in ((0, 4), (1, 4), (2, 2)):
        phys = pt[0, p]
        for h in range(Hkv):
            for d in range(D):
                mean = sum(bf16_fraction(k[phys, h, j, d]) for j in range(nval)) / nval
                s64 = float(sum(bf16_fraction(k[phys, h, j, d]) for j in range(nval)))
                want = O.f64_to_bf16_rne(np.array([s64 / nval]))[0]
                assert sig[phys, h, d] == want
                # the bf16 result is within one bf16 spacing of the exact mean
                assert abs(bf16_fraction(sig[phys, h, d]) - mean) <= abs(mean) / 128 + Fraction(1, 2 ** 133)


# ----------------------------------------------------------------------------
# FP8 E4M3 pages with per-(page, kv head) scales (reading R15)
# ----------------------------------------------------------------------------
def e4m3_fraction(code):
    """Exact value of one E4M3 code from its fields (None for NaN codes)."""
    code = int(code)
    s = -1 if code >> 7 else 1
    e = (code >> 3) & 0xF
    f = code & 0x7
    if e == 0xF and f == 0x7:
        return None
    if e == 0:
        return s * Fraction(f, 8) * Fraction(1, 64)
    return s * (1 + Fraction(f, 8)) * Fraction(2) ** (e - 7)


def rand_e4m3(rng, shape):
    """Random non-NaN E4M3 codes."""
    c = rng.integers(0, 256, size=shape).astype(np.uint8)
    return np.where((c & 0x7F) == 0x7F, c ^ 0x01, c).astype(np.uint8)


def test_e4m3_decode_against_fields_and_library():
    codes = np.arange(256, dtype=np.uint8)
    mine = O.e4m3_to_f64(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        want = e4m3_fraction(c)
        if want is None:
            assert np.isnan(mine[c]) and np.isnan(lib[c])
        else:
            assert mine[c] == float(want) == lib[c]
    # the format's landmarks: largest finite, smallest subnormal, smallest normal, one
    assert mine[0x7E] == 448.0 and mine[0x01] == 2.0 ** -9 and mine[0x08] == 2.0 ** -6
    assert mine[0x38] == 1.0 and mine[0xB8] == -1.0 and np.signbit(mine[0x80])


def _fp8_case(rng, pow2_scales):
    P_pool, Hkv, P, D = 5, 2, 8, 16
    kc = rand_e4m3(rng, (P_pool, Hkv, P, D))
    vc = rand_e4m3(rng, (P_pool, Hkv, P, D))
    if pow2_scales:
        ks = np.ldexp(1.0, rng.integers(-12, 4, size=(P_pool, Hkv))).astype(np.float32)
        vs = np.ldexp(1.0, rng.integers(-12, 4, size=(P_pool, Hkv))).astype(np.float32)
    else:
        ks = (rng.random((P_pool, Hkv)) * 0.02 + 1e-3).astype(np.float32)
        vs = (rng.random((P_pool, Hkv)) * 0.02 + 1e-3).astype(np.float32)
    return kc, vc, ks, vs


def _to_bf16_bits(x):
    """bf16 patterns of float64 values that are exactly bf16 (checked)."""
    f = x.astype(np.float32)
    assert np.array_equal(f.astype(np.float64), x)
    b = f.view(np.uint32)
    assert np.all((b & 0xFFFF) == 0)
    return (b >> 16).astype(np.uint16)


def test_fp8_attention_reduces_to_bf16_with_power_of_two_scales():
    # With power-of-two scales every dequantized key and value is a bf16 value,
    # so the FP8 oracle must give exactly the bf16 oracle's result on them.
    rng = np.random.default_rng(90)
    kc, vc, ks, vs = _fp8_case(rng, True)
    P = kc.shape[2]
    kb = _to_bf16_bits(O.e4m3_to_f64(kc) * ks.astype(np.float64)[..., None, None])
    vb = _to_bf16_bits(O.e4m3_to_f64(vc) * vs.astype(np.float64)[..., None, None])
    B, T, Hq = 2, 2, 4
    q = rand_bf16(rng, (B, T, Hq, kc.shape[3]))
    pt = np.array([[3, 1, 4], [0, 2, 1]], dtype=np.int32)
    sl = np.array([21, 13], dtype=np.int32)
    lists = np.array([[[0, 2, 1]], [[1, 0, 0]]], dtype=np.int32)
    cnt = np.array([[3], [2]], dtype=np.int32)
    h2l = [0] * Hq
    o8, l8 = O.sparse_attention_fp8(q, kc, ks, vc, vs, pt, sl, lists, cnt, h2l, 0.25, P)
    ob, lb = O.sparse_attention(q, kb, vb, pt, sl, lists, cnt, h2l, 0.25, P)
    np.testing.assert_array_equal(o8, ob)
    np.testing.assert_array_equal(l8, lb)
    s8 = O.page_summaries_fp8(kc, ks, pt, sl, P)
    sb = O.page_summaries(kb, pt, sl, P)
    np.testing.assert_array_equal(s8, sb)


def test_fp8_summaries_exact_mean_general_scale():
    # Non-power-of-two scales: the summary is RNE_bf16(RN64(RN64(exact sum of
    # the dequantized keys) / n)), checked with exact rationals per element.
    rng = np.random.default_rng(91)
    kc, _, ks, _ = _fp8_case(rng, False)
    P = kc.shape[2]
    pt = np.array([[2, 0, 3]], dtype=np.int32)
    sl = np.array([19], dtype=np.int32)                  # last page: 3 valid keys
    sig = O.page_summaries_fp8(kc, ks, pt, sl, P)
    for p, nval in ((0, 8), (1, 8), (2, 3)):
        phys = pt[0, p]
        for h in range(kc.shape[1]):
            sc = Fraction(float(ks[phys, h]))
            for d in range(kc.shape[3]):
                tot = sum(e4m3_fraction(kc[phys, h, j, d]) * sc for j in range(nval))
                want = O.f64_to_bf16_rne(np.array([float(tot) / nval]))[0]
                assert sig[phys, h, d] == want


def test_fp8_attention_closed_forms():
    rng = np.random.default_rng(92)
    kc, vc, ks, vs = _fp8_case(rng, False)
    P, D = kc.shape[2], kc.shape[3]
    q = rand_bf16(rng, (1, 1, 2, D))                     # head 0 reads kv head 0
    pt = np.array([[3]], dtype=np.int32)
    lists = np.array([[[0]]], dtype=np.int32)
    cnt = np.array([[1]], dtype=np.int32)
    # one key: O = its dequantized value, lse = scale q . k
    o, lse = O.sparse_attention_fp8(q, kc, ks, vc, vs, pt, np.array([1]), lists, cnt, [0, 0], 0.5,
                                    P)
    v0 = [e4m3_fraction(c) * Fraction(float(vs[3, 0])) for c in vc[3, 0, 0]]
    np.testing.assert_array_equal(o[0, 0, 0], np.array([float(x) for x in v0]))
    qk = sum(bf16_fraction(a) * e4m3_fraction(c) for a, c in zip(q[0, 0, 0], kc[3, 0, 0]))
    assert abs(lse[0, 0, 0] - 0.5 * float(qk * Fraction(float(ks[3, 0])))) < 1e-12


# ----------------------------------------------------------------------------
# appending tokens to the paged cache
# ----------------------------------------------------------------------------
def _append_case(seed, P=4, Hkv=2, D=3, lens=(5, 8, 0), max_new=6):
    rng = np.random.default_rng(seed)
    B = len(lens)
    npg = [-(-(L + max_new) // P) for L in lens]
    pool = sum(npg) + 2                                  # two pages no sequence uses
    perm = rng.permutation(pool)
    pt = np.full((B, max(npg)), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(npg):
        pt[b, :n] = perm[off:off + n]
        off += n
    k = rand_bf16(rng, (pool, Hkv, P, D))
    v = rand_bf16(rng, (pool, Hkv, P, D))
    sig = rand_bf16(rng, (pool, Hkv, D))                 # stale rows: must stay unless touched
    kn = rand_bf16(rng, (B, max_new, Hkv, D))
    vn = rand_bf16(rng, (B, max_new, Hkv, D))
    return k, v, sig, pt, np.array(lens, dtype=np.int32), kn, vn


def test_append_kv_against_positions_and_exact_means():
    P = 4
    k, v, sig, pt, sl, kn, vn = _append_case(90, P=P)
    nn = np.array([3, 6, 2], dtype=np.int32)             # crosses page boundaries
    k2, v2, sig2, sl2 = O.append_kv(k, v, sig, pt, sl, kn, vn, nn, P)
    assert list(sl2) == list(sl + nn)
    written = set()
    for b in range(len(sl)):
        for i in range(int(nn[b])):
            pos = int(sl[b]) + i
            page, row = divmod(pos, P)                   # position -> (logical page, row)
            ph = int(pt[b, page])
            assert np.array_equal(k2[ph, :, row], kn[b, i])
            assert np.array_equal(v2[ph, :, row], vn[b, i])
            written.add((ph, row))
    for ph in range(k.shape[0]):                         # nothing else moved
        for row in range(P):
            if (ph, row) not in written:
                assert np.array_equal(k2[ph, :, row], k[ph, :, row])
                assert np.array_equal(v2[ph, :, row], v[ph, :, row])
    touched = {int(pt[b, (int(sl[b]) + i) // P]) for b in range(len(sl)) for i in range(int(nn[b]))}
    for ph in range(k.shape[0]):
        if ph not in touched:
            assert np.array_equal(sig2[ph], sig[ph])
            continue
        b, p = [(b, p) for b in range(len(sl)) for p in range(pt.shape[1]) if pt[b, p] == ph][0]
        nval = min(P, int(sl2[b]) - p * P)
        for h in range(k.shape[1]):
            for d in range(k.shape[3]):
                s = sum(bf16_fraction(k2[ph, h, j, d]) for j in range(nval))
                want = O.f64_to_bf16_rne(np.array([float(s) / nval]))[0]
                assert sig2[ph, h, d] == want


def test_append_kv_in_two_parts_equals_one_and_zero_is_identity():
    P = 4
    k, v, sig, pt, sl, kn, vn = _append_case(91, P=P)
    n1 = np.array([2, 1, 4], dtype=np.int32)
    n2 = np.array([3, 5, 1], dtype=np.int32)
    ka, va, sa_, la = O.append_kv(k, v, sig, pt, sl, kn, vn, n1 + n2, P)
    kb, vb, sb, lb = O.append_kv(k, v, sig, pt, sl, kn, vn, n1, P)
    kn2 = np.zeros_like(kn)
    vn2 = np.zeros_like(vn)
    for b in range(len(sl)):                             # the second part's tokens, shifted
        kn2[b, :n2[b]] = kn[b, n1[b]:n1[b] + n2[b]]
        vn2[b, :n2[b]] = vn[b, n1[b]:n1[b] + n2[b]]
    kc, vc, sc, lc = O.append_kv(kb, vb, sb, pt, lb, kn2, vn2, n2, P)
    assert np.array_equal(ka, kc) and np.array_equal(va, vc)
    assert np.array_equal(la, lc)
    # both touch the same pages (the union of the parts'), and a page only the
    # first part touches is full before the second part starts
    assert np.array_equal(sa_, sc)
    k0, v0, s0, l0 = O.append_kv(k, v, sig, pt, sl, kn, vn, np.zeros(3, np.int32), P)
    assert np.array_equal(k0, k) and np.array_equal(v0, v) and np.array_equal(s0, sig)
    assert np.array_equal(l0, sl)


# ----------------------------------------------------------------------------
# the ambient head set (reading R16: estimated attention-mass coverage)
# ----------------------------------------------------------------------------
def _bf16_of(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def _head_case(seed, B=2, T=2, Hq=6, Dk=8, P=4, lens=(22, 13)):
    rng = np.random.default_rng(seed)
    npg = [-(-L // P) for L in lens]
    pool = sum(npg)
    perm = rng.permutation(pool)
    pt = np.full((B, max(npg)), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(npg):
        pt[b, :n] = perm[off:off + n]
        off += n
    sig = _bf16_of(rng.integers(-3, 4, size=(pool, 1, Dk)))   # small integers: exact shifts
    q = _bf16_of(rng.integers(-2, 3, size=(B, T, Hq, Dk)))
    crit = [np.array([0, 2]), np.array([1])]
    amb = [np.array([0, 2, 3, 5]), np.array([1, 3])]            # crit + ambient, as tiered lists
    return q, sig, pt, np.array(lens, np.int32), crit, amb, npg


def _counts(lists):
    return np.array([len(x) for x in lists], dtype=np.int32)


def test_ambient_heads_equal_scores_give_the_token_share():
    # q = 0: every page's estimated mass is its token count, so each (b, t, h)
    # covers (ambient tokens) / (all tokens), the partial last page counted by its
    # valid tokens; all heads tie and the h lowest win
    q, sig, pt, sl, crit, amb, npg = _head_case(100)
    q[:] = 0
    P = 4
    sc = O.ambient_head_scores(q, sig, pt, sl, crit, _counts(crit), amb, _counts(amb), 0.7, P)
    want = 0.0
    for b, L in enumerate(sl):
        n = [min(P, int(L) - p * P) for p in range(npg[b])]
        amb_only = set(amb[b].tolist()) - set(crit[b].tolist())
        want += 2 * sum(n[p] for p in amb_only) / sum(n)          # T = 2 tokens
    assert np.allclose(sc, want, rtol=0, atol=1e-15)
    heads, _ = O.select_ambient_heads(q, sig, pt, sl, crit, _counts(crit), amb, _counts(amb),
                                      0.7, P, 3)
    assert list(heads) == [0, 1, 2]


def test_ambient_heads_follow_where_each_head_looks():
    # head 4 looks hard at an ambient page of each sequence, head 1 at a critical
    # one, the others see nothing (q = 0): head 4 covers ~1, head 1 ~0
    q, sig, pt, sl, crit, amb, npg = _head_case(101)
    q[:] = 0
    for b, (a_page, c_page) in enumerate(((3, 0), (3, 1))):
        q[b, :, 4, :] = sig[pt[b, a_page], 0, :]
        q[b, :, 1, :] = sig[pt[b, c_page], 0, :]
    sc = O.ambient_head_scores(q, sig, pt, sl, crit, _counts(crit), amb, _counts(amb), 40.0, 4)
    assert sc[4] > 4 - 1e-6 and sc[1] < 1e-6              # 2 sequences x 2 tokens
    heads, _ = O.select_ambient_heads(q, sig, pt, sl, crit, _counts(crit), amb, _counts(amb),
                                      40.0, 4, 2)
    assert 4 in heads and 1 not in heads
    # all heads and no head
    assert len(O.select_ambient_heads(q, sig, pt, sl, crit, _counts(crit), amb, _counts(amb),
                                      40.0, 4, 6)[0]) == 6
    assert len(O.select_ambient_heads(q, sig, pt, sl, crit, _counts(crit), amb, _counts(amb),
                                      40.0, 4, 0)[0]) == 0


def test_ambient_heads_invariant_to_page_ids_and_a_common_key_shift():
    q, sig, pt, sl, crit, amb, npg = _head_case(102)
    args = (crit, _counts(crit), amb, _counts(amb), 0.9, 4)
    base = O.ambient_head_scores(q, sig, pt, sl, *args)
    # relabel the physical pages
    perm = np.random.default_rng(5).permutation(sig.shape[0])
    inv = np.argsort(perm)
    sig2 = sig[perm]
    pt2 = np.where(pt >= 0, inv[np.clip(pt, 0, None)], -1).astype(np.int32)
    assert np.allclose(O.ambient_head_scores(q, sig2, pt2, sl, *args), base, rtol=1e-13, atol=0)
    # every summary moved by the same vector c: each row's scores move by q . c
    # on every page alike, which the softmax shares cancel (small integers: exact)
    c = np.array([1, -2, 0, 3, 1, 0, -1, 2], dtype=np.float32)
    sig3 = _bf16_of(O.bf16_to_f64(sig) + c[None, None, :])
    assert np.allclose(O.ambient_head_scores(q, sig3, pt, sl, *args), base, rtol=1e-12, atol=0)
