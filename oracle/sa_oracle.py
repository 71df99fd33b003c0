"""Float64 CPU oracle: page scoring + top-k selection, sparse attention over
per-head page lists, LSE combine, block-union tables and page key summaries.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA library never
imports this module, and this module imports nothing from the library.

Sources (page title, then section):
  [UAE]   "Universal Attention Engine — Declarative Sparse Attention for
          Production": "The Product" (sink_tokens=32, local_window=512,
          cache_budget=1024), "Content-Dependent Dynamic Routing"
          (router = top_k_blocks(q @ mean(k_blocks)), selected blocks get full
          attention), "Architecture" (gather-based sparse KV decode over a
          PagedAttention-compatible layout), "Key Design Decisions" 3.
  [TS]    "TileSparse: Arithmetic-Intensity-Aware Sparse Attention for
          Compute-Bound LLM Decoding" (vllm README): "Motivation" (QK 2D
          sparsity; Critical Tier alpha pages x all heads, Ambient Tier beta
          pages x h heads), "Two implementations, by design" (mask-based path
          vs per-head page-list Flash-decode), "Configuration" (streaming mode).
  [CA]    CompactAttention abstract (on the page titled "Causal Attention on
          CPU: A Cache-Aware and Load-Balanced Scheduling Kernel for Prefill"):
          Block-Union KV Selection, Q-block union + intra-group union into
          GQA-aware per-group KV block tables, blocks used in place.
  [SPIN]  SPIN abstract (on the page titled "Vortex: Efficient and
          Programmable Sparse Attention Serving for AI Agents"): a two-level
          hierarchical page-metadata layout sized to the active working set.

Readings where the pages are silent (each also listed in the design notes):
  R1 page budget: n_sink = ceil(sink/P), n_local = ceil(local/P),
     budget_pages = floor(budget/P), k_top = budget_pages - n_sink - n_local;
     sink = logical pages [0, n_sink), local = the last n_local logical pages;
     N_b <= budget_pages selects every page.
  R2 summary of a (possibly partial) page: mean over its valid keys,
     sigma = RNE_bf16(RN64(RN64(exact sum) / n_valid)).
  R3 score of page p = max over the group's (token, head) query rows of the
     real dot product q . sigma_p, correctly rounded to float64, unscaled.
  R4 ties go to the lowest logical page index; output lists sorted ascending.
  R5 GQA head h reads kv head h // (Hq/Hkv).
  R6 query token t of a sequence of length L sits at position L - T + t and
     sees keys at positions <= its own (MTP and chunked prefill are causal).
  R7 MLA: one latent KV head, V = the first Dv columns of K, scale given by
     the caller (1/sqrt(Dk) in the workloads), selection pools all heads and
     tokens, no forced pages; critical = rank < alpha, ambient = next beta.
  R8 block union: sink block(s) + the Q-block's diagonal block + the top_k of
     the blocks strictly between them, by (score desc, index asc).
  R15 quantized KV pages ([UAE] "Key Design Decisions" 2: cache format
     (paged, block-sparse, quantized); "Roadmap": quantized KV cache support):
     K and V pages stored as FP8 E4M3 codes with one float32 scale per
     (physical page, kv head); a key is e4m3(code) * scale, likewise a value.
     Attention and summaries are those of the dequantized pages.
  R19 two-level page map ([SPIN] abstract on the page titled "Vortex:
     Efficient and Programmable Sparse Attention Serving for AI Agents": page
     metadata in two levels sized to the working set): a directory
     [B, n_dir] of block ids and blocks [n_blocks, 2^e] of physical page
     ids; logical page p of sequence b is blocks[dir[b, p >> e], p mod 2^e],
     and a directory entry that names no block gives no page (-1).  Every
     computation over such a map is the flat computation over the table it
     defines.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "bf16_to_f64", "f64_to_bf16_rne", "e4m3_to_f64", "page_budget", "exact_dots",
    "page_summaries", "page_summaries_fp8", "page_scores", "rank_select", "select_pages",
    "select_pages_mla", "sparse_attention", "sparse_attention_fp8", "masked_dense_attention",
    "combine", "block_union", "append_kv", "ambient_head_scores", "select_ambient_heads",
    "page_table_from_dir", "NEG_INF",
]

NEG_INF = float("-inf")


# --------------------------------------------------------------------------
# bf16 <-> float64 (IEEE-754 binary16 "brain" format: 1 sign, 8 exponent, 7 fraction bits)
# --------------------------------------------------------------------------
def bf16_to_f64(bits) -> np.ndarray:
    """Exact value of bf16 bit patterns: they are the top half of a binary32."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def f64_to_bf16_rne(x) -> np.ndarray:
    """Round float64 values to the nearest bf16, ties to even, in one rounding.

    The bf16 spacing at |x| in [2^(e-1), 2^e) is 2^(e-8), and 2^-133 below the
    normal range; x / spacing is exact (a power-of-two scale), ``np.rint``
    rounds it half-to-even, and the product is exactly representable.
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    ulp_exp = np.maximum(e.astype(np.int64) - 8, -133)
    scaled = np.ldexp(x, -ulp_exp)
    r = np.ldexp(np.rint(scaled), ulp_exp)
    if np.any(np.abs(r) > 3.3895313892515355e38):
        raise OverflowError("value outside the bf16 range")
    return (r.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# --------------------------------------------------------------------------
# FP8 E4M3 -> float64 (R15): 1 sign, 4 exponent (bias 7), 3 fraction bits;
# exponent field 0 holds the subnormals 2^-6 * f/8; S.1111.111 is NaN; no
# infinities (largest finite value 1.75 * 2^8 = 448)
# --------------------------------------------------------------------------
def e4m3_to_f64(codes) -> np.ndarray:
    """Exact value of FP8 E4M3 codes (NaN for the two NaN codes)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    f = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, np.ldexp(f / 8.0, -6), np.ldexp(1.0 + f / 8.0, e - 7))
    mag = np.where((c & 0x7F) == 0x7F, np.nan, mag)
    return sign * mag


def _dequant(codes, scale, phys, kvh):
    """float64 values of pages `phys` of kv head `kvh`: e4m3(code) * scale (R15).
    Each product is exact in float64 (4 x 24 significant bits)."""
    return e4m3_to_f64(codes[phys, kvh]) * np.asarray(scale, dtype=np.float32)[phys, kvh].astype(
        np.float64)[..., None, None]


# --------------------------------------------------------------------------
# R1: token budget -> page budget  ([UAE] "The Product": sink/local/cache_budget)
# --------------------------------------------------------------------------
def page_budget(sink_tokens: int, local_tokens: int, budget_tokens: int, page_size: int):
    """(n_sink, n_local, budget_pages, k_top) in pages, reading R1."""
    n_sink = -(-sink_tokens // page_size)
    n_local = -(-local_tokens // page_size)
    budget_pages = budget_tokens // page_size
    k_top = budget_pages - n_sink - n_local
    if k_top < 0:
        raise ValueError("sink + local pages exceed the page budget")
    return n_sink, n_local, budget_pages, k_top


# --------------------------------------------------------------------------
# exact sums of bf16 products, correctly rounded to float64
# --------------------------------------------------------------------------
def _exp_and_ulp(vals: np.ndarray):
    """For bf16-valued float64 entries: e with |v| < 2^e, and the exponent of
    their last significand bit (2^-133 for subnormals); zeros get (-inf, +inf)."""
    _, e = np.frexp(vals)
    e = e.astype(np.int64)
    u = np.maximum(e - 8, -133)
    nz = vals != 0
    return np.where(nz, e, -10 ** 6), np.where(nz, u, 10 ** 6)


def _exact_row_sums(terms: np.ndarray, e_hi: np.ndarray, u_lo: np.ndarray) -> np.ndarray:
    """RN64 of the exact sum over the last axis of exactly-representable terms.

    All terms are integer multiples of 2^min(u) and the running sums stay
    below 2^(max(e) + ceil(log2 n)); when that range spans <= 53 bits every
    partial sum is representable, so float64 summation in any order is exact.
    The rest are summed with ``math.fsum`` (correctly rounded).
    """
    n = terms.shape[-1]
    lg = int(math.ceil(math.log2(max(n, 1)))) + 1
    emax = e_hi.max(axis=-1)
    umin = u_lo.min(axis=-1)
    ok = (emax + lg - umin <= 53) | (emax < -10 ** 5)
    out = terms.sum(axis=-1)
    bad = np.argwhere(~ok)
    for idx in bad:
        idx = tuple(idx)
        out[idx] = math.fsum(terms[idx].tolist())
    return out


def exact_dots(A: np.ndarray, Bm: np.ndarray, chunk: int = 256) -> np.ndarray:
    """[na, nb] matrix of RN64(sum_d A[i,d] * B[j,d]) for bf16-valued A, B.

    Products of two bf16 values (8-bit significands) are exact in float64, so
    only the summation needs care (see ``_exact_row_sums``).
    """
    A = np.asarray(A, dtype=np.float64)
    Bm = np.asarray(Bm, dtype=np.float64)
    na, nb = A.shape[0], Bm.shape[0]
    out = np.empty((na, nb), dtype=np.float64)
    eA, uA = _exp_and_ulp(A)
    eB, uB = _exp_and_ulp(Bm)
    for j0 in range(0, nb, chunk):
        j1 = min(nb, j0 + chunk)
        P = A[:, None, :] * Bm[None, j0:j1, :]
        e_hi = eA[:, None, :] + eB[None, j0:j1, :]
        u_lo = uA[:, None, :] + uB[None, j0:j1, :]
        out[:, j0:j1] = _exact_row_sums(P, e_hi, u_lo)
    return out


# --------------------------------------------------------------------------
# R2: per-page key summaries  ([UAE] "Content-Dependent Dynamic Routing": mean(k_blocks))
# --------------------------------------------------------------------------
def page_summaries(k_bits, page_table, seq_lens, page_size: int, units=None) -> np.ndarray:
    """sigma [P_pool, Hkv, D] bf16 bits: for every page a sequence references,
    RNE_bf16(RN64(RN64(exact sum of its valid keys) / n_valid)); other rows 0.

    ``units``: optional iterable of (b, logical page) to restrict the work.
    """
    k_bits = np.asarray(k_bits, dtype=np.uint16)
    return _summaries(lambda phys, n: bf16_to_f64(k_bits[phys, :, :n, :]), k_bits.shape,
                      page_table, seq_lens, page_size, units)


def page_summaries_fp8(k_codes, k_scale, page_table, seq_lens, page_size: int,
                       units=None) -> np.ndarray:
    """page_summaries of FP8 pages (R15): the mean of the dequantized valid keys.

    All keys of a (page, kv head) share its scale, so the exact sum of the
    dequantized keys is scale * (exact sum of the E4M3 values); that product is
    exact in float64 (24 x 25 significant bits: at most 128 E4M3 values, each a
    multiple of 2^-9 below 2^9)."""
    k_codes = np.asarray(k_codes, dtype=np.uint8)
    assert k_codes.shape[2] <= 128
    sc = np.asarray(k_scale, dtype=np.float32).astype(np.float64)
    return _summaries(lambda phys, n: e4m3_to_f64(k_codes[phys, :, :n, :]), k_codes.shape,
                      page_table, seq_lens, page_size, units, post_scale=lambda phys: sc[phys])


def _summaries(keys_of, shape, page_table, seq_lens, page_size: int, units,
               post_scale=None) -> np.ndarray:
    pt = np.asarray(page_table, dtype=np.int64)
    sl = np.asarray(seq_lens, dtype=np.int64)
    P_pool, Hkv, P, D = shape
    assert P == page_size
    out = np.zeros((P_pool, Hkv, D), dtype=np.uint16)
    if units is None:
        units = [(b, p) for b in range(len(sl)) for p in range(-(-int(sl[b]) // P))]
    for b, p in units:
        n_valid = min(P, int(sl[b]) - p * P)
        if n_valid <= 0:
            continue
        phys = int(pt[b, p])
        keys = keys_of(phys, n_valid)                            # [Hkv, n_valid, D]
        terms = np.moveaxis(keys, 1, -1)                         # [Hkv, D, n_valid]
        e, u = _exp_and_ulp(terms)
        s = _exact_row_sums(terms.copy(), e, u)                  # [Hkv, D]
        if post_scale is not None:
            s = s * post_scale(phys)[:, None]
        out[phys] = f64_to_bf16_rne(s / float(n_valid))
    return out


# --------------------------------------------------------------------------
# R3/R4: scoring and top-k selection  ([UAE] "Content-Dependent Dynamic Routing")
# --------------------------------------------------------------------------
def page_scores(q_rows: np.ndarray, sig: np.ndarray) -> np.ndarray:
    """score_p = max_r RN64(q_r . sigma_p) over the group's query rows (R3)."""
    return exact_dots(q_rows, sig).max(axis=0)


def rank_select(scores: np.ndarray, idx: np.ndarray, k: int) -> np.ndarray:
    """Boolean mask of the k winners: item i wins iff fewer than k items j have
    (score_j > score_i) or (score_j == score_i and idx_j < idx_i)  (R4)."""
    n = len(scores)
    win = np.zeros(n, dtype=bool)
    if k <= 0 or n == 0:
        return win
    for i0 in range(0, n, 1024):
        i1 = min(n, i0 + 1024)
        si = scores[i0:i1, None]
        ii = idx[i0:i1, None]
        beats = (scores[None, :] > si) | ((scores[None, :] == si) & (idx[None, :] < ii))
        win[i0:i1] = beats.sum(axis=1) < k
    return win


def select_pages(q_bits, sig_bits, page_table, seq_lens, page_size: int, sink_tokens: int,
                 local_tokens: int, budget_tokens: int, units=None):
    """Per (b, kv head): forced sink/local pages plus the top k_top candidates.

    q_bits [B,T,Hq,D], sig_bits [P_pool,Hkv,D] (indexed by physical page),
    page_table [B,max_pages], seq_lens [B].  Returns pages [B,Hkv,budget_pages]
    (logical ids ascending, -1 padded) and counts [B,Hkv].  ``units``: optional
    list of (b, kvh) to compute; the others stay -1 / 0.
    """
    q = bf16_to_f64(q_bits)
    sig_bits = np.asarray(sig_bits, dtype=np.uint16)
    pt = np.asarray(page_table, dtype=np.int64)
    sl = np.asarray(seq_lens, dtype=np.int64)
    B, T, Hq, D = q.shape
    Hkv = sig_bits.shape[1]
    G = Hq // Hkv
    n_sink, n_local, budget_pages, k_top = page_budget(sink_tokens, local_tokens, budget_tokens,
                                                       page_size)
    pages = np.full((B, Hkv, max(budget_pages, 1)), -1, dtype=np.int32)
    counts = np.zeros((B, Hkv), dtype=np.int32)
    if units is None:
        units = [(b, h) for b in range(B) for h in range(Hkv)]
    for b, kvh in units:
        nb = -(-int(sl[b]) // page_size)
        if nb <= budget_pages:
            chosen = np.arange(nb)
        else:
            cand = np.arange(n_sink, nb - n_local)
            rows = q[b, :, kvh * G:(kvh + 1) * G, :].reshape(T * G, D)
            sig = bf16_to_f64(sig_bits[pt[b, cand], kvh, :])
            sc = page_scores(rows, sig)
            top = cand[rank_select(sc, cand, k_top)]
            chosen = np.concatenate([np.arange(n_sink), top, np.arange(nb - n_local, nb)])
        chosen = np.sort(chosen)
        pages[b, kvh, :len(chosen)] = chosen
        counts[b, kvh] = len(chosen)
    return pages, counts


def select_pages_mla(q_bits, sig_bits, page_table, seq_lens, page_size: int, alpha: int,
                     beta: int, units=None):
    """Tiered selection for one shared latent head ([TS] "Motivation", reading R7).

    Every logical page of the sequence is a candidate; the score takes the max
    over all T x Hq query rows.  Critical = the alpha best by (score desc,
    index asc), ambient = the next beta.  Returns crit [B,alpha], crit_counts,
    amb [B,beta], amb_counts, each list ascending and -1 padded.
    """
    q = bf16_to_f64(q_bits)
    sig_bits = np.asarray(sig_bits, dtype=np.uint16)
    pt = np.asarray(page_table, dtype=np.int64)
    sl = np.asarray(seq_lens, dtype=np.int64)
    B, T, Hq, Dk = q.shape
    crit = np.full((B, max(alpha, 1)), -1, dtype=np.int32)
    amb = np.full((B, max(beta, 1)), -1, dtype=np.int32)
    cc = np.zeros(B, dtype=np.int32)
    ac = np.zeros(B, dtype=np.int32)
    for b in (range(B) if units is None else units):
        nb = -(-int(sl[b]) // page_size)
        cand = np.arange(nb)
        rows = q[b].reshape(T * Hq, Dk)
        sig = bf16_to_f64(sig_bits[pt[b, cand], 0, :])
        sc = page_scores(rows, sig)
        in_crit = rank_select(sc, cand, alpha)
        in_both = rank_select(sc, cand, alpha + beta)
        c = np.sort(cand[in_crit])
        a = np.sort(cand[in_both & ~in_crit])
        crit[b, :len(c)] = c
        amb[b, :len(a)] = a
        cc[b], ac[b] = len(c), len(a)
    return crit, cc, amb, ac


# --------------------------------------------------------------------------
# sparse attention over per-head page lists  ([UAE] "Architecture": gather-based
# sparse KV decode; [TS] "Two implementations": per-head page-list Flash-decode)
# --------------------------------------------------------------------------
def _softmax_attend(s: np.ndarray, V: np.ndarray):
    """Natural-log LSE and softmax-weighted values of score rows s [R, n]
    (-inf entries excluded).  Rows with no finite score give O = 0, lse = -inf."""
    R = s.shape[0]
    o = np.zeros((R, V.shape[1]), dtype=np.float64)
    lse = np.full(R, NEG_INF, dtype=np.float64)
    for r in range(R):
        fin = np.isfinite(s[r])
        if not fin.any():
            continue
        m = s[r, fin].max()
        w = np.exp(s[r, fin] - m)
        tot = w.sum()
        lse[r] = m + math.log(tot)
        o[r] = (w / tot) @ V[fin]
    return o, lse


def sparse_attention(q_bits, k_bits, v_bits, page_table, seq_lens, lists, counts, head_to_list,
                     scale: float, page_size: int, rows=None, q_pos=None):
    """O [B,T,Hq,Dv] and lse [B,T,Hq] (float64) of softmax attention over the
    keys of each head's page list (reading R6 for the causal positions, R5 for
    the kv head).  Keys are the list's tokens at positions < L_b and <= the
    query's position L_b - T + t (or q_pos[b] + t when the positions are given:
    a prompt chunk computed while the cache already holds tokens past it).
    s_j = scale * q . k_j; an empty key set gives O = 0, lse = -inf.

    q_bits [B,T,Hq,Dk]; k_bits [P_pool,Hkv,P,Dk]; v_bits [P_pool,Hkv,P,Dv];
    lists [B,n_lists,max_list] logical page ids; counts [B,n_lists];
    head_to_list [Hq] (or [B,Hq]).  ``rows``: optional iterable of (b, t, h)
    to compute; the others stay 0 / -inf.
    """
    k_bits = np.asarray(k_bits, dtype=np.uint16)
    v_bits = np.asarray(v_bits, dtype=np.uint16)
    return _sparse_attention(q_bits, lambda phys, kvh: bf16_to_f64(k_bits[phys, kvh]),
                             lambda phys, kvh: bf16_to_f64(v_bits[phys, kvh]), k_bits.shape[1],
                             v_bits.shape[-1], page_table, seq_lens, lists, counts,
                             head_to_list, scale, page_size, rows, q_pos)


def sparse_attention_fp8(q_bits, k_codes, k_scale, v_codes, v_scale, page_table, seq_lens, lists,
                         counts, head_to_list, scale: float, page_size: int, rows=None):
    """sparse_attention over FP8 pages (R15): keys e4m3(k_codes) * k_scale[page,
    kv head], values e4m3(v_codes) * v_scale[page, kv head]; k_codes/v_codes
    [P_pool,Hkv,P,D] uint8, scales [P_pool,Hkv] float32."""
    k_codes = np.asarray(k_codes, dtype=np.uint8)
    v_codes = np.asarray(v_codes, dtype=np.uint8)
    return _sparse_attention(q_bits, lambda phys, kvh: _dequant(k_codes, k_scale, phys, kvh),
                             lambda phys, kvh: _dequant(v_codes, v_scale, phys, kvh),
                             k_codes.shape[1], v_codes.shape[-1], page_table, seq_lens, lists,
                             counts, head_to_list, scale, page_size, rows)


def _sparse_attention(q_bits, k_of, v_of, Hkv, Dv, page_table, seq_lens, lists, counts,
                      head_to_list, scale, page_size, rows, q_pos=None):
    q = bf16_to_f64(q_bits)
    pt = np.asarray(page_table, dtype=np.int64)
    sl = np.asarray(seq_lens, dtype=np.int64)
    lists = np.asarray(lists, dtype=np.int64)
    counts = np.asarray(counts, dtype=np.int64)
    h2l = np.asarray(head_to_list, dtype=np.int64)
    B, T, Hq, Dk = q.shape
    G = Hq // Hkv
    P = page_size
    O = np.zeros((B, T, Hq, Dv), dtype=np.float64)
    L = np.full((B, T, Hq), NEG_INF, dtype=np.float64)
    want = None if rows is None else {tuple(int(x) for x in r) for r in rows}
    for b in range(B):
        Lb = int(sl[b])
        hl = h2l[b] if h2l.ndim == 2 else h2l
        groups = {}
        for h in range(Hq):
            groups.setdefault((int(hl[h]), h // G), []).append(h)
        for (li, kvh), heads in groups.items():
            pages = lists[b, li, :int(counts[b, li])]
            phys = pt[b, pages]
            pos = (pages[:, None] * P + np.arange(P)[None, :]).reshape(-1)
            K = k_of(phys, kvh).reshape(-1, Dk)
            V = v_of(phys, kvh).reshape(-1, Dv)
            valid = pos < Lb
            pos, K, V = pos[valid], K[valid], V[valid]
            for t in range(T):
                hs = [h for h in heads if want is None or (b, t, h) in want]
                if not hs:
                    continue
                qpos = (Lb - T if q_pos is None else int(q_pos[b])) + t
                s = scale * (q[b, t, hs, :] @ K.T) if len(pos) else np.zeros((len(hs), 0))
                s = np.where((pos <= qpos)[None, :], s, NEG_INF) if len(pos) else s
                o, lse = _softmax_attend(s, V)
                O[b, t, hs] = o
                L[b, t, hs] = lse
    return O, L


def masked_dense_attention(q_bits, k_bits, v_bits, page_table, seq_lens, lists, counts,
                           head_to_list, scale: float, page_size: int):
    """The mask-based formulation ([TS] "Two implementations, by design"): full
    scores over every key of the sequence, then -inf for keys whose logical
    page is not in the head's list, and causal masking as in R6."""
    q = bf16_to_f64(q_bits)
    K_all = bf16_to_f64(k_bits)
    V_all = bf16_to_f64(v_bits)
    pt = np.asarray(page_table, dtype=np.int64)
    sl = np.asarray(seq_lens, dtype=np.int64)
    lists = np.asarray(lists, dtype=np.int64)
    counts = np.asarray(counts, dtype=np.int64)
    h2l = np.asarray(head_to_list, dtype=np.int64)
    B, T, Hq, Dk = q.shape
    Hkv = K_all.shape[1]
    Dv = V_all.shape[-1]
    G = Hq // Hkv
    P = page_size
    O = np.zeros((B, T, Hq, Dv))
    L = np.full((B, T, Hq), NEG_INF)
    for b in range(B):
        Lb = int(sl[b])
        nb = -(-Lb // P)
        phys = pt[b, :nb]
        pos = np.arange(nb * P)
        hl = h2l[b] if h2l.ndim == 2 else h2l
        for h in range(Hq):
            kvh = h // G
            K = K_all[phys, kvh].reshape(nb * P, Dk)
            V = V_all[phys, kvh].reshape(nb * P, Dv)
            li = int(hl[h])
            keep_page = np.zeros(nb, dtype=bool)
            keep_page[lists[b, li, :int(counts[b, li])]] = True
            keep = np.repeat(keep_page, P) & (pos < Lb)
            for t in range(T):
                s = scale * (K @ q[b, t, h])
                s = np.where(keep & (pos <= Lb - T + t), s, NEG_INF)
                o, lse = _softmax_attend(s[None, :], V)
                O[b, t, h] = o[0]
                L[b, t, h] = lse[0]
    return O, L


# --------------------------------------------------------------------------
# LSE combine of split partials (the merge step of a split-KV Flash-decode,
# [TS] "Configuration": full = fused Flash-decode)
# --------------------------------------------------------------------------
def combine(o_parts: np.ndarray, lse_parts: np.ndarray):
    """o_parts [S, ..., Dv] (each normalised over its own keys), lse_parts [S, ...].
    lse = log sum_s exp(lse_s); O = sum_s exp(lse_s - lse) O_s; splits with
    lse_s = -inf weigh 0; if every split is empty, O = 0 and lse = -inf."""
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m = lse_parts.max(axis=0)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    w = np.exp(lse_parts - m_safe[None])
    tot = w.sum(axis=0)
    lse = np.where(empty, NEG_INF, m_safe + np.log(np.where(empty, 1.0, tot)))
    scale = np.where(empty[None], 0.0, w / np.where(empty, 1.0, tot)[None])
    O = (scale[..., None] * o_parts).sum(axis=0)
    return O, lse


# --------------------------------------------------------------------------
# R8: block-union KV tables for chunked prefill ([CA] Block-Union KV Selection)
# --------------------------------------------------------------------------
def block_union(scores, Hkv: int, q_block_offset: int, top_k: int, n_sink_blocks: int = 1):
    """scores [Hq, NQB, NKB] float32.  For head h and Q-block j the mask is the
    sink blocks [0, n_sink), the diagonal block d = q_block_offset + j, and the
    top_k of the blocks [n_sink, d) by (score desc, index asc).  Table of group
    g = union over its heads h (h // (Hq/Hkv) == g) and all Q-blocks, ascending.
    Returns tables [Hkv, NKB] (-1 padded) and counts [Hkv]."""
    s = np.asarray(scores, dtype=np.float32)
    Hq, NQB, NKB = s.shape
    G = Hq // Hkv
    tables = np.full((Hkv, NKB), -1, dtype=np.int32)
    counts = np.zeros(Hkv, dtype=np.int32)
    for g in range(Hkv):
        keep = np.zeros(NKB, dtype=bool)
        for h in range(g * G, (g + 1) * G):
            for j in range(NQB):
                d = q_block_offset + j
                keep[:min(n_sink_blocks, d + 1)] = True
                keep[d] = True
                cand = np.arange(n_sink_blocks, d)
                if len(cand):
                    win = rank_select(s[h, j, cand].astype(np.float64), cand, top_k)
                    keep[cand[win]] = True
        ids = np.nonzero(keep)[0]
        tables[g, :len(ids)] = ids
        counts[g] = len(ids)
    return tables, counts


# --------------------------------------------------------------------------
# R19: the two-level page map ([SPIN]: metadata sized to the working set)
# --------------------------------------------------------------------------
def page_table_from_dir(page_dir, page_blocks, block_shift: int) -> np.ndarray:
    """The flat page table [B, n_dir * 2^e] a two-level map defines (e =
    block_shift): entry (b, p) is page_blocks[page_dir[b, p >> e], p mod 2^e]
    when that directory entry is a block id in [0, n_blocks), else -1."""
    d = np.asarray(page_dir, dtype=np.int64)
    blk = np.asarray(page_blocks, dtype=np.int64).reshape(-1, 1 << block_shift)
    n_blocks = blk.shape[0]
    B, n_dir = d.shape
    width = 1 << block_shift
    out = np.full((B, n_dir * width), -1, dtype=np.int32)
    for b in range(B):
        for j in range(n_dir):
            if 0 <= d[b, j] < n_blocks:
                out[b, j * width:(j + 1) * width] = blk[d[b, j]]
    return out


# --------------------------------------------------------------------------
# appending tokens to the paged cache ([UAE] "Content-Dependent Dynamic
# Routing": the router reads mean(k_blocks), so a block's summary changes when
# tokens land in it; "Architecture": a PagedAttention-compatible cache)
# --------------------------------------------------------------------------
def append_kv(k_bits, v_bits, sig_bits, page_table, seq_lens, k_new_bits, v_new_bits, n_new,
              page_size: int):
    """New pools, summaries and lengths after sequence b appends its n_new[b]
    tokens (k_new[b, i], v_new[b, i] for i < n_new[b]; [B, max_new, Hkv, D] bf16
    bits) at positions seq_lens[b] + i, i.e. page page_table[b, pos // P], row
    pos % P.  The summaries of the pages those positions fall in are recomputed
    from their definition (page_summaries over the new lengths); every other row
    of the pools and of the summaries is left as it was."""
    k = np.array(k_bits, dtype=np.uint16, copy=True)
    v = np.array(v_bits, dtype=np.uint16, copy=True)
    sig = np.array(sig_bits, dtype=np.uint16, copy=True)
    pt = np.asarray(page_table, dtype=np.int64)
    sl = np.asarray(seq_lens, dtype=np.int64)
    nn = np.asarray(n_new, dtype=np.int64)
    kn = np.asarray(k_new_bits, dtype=np.uint16)
    vn = np.asarray(v_new_bits, dtype=np.uint16)
    P = page_size
    touched = set()
    for b in range(len(sl)):
        for i in range(int(nn[b])):
            pos = int(sl[b]) + i
            ph = int(pt[b, pos // P])
            k[ph, :, pos % P, :] = kn[b, i]
            v[ph, :, pos % P, :] = vn[b, i]
            touched.add((b, pos // P))
    new_lens = sl + nn
    fresh = page_summaries(k, pt, new_lens, P, units=sorted(touched))
    for b, p in touched:
        ph = int(pt[b, p])
        sig[ph] = fresh[ph]
    return k, v, sig, new_lens.astype(np.int32)


# --------------------------------------------------------------------------
# R16: the ambient head set ([TS] "Motivation": the Ambient Tier is computed
# with h heads; "Configuration": an AutoTuner picks them per layer by
# estimated attention-mass coverage)
# --------------------------------------------------------------------------
def ambient_head_scores(q_bits, sig_bits, page_table, seq_lens, crit_lists, crit_counts,
                        amb_lists, amb_counts, scale: float, page_size: int):
    """Estimated attention-mass coverage of the ambient pages per head (R16).

    For sequence b, query token t and head h, page p of the sequence (all
    N_b pages, one latent kv head) carries the estimated mass
    m_p = n_p * exp(scale * (q[b,t,h] . sigma_p)), n_p its valid tokens: every
    key of the page replaced by the page's mean key.  The coverage of (b, t, h)
    is sum over ambient pages of m_p / sum over all pages of m_p; a head's score
    is the sum of its coverages over b and t.  Dots are the exact ones rounded to
    float64 (exact_dots), the rest float64.  Returns scores [Hq] float64."""
    q = bf16_to_f64(q_bits)
    sig = np.asarray(sig_bits, dtype=np.uint16)
    pt = np.asarray(page_table, dtype=np.int64)
    sl = np.asarray(seq_lens, dtype=np.int64)
    B, T, Hq, Dk = q.shape
    P = page_size
    scores = np.zeros(Hq, dtype=np.float64)
    for b in range(B):
        L = int(sl[b])
        nb = -(-L // P)
        if nb == 0:
            continue
        pages = np.arange(nb)
        n_p = np.minimum(P, L - pages * P).astype(np.float64)
        amb = np.zeros(nb, dtype=bool)
        amb[np.asarray(amb_lists[b][:int(amb_counts[b])], dtype=np.int64)] = True
        crit = np.asarray(crit_lists[b][:int(crit_counts[b])], dtype=np.int64)
        amb[crit] = False                                   # ambient = the tier past critical
        s = bf16_to_f64(sig[pt[b, pages], 0, :])            # [nb, Dk]
        dots = exact_dots(q[b].reshape(T * Hq, Dk), s)      # [T*Hq, nb]
        z = scale * dots
        m = z.max(axis=1, keepdims=True)
        w = n_p[None, :] * np.exp(z - m)
        cov = w[:, amb].sum(axis=1) / w.sum(axis=1)
        scores += cov.reshape(T, Hq).sum(axis=0)
    return scores


def select_ambient_heads(q_bits, sig_bits, page_table, seq_lens, crit_lists, crit_counts,
                         amb_lists, amb_counts, scale: float, page_size: int, h: int):
    """The h heads of largest ambient coverage (R16), ties to the lower head,
    ascending; and the scores."""
    sc = ambient_head_scores(q_bits, sig_bits, page_table, seq_lens, crit_lists, crit_counts,
                             amb_lists, amb_counts, scale, page_size)
    heads = np.arange(len(sc))
    win = rank_select(sc, heads, h)
    return heads[win].astype(np.int32), sc
