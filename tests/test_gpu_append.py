"""sa_append_kv against the oracle's append (marked gpu).

The new tokens land in their pages and the touched pages' summaries are
rewritten in the same launch; both the pools and the summaries must equal the
oracle's bit for bit, every other row must stay as it was, and the new lengths
come back in out_seq_lens.  Appends of 1, 3 and 40 tokens per sequence, a
ragged append (0, 1, 17 and 40 tokens), sequences that start empty or end
mid-page, pages of 16 and 64 tokens, a token-minor input layout (strides), and
tokens that fall past a sequence's page-table row (flagged and dropped).
"""
import numpy as np
import pytest
import torch

import oracle as O
import paged_sparse_kv_sa_b200 as sa

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def _case(seed, lens, max_new, P, Hkv, D, spare_pages=0):
    g = torch.Generator().manual_seed(seed)
    B = len(lens)
    npg = [-(-(L + max_new) // P) - spare_pages for L in lens]
    npg = [max(n, -(-L // P)) for n, L in zip(npg, lens)]
    pool = sum(npg) + 3
    perm = torch.randperm(pool, generator=g).numpy()
    pt = np.full((B, max(max(npg), 1)), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(npg):
        pt[b, :n] = perm[off:off + n]
        off += n
    k = _bits(torch.randn((pool, Hkv, P, D), generator=g).to(torch.bfloat16))
    v = _bits(torch.randn((pool, Hkv, P, D), generator=g).to(torch.bfloat16))
    sl = np.array(lens, dtype=np.int32)
    sig = O.page_summaries(k, pt, sl, P)
    kn = _bits(torch.randn((B, max_new, Hkv, D), generator=g).to(torch.bfloat16))
    vn = _bits(torch.randn((B, max_new, Hkv, D), generator=g).to(torch.bfloat16))
    return k, v, sig, pt, sl, kn, vn


def _run(k, v, sig, pt, sl, kn, vn, nn, token_minor=False):
    kd, vd, sd = _dev_bf16(k), _dev_bf16(v), _dev_bf16(sig)
    if token_minor:   # [B, Hkv, max_new, D] storage viewed as [B, max_new, Hkv, D]
        knd = _dev_bf16(np.ascontiguousarray(kn.transpose(0, 2, 1, 3))).permute(0, 2, 1, 3)
        vnd = _dev_bf16(np.ascontiguousarray(vn.transpose(0, 2, 1, 3))).permute(0, 2, 1, 3)
        assert not knd.is_contiguous()
    else:
        knd, vnd = _dev_bf16(kn), _dev_bf16(vn)
    out_len = torch.full((len(sl),), -1, dtype=torch.int32, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    sa.sa_append_kv(knd, vnd, torch.from_numpy(nn).to(DEV), kd, vd,
                    torch.from_numpy(pt).to(DEV), torch.from_numpy(sl).to(DEV), sd,
                    out_seq_lens=out_len, dev_error=err)
    torch.cuda.synchronize()
    return _bits(kd), _bits(vd), _bits(sd), out_len.cpu().numpy(), int(err.item())


@pytest.mark.parametrize("n,P,D,Hkv", [(1, 16, 128, 8), (3, 16, 128, 2), (40, 16, 64, 4),
                                       (40, 64, 128, 2), (3, 64, 64, 8)])
def test_append_matches_oracle(n, P, D, Hkv):
    lens = [0, P - 1, 5 * P, 3 * P + 7]
    k, v, sig, pt, sl, kn, vn = _case(100 + n + P, lens, 40, P, Hkv, D)
    nn = np.full(len(lens), n, dtype=np.int32)
    gk, gv, gs, gl, err = _run(k, v, sig, pt, sl, kn, vn, nn)
    rk, rv, rs, rl = O.append_kv(k, v, sig, pt, sl, kn, vn, nn, P)
    assert err == 0
    assert np.array_equal(gl, rl)
    assert np.array_equal(gk, rk) and np.array_equal(gv, rv)
    assert np.array_equal(gs, rs)


def test_append_ragged_and_strided_input():
    P, D, Hkv = 16, 128, 4
    lens = [100, 0, 31, 64]
    k, v, sig, pt, sl, kn, vn = _case(7, lens, 40, P, Hkv, D)
    nn = np.array([0, 1, 17, 40], dtype=np.int32)
    gk, gv, gs, gl, err = _run(k, v, sig, pt, sl, kn, vn, nn, token_minor=True)
    rk, rv, rs, rl = O.append_kv(k, v, sig, pt, sl, kn, vn, nn, P)
    assert err == 0
    assert np.array_equal(gl, rl)
    assert np.array_equal(gk, rk) and np.array_equal(gv, rv)
    assert np.array_equal(gs, rs)


def test_append_past_the_page_table_is_flagged_and_dropped():
    # each sequence has one page fewer than its append needs.  Sequence 0's row
    # ends in -1 padding (a page id outside the pool: SA_DEVERR_POOL_RANGE),
    # sequence 1's row is full (positions past it: SA_DEVERR_PAGE_RANGE); the
    # tokens without a page are dropped, every other one is written
    P, D, Hkv = 16, 64, 2
    lens = [10, 40]
    k, v, sig, pt, sl, kn, vn = _case(8, lens, 30, P, Hkv, D, spare_pages=1)
    assert list((pt >= 0).sum(axis=1)) == [2, 4] and pt.shape[1] == 4
    nn = np.array([30, 30], dtype=np.int32)
    gk, gv, gs, gl, err = _run(k, v, sig, pt, sl, kn, vn, nn)
    assert err & 3 == 3
    kept = np.array([2 * P - 10, 4 * P - 40], dtype=np.int32)   # tokens that have a page
    rk, rv, rs, rl = O.append_kv(k, v, sig, pt, sl, kn, vn, kept, P)
    assert np.array_equal(gk, rk) and np.array_equal(gv, rv)
    assert np.array_equal(gs, rs)
