"""The whole GPU path at the full decode workload sizes vs the float64 oracle
(marked gpu and slow).

The GPU runs every stage over the whole batch exactly as the benchmark does
(summaries, page selection, split decode, merge); the oracle recomputes a
seeded sample of (sequence, kv head) units from the same generated tensors.
For a sampled unit the oracle sees only that unit's pages, as a local problem
(one sequence, one kv head, an identity page table over the unit's pages), which
gives the same selection and attention as the full batch: both only depend on
the unit's own pages, query rows and length.

  * summaries of every page of the unit: bit-exact;
  * the unit's selected page list and count: bit-exact;
  * O (float32) within 2e-3 and LSE within 1e-3 on every query row of the unit.

Workloads: the Llama-3-8B-shaped decode (16 sequences of 32768 tokens, 2048
pages each, 5% lifted pages, the benchmark's split count) and the
Llama-70B-shaped long decode (32 sequences of 65536-131072 tokens, 4096-8192
pages each, 128-page lists), the latter also with one split (a split holds the
whole 128-entry list) and with 13 splits, where the decode has more work items
(13 x 8 x 32 = 3328) than resident warps (12 per SM), so warps run several
items and carry their copy-ring phases from one item to the next.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import paged_sparse_kv_sa_b200 as sa
from paged_sparse_kv_sa_b200 import workloads as W

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

O_TOL = 2e-3
LSE_TOL = 1e-3


def _units(cfg, n, seed):
    """A seeded sample of (b, kv head) units, always with the first and last sequence."""
    rng = np.random.default_rng(seed)
    picks = {(0, int(rng.integers(cfg.Hkv))), (cfg.B - 1, int(rng.integers(cfg.Hkv)))}
    while len(picks) < n:
        picks.add((int(rng.integers(cfg.B)), int(rng.integers(cfg.Hkv))))
    return sorted(picks)


def _local_unit(inp, cfg, b, kvh):
    """The unit's pages as a local problem: q rows of the group [1,T,G,D], K and V
    [N,1,P,D] (bf16 bits), identity page table [1,N], seq_lens [1], and the
    physical ids of the pages (to index the GPU's summaries)."""
    L = int(inp["seq_lens"][b].item())
    N = -(-L // cfg.page_size)
    phys = inp["page_table"][b, :N].to(torch.int64)
    G = cfg.Hq // cfg.Hkv
    k = W.bf16_bits(inp["k"][phys, kvh].unsqueeze(1))
    v = W.bf16_bits(inp["v"][phys, kvh].unsqueeze(1))
    q = W.bf16_bits(inp["q"][b:b + 1, :, kvh * G:(kvh + 1) * G])
    pt = np.arange(N, dtype=np.int32).reshape(1, N)
    sl = np.array([L], dtype=np.int32)
    return q, k, v, pt, sl, phys


def _check_units(inp, cfg, sig, pages, counts, o, lse, units, scale):
    G = cfg.Hq // cfg.Hkv
    sig_cpu = sig  # indexed per unit below (device tensor)
    for b, kvh in units:
        q, k, v, pt, sl, phys = _local_unit(inp, cfg, b, kvh)
        ref_sig = O.page_summaries(k, pt, sl, cfg.page_size)            # [N, 1, D]
        got_sig = W.bf16_bits(sig_cpu[phys, kvh])                         # [N, D]
        assert np.array_equal(got_sig, ref_sig[:, 0]), f"summaries differ, unit {(b, kvh)}"
        rp, rc = O.select_pages(q, ref_sig, pt, sl, cfg.page_size, cfg.sink_tokens,
                                cfg.local_tokens, cfg.budget_tokens)
        gp = pages[b, kvh].cpu().numpy()
        gc = int(counts[b, kvh].item())
        assert gc == int(rc[0, 0]), f"count differs, unit {(b, kvh)}"
        assert np.array_equal(gp, rp[0, 0]), f"selection differs, unit {(b, kvh)}"
        ro, rl = O.sparse_attention(q, k, v, pt, sl, rp[:, :1], rc[:, :1], np.zeros(G, np.int64),
                                    scale, cfg.page_size)
        go = o[b:b + 1, :, kvh * G:(kvh + 1) * G].double().cpu().numpy()
        gl = lse[b:b + 1, :, kvh * G:(kvh + 1) * G].double().cpu().numpy()
        assert np.isfinite(rl).all() and np.isfinite(gl).all()
        err_o = float(np.abs(go - ro).max())
        err_l = float(np.abs(gl - rl).max())
        assert err_o <= O_TOL, f"max |O - O_ref| = {err_o}, unit {(b, kvh)}"
        assert err_l <= LSE_TOL, f"max |lse - lse_ref| = {err_l}, unit {(b, kvh)}"


def _run_path(cfg, inp, n_splits, attend):
    """summaries -> select -> decode -> merge over the whole batch on the GPU, with
    the benchmark's step object; attend=True merges inside the one-call entry."""
    sig = sa.sa_build_page_summaries(inp["k"], inp["page_table"], inp["seq_lens"])
    step = sa.SparseDecodeStep(cfg.B, cfg.T, cfg.Hq, cfg.Hkv, cfg.D, cfg.page_size,
                               inp["page_table"].shape[1], cfg.sink_tokens, cfg.local_tokens,
                               cfg.budget_tokens, n_splits=n_splits, device="cuda")
    step.dev_error.zero_()
    step.select(inp["q"], sig, inp["page_table"], inp["seq_lens"])
    if attend:
        step.attend(inp["q"], inp["k"], inp["v"], inp["page_table"], inp["seq_lens"])
    else:
        step.decode(inp["q"], inp["k"], inp["v"], inp["page_table"], inp["seq_lens"])
        step.combine()
    torch.cuda.synchronize()
    assert int(step.dev_error.item()) == 0
    return sig, step


def test_llama8b_workload_end_to_end_sampled():
    cfg = W.LLAMA8B_DECODE
    inp = W.gqa_decode_inputs(cfg, seed=0, device="cuda")
    sig, step = _run_path(cfg, inp, None, attend=False)
    # the split count the benchmark uses at this workload
    assert step.n_splits == sa.default_splits(cfg.B * cfg.Hkv, step.budget_pages)
    _check_units(inp, cfg, sig, step.pages, step.counts, step.o, step.lse,
                 _units(cfg, 12, seed=1), 1.0 / math.sqrt(cfg.D))
    # the one-call attention entry gives the same result on the same selection
    o2, _, lse2 = sa.sa_sparse_attention(inp["q"], inp["k"], inp["v"], inp["page_table"],
                                         inp["seq_lens"], step.pages, step.counts,
                                         step.head_to_list, step.scale, step.n_splits)
    torch.cuda.synchronize()
    assert torch.equal(o2, step.o) and torch.equal(lse2, step.lse)
    # and so does the one-call step (selection + attention + merge, sa_sparse_step)
    pages, counts, o_ref, lse_ref = (step.pages.clone(), step.counts.clone(), step.o.clone(),
                                     step.lse.clone())
    step.pages.fill_(-7)
    step.o.zero_()
    step.run(inp["q"], inp["k"], inp["v"], sig, inp["page_table"], inp["seq_lens"])
    torch.cuda.synchronize()
    assert torch.equal(step.pages, pages) and torch.equal(step.counts, counts)
    assert torch.equal(step.o, o_ref) and torch.equal(step.lse, lse_ref)


@pytest.fixture(scope="module")
def llama70b_inputs():
    cfg = W.LLAMA70B_LONG
    inp = W.gqa_decode_inputs(cfg, seed=0, device="cuda")
    yield cfg, inp
    del inp
    torch.cuda.empty_cache()


@pytest.mark.parametrize("n_splits,attend", [(None, False), (1, True), (13, True)])
def test_llama70b_workload_end_to_end_sampled(llama70b_inputs, n_splits, attend):
    cfg, inp = llama70b_inputs
    L = inp["seq_lens"].cpu()
    assert int(L.min()) >= 65536 and int(L.max()) <= 131072
    sig, step = _run_path(cfg, inp, n_splits, attend)
    if n_splits == 13:
        warps = 12 * torch.cuda.get_device_properties(0).multi_processor_count
        assert 13 * cfg.Hkv * cfg.B > warps      # several items per warp
    _check_units(inp, cfg, sig, step.pages, step.counts, step.o, step.lse,
                 _units(cfg, 8, seed=2 + (n_splits or 0)), 1.0 / math.sqrt(cfg.D))
