"""Seeded synthetic inputs for paged sparse-KV attention.

This module only draws random numbers and lays them out (pools, page tables,
sequence lengths, block scores).  It holds none of the attention, selection,
summary or combine arithmetic: both the CUDA path and the float64 oracle take
the tensors it returns as plain data.

Every tensor is drawn with ``torch.Generator(device).manual_seed(seed)``
(float32 N(0,1) rounded to bf16 by torch's round-to-nearest-even), on the
device the caller names: the CPU for the small cases the oracle finishes in
seconds, the GPU for the multi-GiB pools.  The same seed on a different
device gives different (but equally distributed) values; each run hands the
exact tensors it generated to both sides.

Workload shapes follow the decode, MLA and chunked-prefill settings the
sparse-attention pages describe: the sink 32 / local 512 / budget 1024 token
pattern of the Universal Attention Engine spec ("The Product"), the
critical/ambient tiers of TileSparse ("Motivation"), and CompactAttention's
block-union chunked prefill at 128K context.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Optional

import torch


# --------------------------------------------------------------------------
# workload descriptions
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class GQADecode:
    """Sparse GQA decode over a paged cache (T query tokens per sequence)."""
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    page_size: int
    seq_len_lo: int
    seq_len_hi: int            # inclusive; equal to seq_len_lo for a fixed length
    sink_tokens: int
    local_tokens: int
    budget_tokens: int
    T: int = 1
    table: str = "shuffled"    # "identity" | "shuffled" (pool = sum of pages, random permutation)
    lift_frac: float = 0.0     # fraction of pages per (b, kv-head) whose keys move along the group query
    lift_sigma: float = 0.0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv


@dataclass(frozen=True)
class MLADecode:
    """MLA + MTP decode: one shared latent KV head, V = first Dv columns of K."""
    name: str
    B: int
    T: int
    Hq: int
    Dk: int
    Dv: int
    page_size: int
    seq_len: int
    alpha: int                 # critical tier pages (all heads)
    beta: int                  # ambient tier pages (h heads)
    h_ambient: int
    Hkv: int = 1


@dataclass(frozen=True)
class BlockUnionPrefill:
    """Chunked prefill over block-union KV tables (blocks = pages of block tokens)."""
    name: str
    Hq: int
    Hkv: int
    D: int
    block: int
    chunk: int                 # query tokens in the chunk
    q_offset: int              # position of the first chunk token
    top_k: int
    n_sink_blocks: int = 1

    @property
    def kv_len(self) -> int:
        return self.q_offset + self.chunk

    @property
    def n_q_blocks(self) -> int:
        return self.chunk // self.block

    @property
    def n_kv_blocks(self) -> int:
        return (self.kv_len + self.block - 1) // self.block


TINY_GQA = GQADecode("tiny_gqa_b1_hq8_hkv2_d64_p16_l2048", B=1, Hq=8, Hkv=2, D=64, page_size=16,
                     seq_len_lo=2048, seq_len_hi=2048, sink_tokens=32, local_tokens=64,
                     budget_tokens=256, table="identity")
LLAMA8B_DECODE = GQADecode("llama8b_decode_b16_hq32_hkv8_d128_p16_l32768", B=16, Hq=32, Hkv=8, D=128,
                           page_size=16, seq_len_lo=32768, seq_len_hi=32768, sink_tokens=32,
                           local_tokens=512, budget_tokens=1024, table="shuffled",
                           lift_frac=0.05, lift_sigma=3.0)
LLAMA70B_LONG = GQADecode("llama70b_long_b32_hq64_hkv8_d128_p16_l64k-128k", B=32, Hq=64, Hkv=8, D=128,
                          page_size=16, seq_len_lo=65536, seq_len_hi=131072, sink_tokens=32,
                          local_tokens=512, budget_tokens=2048, table="shuffled")
MLA_MTP = MLADecode("mla_mtp_b8_t2_hq128_dk576_dv512_p64_l65536", B=8, T=2, Hq=128, Dk=576, Dv=512,
                    page_size=64, seq_len=65536, alpha=8, beta=24, h_ambient=32)
# Million-token page tables (SPIN's two-level metadata, on the page titled
# "Vortex: Efficient and Programmable Sparse Attention Serving for AI Agents"):
# 8 sequences of 64K to 1M tokens in 64-token pages, their page maps as
# directories over blocks of 64 pages (block_shift 6); the UAE sink / local
# pattern with a 2048-token budget.
LLAMA8B_DIR_1M = GQADecode("llama8b_dir_b8_hq32_hkv8_d128_p64_l64k-1m", B=8, Hq=32, Hkv=8, D=128,
                           page_size=64, seq_len_lo=65536, seq_len_hi=1048576, sink_tokens=64,
                           local_tokens=512, budget_tokens=2048, table="shuffled")
DIR_BLOCK_SHIFT = 6
UNION_PREFILL = BlockUnionPrefill("union_prefill_c2048_off126976_hq32_hkv8_d128_b64", Hq=32, Hkv=8,
                                  D=128, block=64, chunk=2048, q_offset=126976, top_k=8)


def scaled(cfg, **kw):
    """A copy of ``cfg`` with some fields replaced (smaller parity cases)."""
    return dataclasses.replace(cfg, **kw)


# --------------------------------------------------------------------------
# helpers
# --------------------------------------------------------------------------
def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn_bf16(shape, g, device) -> torch.Tensor:
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def _seq_lens(cfg: GQADecode, g, device) -> torch.Tensor:
    if cfg.seq_len_lo == cfg.seq_len_hi:
        return torch.full((cfg.B,), cfg.seq_len_lo, dtype=torch.int32, device=device)
    return torch.randint(cfg.seq_len_lo, cfg.seq_len_hi + 1, (cfg.B,), generator=g,
                         device=device, dtype=torch.int64).to(torch.int32)


def _page_table(n_pages: torch.Tensor, table: str, g, device):
    """Page table [B, max_pages] int32 (-1 past each sequence's pages) and pool size."""
    n_pages_l = [int(x) for x in n_pages.tolist()]
    B = len(n_pages_l)
    max_pages = max(n_pages_l) if n_pages_l else 0
    pool = sum(n_pages_l)
    pt = torch.full((B, max(max_pages, 1)), -1, dtype=torch.int32, device=device)
    if table == "identity":
        ids = torch.arange(pool, device=device, dtype=torch.int32)
    elif table == "shuffled":
        ids = torch.randperm(pool, generator=g, device=device).to(torch.int32)
    else:
        raise ValueError(table)
    off = 0
    for b, n in enumerate(n_pages_l):
        pt[b, :n] = ids[off:off + n]
        off += n
    return pt, pool


# --------------------------------------------------------------------------
# generators
# --------------------------------------------------------------------------
def gqa_decode_inputs(cfg: GQADecode, seed: int = 0, device="cpu", seq_lens: Optional[list] = None):
    """q [B,T,Hq,D], k/v pools [P_pool,Hkv,P,D] (bf16), page table [B,max_pages], seq_lens [B].

    ``lift_frac`` > 0: for each (b, kv-head) a seeded set of round(lift_frac * N_b) logical
    pages, drawn from all of the sequence's pages, has every key moved by
    ``lift_sigma`` along the unit vector of the group's mean query, then rounded
    back to bf16 (a planted set of pages that content-based scoring should find).
    """
    device = torch.device(device)
    g = _gen(device, seed)
    q = _randn_bf16((cfg.B, cfg.T, cfg.Hq, cfg.D), g, device)
    sl = (torch.tensor(seq_lens, dtype=torch.int32, device=device) if seq_lens is not None
          else _seq_lens(cfg, g, device))
    n_pages = (sl.to(torch.int64) + cfg.page_size - 1) // cfg.page_size
    pt, pool = _page_table(n_pages, cfg.table, g, device)
    pool = max(pool, 1)
    k = _randn_bf16((pool, cfg.Hkv, cfg.page_size, cfg.D), g, device)
    v = _randn_bf16((pool, cfg.Hkv, cfg.page_size, cfg.D), g, device)
    if cfg.lift_frac > 0:
        G = cfg.G
        for b in range(cfg.B):
            nb = int(n_pages[b])
            n_lift = int(round(cfg.lift_frac * nb))
            if n_lift == 0:
                continue
            for kvh in range(cfg.Hkv):
                qm = q[b, :, kvh * G:(kvh + 1) * G, :].float().reshape(-1, cfg.D).mean(0)
                u = qm / qm.norm()
                logical = torch.randperm(nb, generator=g, device=device)[:n_lift]
                phys = pt[b, logical].to(torch.int64)
                shifted = k[phys, kvh].float() + cfg.lift_sigma * u
                k[phys, kvh] = shifted.to(torch.bfloat16)
    return dict(q=q, k=k, v=v, page_table=pt, seq_lens=sl, pool=pool)


def page_directory(page_table: torch.Tensor, seq_lens: torch.Tensor, page_size: int,
                   block_shift: int, seed: int = 0):
    """A two-level page map holding ``page_table``: a directory [B, n_dir] of block
    ids (-1 where a run of 2^block_shift logical pages holds none of the
    sequence's pages) and blocks [n_blocks, 2^block_shift] of physical page ids
    (-1 past the sequence's last page).  Only the runs a sequence uses get a
    block; blocks are numbered in a seeded random order.  Pure layout: the
    table's entries are moved, not computed."""
    device = page_table.device
    B, W = page_table.shape
    width = 1 << block_shift
    n_dir = max(1, -(-W // width))
    n_pages = ((seq_lens.to(torch.int64) + page_size - 1) // page_size).tolist()
    runs = [(b, j) for b in range(B) for j in range(-(-int(n_pages[b]) // width))]
    g = _gen("cpu", seed)
    order = torch.randperm(max(len(runs), 1), generator=g)[:len(runs)].tolist()
    padded = torch.full((B, n_dir * width), -1, dtype=torch.int32, device=device)
    padded[:, :W] = page_table
    for b in range(B):   # entries past a sequence's pages stay -1
        padded[b, int(n_pages[b]):] = -1
    page_dir = torch.full((B, n_dir), -1, dtype=torch.int32)
    src = torch.empty(max(len(runs), 1), dtype=torch.int64)
    for (b, j), bid in zip(runs, order):
        page_dir[b, j] = bid
        src[bid] = b * n_dir + j
    blocks = torch.full((max(len(runs), 1), width), -1, dtype=torch.int32, device=device)
    if runs:
        blocks[:len(runs)] = padded.view(B * n_dir, width)[src[:len(runs)].to(device)]
    return page_dir.to(device), blocks


def fp8_pages(x):
    """FP8 E4M3 codes and per-(page, kv head) float32 scales of a bf16 pool x
    [P_pool, Hkv, P, D] (input preparation for the FP8-page workloads): scale =
    max |x| over the (page, kv head) / 448 (1 for an all-zero page), codes =
    x / scale rounded to the nearest E4M3 value (ties to even; torch's float8 cast),
    clamped to the format's +-448.  Returns (codes uint8, scales float32)."""
    xf = x.float()
    amax = xf.abs().amax(dim=(2, 3))
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    y = (xf / scale[:, :, None, None]).clamp(-448.0, 448.0)
    return y.to(torch.float8_e4m3fn).view(torch.uint8), scale.contiguous()


def mla_decode_inputs(cfg: MLADecode, seed: int = 0, device="cpu", seq_len: Optional[int] = None):
    """q [B,T,Hq,Dk], latent pool [P_pool,1,P,Dk] (V = first Dv columns), page table,
    seq_lens, and the ambient head set (``h_ambient`` sorted head ids, seeded)."""
    device = torch.device(device)
    g = _gen(device, seed)
    L = cfg.seq_len if seq_len is None else seq_len
    q = _randn_bf16((cfg.B, cfg.T, cfg.Hq, cfg.Dk), g, device)
    sl = torch.full((cfg.B,), L, dtype=torch.int32, device=device)
    n_pages = (sl.to(torch.int64) + cfg.page_size - 1) // cfg.page_size
    pt, pool = _page_table(n_pages, "shuffled", g, device)
    kv = _randn_bf16((max(pool, 1), 1, cfg.page_size, cfg.Dk), g, device)
    gh = _gen("cpu", seed + 1)
    amb = torch.randperm(cfg.Hq, generator=gh)[:cfg.h_ambient].sort().values.to(torch.int32)
    return dict(q=q, kv=kv, page_table=pt, seq_lens=sl, pool=max(pool, 1), ambient_heads=amb.to(device))


def block_union_scores(cfg: BlockUnionPrefill, seed: int = 0, device="cpu") -> torch.Tensor:
    """Block score matrix [Hq, n_q_blocks, n_kv_blocks] float32, i.i.d. N(0,1)."""
    g = _gen(torch.device(device), seed)
    return torch.randn((cfg.Hq, cfg.n_q_blocks, cfg.n_kv_blocks), generator=g,
                       device=device, dtype=torch.float32)


def prefill_inputs(cfg: BlockUnionPrefill, seed: int = 0, device="cpu"):
    """q [1,chunk,Hq,D], k/v block pools [n_kv_blocks,Hkv,block,D] (identity table), seq_lens."""
    device = torch.device(device)
    g = _gen(device, seed + 7)
    nkb = cfg.n_kv_blocks
    q = _randn_bf16((1, cfg.chunk, cfg.Hq, cfg.D), g, device)
    k = _randn_bf16((nkb, cfg.Hkv, cfg.block, cfg.D), g, device)
    v = _randn_bf16((nkb, cfg.Hkv, cfg.block, cfg.D), g, device)
    pt = torch.arange(nkb, dtype=torch.int32, device=device).reshape(1, nkb)
    sl = torch.tensor([cfg.kv_len], dtype=torch.int32, device=device)
    return dict(q=q, k=k, v=v, page_table=pt, seq_lens=sl, pool=nkb)


def bf16_bits(t: torch.Tensor):
    """The raw bf16 bit patterns of ``t`` as a numpy uint16 array (CPU copy)."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view("uint16")
