"""Benchmark: sparse-attention decode steps on the Llama-3-8B-shaped workload.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one pass of the whole hot path over one batch: page selection
(sa_select_pages), the gather split-KV decode (sa_sparse_decode) and the
split merge (sa_combine).  Workload: B=16 sequences of 32768 tokens, Hq=32,
Hkv=8, D=128, 16-token pages in a shuffled 2 GiB pool, budget 1024 tokens
(2 sink + 32 local + 30 top-k pages per kv head), 5% of pages per kv head
lifted 3 sigma along the group query; bf16 N(0,1) data, seed 0; summaries
built once by sa_build_page_summaries (not part of a step).

The metric is selected-KV GB/s: K+V bytes of the selected pages' valid
tokens per step divided by the step time (inputs resident in HBM, L2 flushed
before every timed step by writing a 256 MiB buffer and reading another
outside the timed events).  The line also carries calls/s, the decode
kernel's roofline fraction against the measured HBM copy bandwidth (with two
references beside it: a library copy of the same bytes in one launch, and
the event-timed cost of launching a one-element kernel), an end-to-end number
through the same API with the per-step inputs (q, page table, seq_lens)
copied from pinned host memory and the outputs (O, LSE) copied back inside
the timed region (each side packed into one buffer: one copy each way), and
the float64 oracle timed on a bounded sample on the host cores.

With --gpus N (torchrun), every rank runs its own batch of the same shape
(replicas: the path has no exchange step); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "selected-KV GB/s (fraction of HBM peak) and sparse-attn calls/sec at 1 B200"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--splits", type=int, default=0, help="decode split count (0 = heuristic)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--workload", choices=["llama8b", "llama70b", "mla", "prefill", "llama8b_fp8"],
                    default="llama8b",
                    help="llama8b (default, the headline workload); the others print the same "
                         "line for the Llama-70B long decode, MLA+MTP tiered decode and "
                         "block-union prefill workloads")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def selected_kv_bytes(counts, pages, seq_lens, P, D, elem_bytes=2):
    """K+V bytes of the valid tokens of every selected page (per step); FP8 pages
    (elem_bytes 1) add their two float32 scales per selected (page, kv head)."""
    import torch
    B, Hkv, cap = pages.shape
    L = seq_lens.to(torch.int64).view(B, 1, 1)
    idx = torch.arange(cap, device=pages.device).view(1, 1, cap)
    valid = idx < counts.view(B, Hkv, 1)
    p = pages.to(torch.int64).clamp_min(0)
    toks = (L - p * P).clamp(0, P)
    toks = torch.where(valid, toks, torch.zeros_like(toks))
    scales = int(valid.sum().item()) * 8 if elem_bytes == 1 else 0
    return int(toks.sum().item()) * D * elem_bytes * 2 + scales


def cpu_baseline(cfg, inp, sig_bits, n_units: int, budget_s: float = 20.0, f8=None,
                 min_s: float = 0.0):
    """Oracle (float64, host cores) on a bounded sample: n_units (b, kv head)
    pairs, select + attention (over FP8 pages when f8 holds their codes and
    scales), in repeated passes until min_s seconds have elapsed (and never
    past budget_s).  Returns GB/s of selected KV, units done, seconds."""
    import numpy as np

    import oracle as O
    from paged_sparse_kv_sa_b200 import workloads as W

    pt = inp["page_table"].cpu().numpy()
    sl = inp["seq_lens"].cpu().numpy()
    qb = W.bf16_bits(inp["q"])
    units = [(b, h) for b in range(cfg.B) for h in range(cfg.Hkv)][:n_units]
    G = cfg.G
    t0 = time.perf_counter()
    done, kv_bytes = 0, 0
    import itertools
    for (b, h) in itertools.cycle(units):   # (ends by the checks at the bottom)
        pages_np, counts_np = O.select_pages(qb, sig_bits, pt, sl, cfg.page_size, cfg.sink_tokens,
                                             cfg.local_tokens, cfg.budget_tokens, units=[(b, h)])
        lst = pages_np[b, h, :counts_np[b, h]]
        phys = pt[b, lst]
        # gather only this unit's pages from the device pool
        import torch
        loc_pt = np.full_like(pt, -1)
        loc_pt[b, lst] = np.arange(len(lst))
        lists = np.full((cfg.B, cfg.Hkv, pages_np.shape[2]), -1, dtype=np.int32)
        counts = np.zeros((cfg.B, cfg.Hkv), dtype=np.int32)
        lists[b, h, :len(lst)] = lst
        counts[b, h] = len(lst)
        rows = [(b, 0, hh) for hh in range(h * G, (h + 1) * G)]
        # gather only this unit's pages from the device pool
        ix = torch.as_tensor(phys, device=inp["q"].device)
        if f8 is None:
            O.sparse_attention(qb, W.bf16_bits(inp["k"][ix]), W.bf16_bits(inp["v"][ix]), loc_pt,
                               sl, lists, counts, np.arange(cfg.Hq) // G, 1.0 / math.sqrt(cfg.D),
                               cfg.page_size, rows=rows)
        else:
            O.sparse_attention_fp8(qb, f8["kc"][ix].cpu().numpy(), f8["ks"][ix].cpu().numpy(),
                                   f8["vc"][ix].cpu().numpy(), f8["vs"][ix].cpu().numpy(), loc_pt,
                                   sl, lists, counts, np.arange(cfg.Hq) // G,
                                   1.0 / math.sqrt(cfg.D), cfg.page_size, rows=rows)
        L = int(sl[b])
        eb = 2 if f8 is None else 1
        kv_bytes += sum(min(cfg.page_size, L - int(p) * cfg.page_size) for p in lst) * cfg.D * 2 * eb
        done += 1
        el = time.perf_counter() - t0
        if el > budget_s or (done % len(units) == 0 and el >= min_s):
            break
    dt = time.perf_counter() - t0
    return kv_bytes / dt / 1e9, done, dt


def _timed_graphs(g_step, g_kernel, K, flush_l2, stream, local):
    """Replay a whole-step graph and a single-kernel graph K times each, L2 flushed
    before every replay outside the events; device seconds for each, and clocks."""
    import torch
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(K):
            flush_l2(i)
            ev[i][0].record(stream)
            g_step.replay()
            ev[i][1].record(stream)
            flush_l2(i + 1)
            ev[i][2].record(stream)
            g_kernel.replay()
            ev[i][3].record(stream)
        torch.cuda.synchronize()
    t_step = sum(e[0].elapsed_time(e[1]) for e in ev) / 1e3
    t_kern = sum(e[2].elapsed_time(e[3]) for e in ev) / 1e3
    return t_step, t_kern, clk.summary()


def max_over_ranks(x: float, world: int, dev) -> float:
    """The largest of every rank's x: a multi-GPU job takes as long as its slowest
    rank (replicas: each rank runs its own batch; no data-path collective)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _packed(like, device):
    """One contiguous byte buffer holding tensors shaped like `like` back to back
    (16-byte aligned offsets; pinned when on the host), and a view of each: a
    step's inputs, or its outputs, then cross PCIe in one copy."""
    import torch
    offs, n = [], 0
    for t in like:
        n = (n + 15) // 16 * 16
        offs.append(n)
        n += t.numel() * t.element_size()
    host = torch.device(device).type == "cpu"
    buf = torch.empty(max(n, 16), dtype=torch.uint8, device=device, pin_memory=host)
    views = [buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
             for o, t in zip(offs, like)]
    return buf, views


def _launch_floor(flush_l2, stream, n):
    """Event-timed seconds of one graph-replayed launch of a one-element kernel, L2
    flushed first: the fixed cost inside every kernel time measured here (launch,
    first wave, drain, timestamp granularity)."""
    import torch
    x = torch.zeros(1, device=torch.device("cuda", torch.cuda.current_device()))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        x.add_(1.0)
    for _ in range(3):
        g.replay()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
    for i in range(n):
        flush_l2(i)
        ev[i][0].record(stream)
        g.replay()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in ev) / 1e3 / n


LAUNCH_FLOOR_WHAT = ("event-timed graph replay of a one-element kernel, L2 flushed: the fixed "
                     "cost inside every single-launch kernel time")


def _peak_tflops():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (burst)"
    return 1590.0, "fallback"


def run_extra(args, dev, world, rank, local, cores):
    """MLA+MTP tiered decode or block-union chunked prefill: same timing protocol."""
    import numpy as np
    import torch

    import paged_sparse_kv_sa_b200 as sa
    from paged_sparse_kv_sa_b200 import workloads as W

    if args.impl == "reference":
        print(json.dumps({"impl": "reference", "unavailable":
                          "the oracle arm is timed on the default (Llama-8B decode) workload"}))
        return
    sa.load()
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(64 * 1024 * 1024, dtype=torch.int32, device=dev)
    flush_sink = torch.empty((), dtype=torch.int64, device=dev)

    def flush_l2(i):
        flush.fill_(i & 0xFF)
        torch.sum(flush_rd, dim=0, dtype=torch.int64, out=flush_sink)

    K = args.steps
    if args.workload == "mla":
        cfg = W.MLA_MTP
        inp = W.mla_decode_inputs(cfg, seed=args.seed + rank, device=dev)
        q, kv, pt, sl = inp["q"], inp["kv"], inp["page_table"], inp["seq_lens"]
        sig = sa.sa_build_page_summaries(kv, pt, sl)
        amb = set(int(h) for h in inp["ambient_heads"].tolist())
        h2l = [1 if h in amb else 0 for h in range(cfg.Hq)]
        cap = cfg.alpha + cfg.beta
        lists = torch.empty((cfg.B, 2, cap), dtype=torch.int32, device=dev)
        counts = torch.empty((cfg.B, 2), dtype=torch.int32, device=dev)
        ws = torch.empty(max(int(sa.load().sa_select_tiered_workspace_size(
            cfg.B, cfg.T, cfg.Hq, pt.shape[1])), 16), dtype=torch.uint8, device=dev)
        n_splits = args.splits or 8
        o_p = torch.empty((n_splits, cfg.B, cfg.T, cfg.Hq, cfg.Dv), dtype=torch.float32, device=dev)
        l_p = torch.empty((n_splits, cfg.B, cfg.T, cfg.Hq), dtype=torch.float32, device=dev)
        o = torch.empty((cfg.B, cfg.T, cfg.Hq, cfg.Dv), dtype=torch.float32, device=dev)
        lse = torch.empty((cfg.B, cfg.T, cfg.Hq), dtype=torch.float32, device=dev)
        scale = 1.0 / math.sqrt(cfg.Dk)

        def select(qq, ptt, sll):
            sa.sa_select_pages_tiered(qq, sig, ptt, sll, cfg.page_size, cfg.alpha, cfg.beta,
                                      lists=lists, list_counts=counts, workspace=ws)

        def decode(qq, ptt, sll):
            sa.sa_sparse_decode(qq, kv, kv[..., :cfg.Dv], ptt, sll, lists, counts, h2l, scale,
                                n_splits, o_partial=o_p, lse_partial=l_p)

        step_inputs = (q, pt, sl)
        kern = "mla_kernel"
    else:
        cfg = W.UNION_PREFILL
        inp = W.prefill_inputs(cfg, seed=args.seed + rank, device=dev)
        q, kk, vv, pt, sl = inp["q"], inp["k"], inp["v"], inp["page_table"], inp["seq_lens"]
        scores = W.block_union_scores(cfg, seed=args.seed + rank, device=dev)
        off = cfg.q_offset // cfg.block
        tables = torch.empty((cfg.Hkv, cfg.n_kv_blocks), dtype=torch.int32, device=dev)
        tcounts = torch.empty((cfg.Hkv,), dtype=torch.int32, device=dev)
        h2l = [h // (cfg.Hq // cfg.Hkv) for h in range(cfg.Hq)]
        n_splits = args.splits or 2
        o_p = torch.empty((n_splits, 1, cfg.chunk, cfg.Hq, cfg.D), dtype=torch.float32, device=dev)
        l_p = torch.empty((n_splits, 1, cfg.chunk, cfg.Hq), dtype=torch.float32, device=dev)
        o = torch.empty((1, cfg.chunk, cfg.Hq, cfg.D), dtype=torch.float32, device=dev)
        lse = torch.empty((1, cfg.chunk, cfg.Hq), dtype=torch.float32, device=dev)
        scale = 1.0 / math.sqrt(cfg.D)

        def select(sc, ptt, sll):
            sa.sa_block_union(sc, cfg.Hkv, off, cfg.top_k, cfg.n_sink_blocks, tables=tables,
                              counts=tcounts)

        def decode(qq, ptt, sll):
            sa.sa_sparse_decode(qq, kk, vv, ptt, sll, tables.view(1, cfg.Hkv, -1),
                                tcounts.view(1, cfg.Hkv), h2l, scale, n_splits,
                                o_partial=o_p, lse_partial=l_p)

        step_inputs = (scores, pt, sl)
        kern = "prefill_kernel"

    def run_step(a0, ptt, sll, qq):
        select(a0, ptt, sll)
        decode(qq, ptt, sll)
        sa.sa_combine(o_p, l_p, o_out=o, lse_out=lse)

    first = step_inputs[0]
    for _ in range(max(args.warmup, 3)):
        run_step(first, pt, sl, q)
    torch.cuda.synchronize()

    # algorithmic work of one step (from the lists the step produced)
    if args.workload == "mla":
        L = sl.cpu().numpy()
        ls, cs = lists.cpu().numpy(), counts.cpu().numpy()
        flops, kv_bytes = 0, 0
        for b in range(cfg.B):
            for t in range(cfg.T):
                qpos = int(L[b]) - cfg.T + t
                for li, nh in ((0, cfg.Hq - len(amb)), (1, len(amb))):
                    pg = ls[b, li, :cs[b, li]].astype(np.int64)
                    keys = np.clip(np.minimum(qpos + 1, int(L[b])) - pg * cfg.page_size, 0,
                                   cfg.page_size).sum()
                    flops += 2 * nh * int(keys) * (cfg.Dk + cfg.Dv)
            pg = ls[b, 1, :cs[b, 1]].astype(np.int64)
            kv_bytes += int(np.clip(int(L[b]) - pg * cfg.page_size, 0, cfg.page_size).sum()) \
                * cfg.Dk * 2
    else:
        tb, tc_ = tables.cpu().numpy(), tcounts.cpu().numpy()
        G = cfg.Hq // cfg.Hkv
        qpos = cfg.q_offset + np.arange(cfg.chunk)
        flops, kv_bytes = 0, 0
        for g in range(cfg.Hkv):
            blk = tb[g, :tc_[g]].astype(np.int64)
            vis = np.clip(np.minimum(qpos[:, None] + 1, cfg.kv_len) - blk[None, :] * cfg.block, 0,
                          cfg.block).sum()
            flops += 2 * G * int(vis) * (2 * cfg.D)
            kv_bytes += int(np.clip(cfg.kv_len - blk * cfg.block, 0, cfg.block).sum()) \
                * cfg.D * 2 * 2

    g_step, g_kern = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step):
        run_step(first, pt, sl, q)
    with torch.cuda.graph(g_kern):
        decode(q, pt, sl)
    for _ in range(3):
        g_step.replay()
        g_kern.replay()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    t_step, t_kern, clocks = _timed_graphs(g_step, g_kern, K, flush_l2, stream, local)
    if world > 1:
        dist.barrier()

    # end to end through the same API: the step's inputs from pinned host memory
    # (packed: one host-to-device copy) and its outputs back (packed: one copy)
    srcs = (first, pt, sl) if first is q else (first, pt, sl, q)
    h_in, hosts = _packed(srcs, "cpu")
    for h_, x in zip(hosts, srcs):
        h_.copy_(x.cpu())
    d_in, devs = _packed(srcs, dev)
    d_out, (o, lse) = _packed((o, lse), dev)      # the step now writes these views
    h_out, (o_h, lse_h) = _packed((o, lse), "cpu")

    def e2e():
        d_in.copy_(h_in, non_blocking=True)
        run_step(devs[0], devs[1], devs[2], devs[-1] if len(devs) == 4 else devs[0])
        h_out.copy_(d_out, non_blocking=True)

    for _ in range(3):
        e2e()
    torch.cuda.synchronize()
    e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    for i in range(K):
        flush_l2(i)
        e_ev[i][0].record(stream)
        e2e()
        e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    t_e2e = sum(a.elapsed_time(b) for a, b in e_ev) / 1e3
    h2d = h_in.numel()
    d2h = h_out.numel()
    assert torch.isfinite(o).all().item(), "non-finite output"

    t_step = max_over_ranks(t_step, world, dev)
    t_e2e = max_over_ranks(t_e2e, world, dev)
    peak, kind = _peak_tflops()
    achieved = flops / (t_kern / K) / 1e12
    t_floor = _launch_floor(flush_l2, stream, min(K, 50))
    line = {
        "metric": METRIC, "value": round(world * kv_bytes * K / t_step / 1e9, 3), "unit": "GB/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": round(1e3 * t_step / K, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": cfg.name, "n_splits": n_splits,
                   "l2": "flushed before every timed step (256 MiB write, then 256 MiB read)"},
        "calls_per_sec": round(world * K / t_step, 2),
        "step_tflops": round(world * flops * K / t_step / 1e12, 2),
        "selected_kv_bytes_per_step": kv_bytes, "flops_per_step": flops,
        "roofline": {"kernel": kern, "bound": "tensor", "achieved": round(achieved, 2),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "peak_kind": kind, "traffic": None,
                     "kernel_ms": round(1e3 * t_kern / K, 4),
                     "launch_floor_us": round(1e6 * t_floor, 2),
                     "launch_floor_what": LAUNCH_FLOOR_WHAT},
        "e2e": {"value": round(world * kv_bytes * K / t_e2e / 1e9, 3), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(1e3 * t_e2e / K, 4)},
        "gpu_launches": (5 if args.workload == "prefill" else 4) * K,
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        del g_step, g_kern
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    import numpy as np
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference" and rank != 0:
        return                      # the oracle arm runs on rank 0 only
    if world > 1 and args.impl == "ours":
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    from paged_sparse_kv_sa_b200 import workloads as W

    cores = len(os.sched_getaffinity(0))
    if args.workload in ("mla", "prefill"):
        return run_extra(args, dev, world, rank, local, cores)
    cfg = {"llama8b": W.LLAMA8B_DECODE, "llama70b": W.LLAMA70B_LONG,
           "llama8b_fp8": W.LLAMA8B_DECODE}[args.workload]
    fp8 = args.workload == "llama8b_fp8"

    if args.impl == "reference":
        # the reference arm is the float64 oracle on the host cores
        import paged_sparse_kv_sa_b200 as sa
        sa.load()
        inp = W.gqa_decode_inputs(cfg, seed=args.seed, device=dev)
        f8 = None
        if fp8:
            kc, ks = W.fp8_pages(inp["k"])
            vc, vs = W.fp8_pages(inp["v"])
            f8 = dict(kc=kc, ks=ks, vc=vc, vs=vs)
            sig = sa.sa_build_page_summaries_fp8(kc, ks, inp["page_table"], inp["seq_lens"])
        else:
            sig = sa.sa_build_page_summaries(inp["k"], inp["page_table"], inp["seq_lens"])
        torch.cuda.synchronize()
        sig_bits = W.bf16_bits(sig)
        for _ in range(args.warmup):
            cpu_baseline(cfg, inp, sig_bits, 1, budget_s=5, f8=f8)
        tot_b, tot_t, units = 0.0, 0.0, 0
        for _ in range(args.steps):
            gbs, n, dt = cpu_baseline(cfg, inp, sig_bits, 2, budget_s=10, f8=f8)
            tot_b += gbs * dt
            tot_t += dt
            units += n
        val = tot_b / tot_t
        line = {"metric": METRIC, "value": round(val, 6), "unit": "GB/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(1000 * tot_t / args.steps, 3), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "impl": "reference",
                "config": {"workload": cfg.name + ("_fp8" if fp8 else ""), "B": cfg.B,
                           "seq_len": cfg.seq_len_lo,
                           "Hq": cfg.Hq, "Hkv": cfg.Hkv, "D": cfg.D, "page_size": cfg.page_size,
                           "budget_tokens": cfg.budget_tokens},
                "cpu_baseline": {"value": round(val, 6), "unit": "GB/s", "cores": cores,
                                 "kind": "oracle",
                                 "sample": f"{units} (sequence, kv head) units of select + "
                                           f"attention per {args.steps} steps"},
                "e2e": {"value": round(val, 6), "unit": "GB/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import paged_sparse_kv_sa_b200 as sa
    sa.load()
    inp = W.gqa_decode_inputs(cfg, seed=args.seed + rank, device=dev)
    q, k, v, pt, sl = inp["q"], inp["k"], inp["v"], inp["page_table"], inp["seq_lens"]
    f8 = None
    if fp8:
        # FP8 E4M3 pages with per-(page, kv head) scales, quantized from the bf16 pools
        kc, ks = W.fp8_pages(k)
        vc, vs = W.fp8_pages(v)
        f8 = dict(kc=kc, ks=ks, vc=vc, vs=vs)
        sig = sa.sa_build_page_summaries_fp8(kc, ks, pt, sl)
    else:
        sig = sa.sa_build_page_summaries(k, pt, sl)
    step = sa.SparseDecodeStep(cfg.B, cfg.T, cfg.Hq, cfg.Hkv, cfg.D, cfg.page_size, pt.shape[1],
                               cfg.sink_tokens, cfg.local_tokens, cfg.budget_tokens,
                               n_splits=args.splits or None, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(64 * 1024 * 1024, dtype=torch.int32, device=dev)
    flush_sink = torch.empty((), dtype=torch.int64, device=dev)

    def flush_l2(i):
        # write 256 MiB (evicts everything), then read 256 MiB of another buffer
        # so the dirty lines are written back now, not inside the timed step
        flush.fill_(i & 0xFF)
        torch.sum(flush_rd, dim=0, dtype=torch.int64, out=flush_sink)

    def decode_call(qq, ptt, sll):
        if fp8:
            step.decode_fp8(qq, kc, vc, ks, vs, ptt, sll)
        else:
            step.decode(qq, k, v, ptt, sll)

    def run_step():
        step.select(q, sig, pt, sl)
        decode_call(q, pt, sl)
        step.combine()

    for _ in range(max(args.warmup, 3)):
        run_step()
    torch.cuda.synchronize()
    kv_bytes = selected_kv_bytes(step.counts, step.pages, sl, cfg.page_size, cfg.D,
                                 elem_bytes=1 if fp8 else 2)
    q_bytes = q.numel() * 2
    part_bytes = step.o_part.numel() * 4 + step.lse_part.numel() * 4
    list_bytes = step.pages.numel() * 4 + step.counts.numel() * 4
    decode_alg_bytes = kv_bytes + q_bytes + part_bytes + list_bytes + \
        int(step.counts.sum().item()) * 4

    # Whole steps and the decode kernel alone are replayed from CUDA graphs, so
    # that the events bracket device work only (no host enqueue gaps).
    g_step = torch.cuda.CUDAGraph()
    g_dec = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step):
        run_step()
    with torch.cuda.graph(g_dec):
        decode_call(q, pt, sl)
    for _ in range(3):
        g_step.replay()
        g_dec.replay()
    torch.cuda.synchronize()
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(K):
            flush_l2(i)
            ev[i][0].record(stream)
            g_step.replay()
            ev[i][1].record(stream)
            flush_l2(i + 1)
            ev[i][2].record(stream)
            g_dec.replay()
            ev[i][3].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t_step = sum(e[0].elapsed_time(e[1]) for e in ev) / 1e3           # seconds, K steps
    t_dec = sum(e[2].elapsed_time(e[3]) for e in ev) / 1e3            # decode kernel alone
    # per-stage split of one eager step (informational)
    st_ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    flush_l2(0)
    st_ev[0].record(stream)
    step.select(q, sig, pt, sl)
    st_ev[1].record(stream)
    decode_call(q, pt, sl)
    st_ev[2].record(stream)
    step.combine()
    st_ev[3].record(stream)
    torch.cuda.synchronize()
    t_sel = st_ev[0].elapsed_time(st_ev[1]) / 1e3 * K
    t_cmb = st_ev[2].elapsed_time(st_ev[3]) / 1e3 * K
    t_step_max = max_over_ranks(t_step, world, dev)
    value = world * kv_bytes * K / t_step_max / 1e9
    calls_per_sec = world * K / t_step_max

    # ---- end to end through the same API: host inputs in, host outputs out
    # inputs packed in one pinned buffer (one host-to-device copy), outputs in one
    # device buffer the step writes (one device-to-host copy)
    h_in, (q_h, pt_h, sl_h) = _packed((q, pt, sl), "cpu")
    q_h.copy_(q.cpu())
    pt_h.copy_(pt.cpu())
    sl_h.copy_(sl.cpu())
    d_in, (q_d, pt_d, sl_d) = _packed((q, pt, sl), dev)
    d_out, (step.o, step.lse) = _packed((step.o, step.lse), dev)
    h_out, (o_h, lse_h) = _packed((step.o, step.lse), "cpu")

    def e2e_step():
        d_in.copy_(h_in, non_blocking=True)
        step.select(q_d, sig, pt_d, sl_d)
        decode_call(q_d, pt_d, sl_d)
        step.combine()
        h_out.copy_(d_out, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    e2e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    if world > 1:
        dist.barrier()
    for i in range(K):
        flush_l2(i)
        e2e_ev[i][0].record(stream)
        e2e_step()
        e2e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    t_e2e = sum(a.elapsed_time(b) for a, b in e2e_ev) / 1e3
    t_e2e = max_over_ranks(t_e2e, world, dev)
    e2e_value = world * kv_bytes * K / t_e2e / 1e9
    h2d = h_in.numel()
    d2h = h_out.numel()

    # correctness guard on what was timed: the outputs are finite and selections full
    assert torch.isfinite(step.o).all().item(), "non-finite output"
    assert int(step.dev_error.item()) == 0, "device error flag set"

    hbm_peak, peak_kind = peaks()
    dec_avg = t_dec / K
    achieved = decode_alg_bytes / dec_avg / 1e9
    # context for the roofline: one library device copy moving the same number
    # of bytes (half read, half written) in one launch, from its own graph with
    # L2 flushed first -- the kind of copy the peak is measured with, at this
    # size (a single launch pays a fixed cost that a multi-GiB copy hides)
    half = max(decode_alg_bytes // 2 // 16, 1)
    rd_buf = torch.ones((half, 4), dtype=torch.int32, device=dev)
    rd_out = torch.empty_like(rd_buf)
    g_rd = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_rd):
        rd_out.copy_(rd_buf)
    for _ in range(3):
        g_rd.replay()
    rd_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(min(K, 50))]
    for i in range(len(rd_ev)):
        flush_l2(i)
        rd_ev[i][0].record(stream)
        g_rd.replay()
        rd_ev[i][1].record(stream)
    torch.cuda.synchronize()
    t_rd = sum(a.elapsed_time(b) for a, b in rd_ev) / 1e3 / len(rd_ev)
    read_gbs = 2 * rd_buf.numel() * 4 / t_rd / 1e9
    del rd_buf, rd_out
    t_floor = _launch_floor(flush_l2, stream, min(K, 50))
    traffic = None
    tp = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if os.path.exists(tp):
        with open(tp) as f:
            td = json.load(f)
        if td.get("workload") == cfg.name and td.get("splits") == step.n_splits and not fp8:
            traffic = td.get("bytes_per_launch")

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(1e3 * t_step_max / K, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": cfg.name + ("_fp8" if fp8 else ""), "B": cfg.B,
                   "seq_len": cfg.seq_len_lo, "Hq": cfg.Hq,
                   "Hkv": cfg.Hkv, "D": cfg.D, "page_size": cfg.page_size,
                   "kv_pages": ("fp8 e4m3 + float32 scale per (page, kv head)" if fp8
                                else "bf16"),
                   "budget_tokens": cfg.budget_tokens, "sink_tokens": cfg.sink_tokens,
                   "local_tokens": cfg.local_tokens, "n_splits": step.n_splits,
                   "l2": "flushed before every timed step (256 MiB write, then 256 MiB read)",
                   "parallelism": f"replicas x{world}"},
        "calls_per_sec": round(calls_per_sec, 2),
        "stage_ms": {"select_eager": round(1e3 * t_sel / K, 4),
                     "decode_graph": round(1e3 * t_dec / K, 4),
                     "combine_eager": round(1e3 * t_cmb / K, 4)},
        "selected_kv_bytes_per_step": kv_bytes,
        "roofline": {"kernel": "decode_gqa_kernel" + ("<fp8>" if fp8 else ""), "bound": "hbm", "achieved": round(achieved, 2),
                     "peak": hbm_peak, "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
                     "peak_kind": peak_kind, "traffic": traffic,
                     "alg_bytes_per_launch": decode_alg_bytes,
                     "same_bytes_copy": {"gbs": round(read_gbs, 1),
                                         "what": "one device copy (torch copy_) moving the same "
                                                 "bytes, read + write, L2 flushed"},
                     "frac_of_same_bytes_copy": round(achieved / read_gbs, 4),
                     "kernel_us": round(1e6 * dec_avg, 2),
                     "launch_floor_us": round(1e6 * t_floor, 2),
                     "launch_floor_what": LAUNCH_FLOOR_WHAT},
        "e2e": {"value": round(e2e_value, 3), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "ms_per_step": round(1e3 * t_e2e / K, 4)},
        "gpu_launches": 4 * K,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n_all = cfg.B * cfg.Hkv
        gbs, n, dt = cpu_baseline(cfg, inp, W.bf16_bits(sig), n_units=n_all, budget_s=20.0, f8=f8,
                                  min_s=10.0)
        line["cpu_baseline"] = {"value": round(gbs, 6), "unit": "GB/s", "cores": cores,
                                "kind": "oracle",
                                "sample": f"{n} (sequence, kv head) units = {n / n_all:.2f} passes "
                                          f"over all {n_all} of the workload: select + "
                                          f"attention, {dt:.1f} s"}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
