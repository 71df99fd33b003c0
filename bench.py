"""Benchmark: paged sparse-KV attention on one B200 per rank.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload all|llama8b|llama70b|mla|prefill|llama8b_fp8]

A step is one pass of the whole hot path over one batch: page selection
(scoring against the per-page key summaries, forced sink and local pages,
top-k), the gather split-KV decode over the selected lists and the split merge.
The headline workload is the Llama-3-8B-shaped decode: B=16 sequences of 32768
tokens, Hq=32, Hkv=8, D=128, 16-token pages in a shuffled 2 GiB pool per layer,
budget 1024 tokens (2 sink + 32 local + 30 top-k pages per kv head), 5% of the
pages per kv head lifted 3 sigma along the group query; bf16 N(0,1) data.  A
step is the library's one-call entry (sa_sparse_step: four launches).

Timing.  Steps run back to back, each on its own layer's cache: four layers
with distinct caches, cycled, so a step's inputs (64 MiB of summaries + 64 MiB
of selected K/V) are not in L2 from the step before (the L2 holds 126 MB; a
cache comes back every fourth step).  Every step is one CUDA-graph replay;
CUDA events bracket exactly K steps on the launching stream, with a barrier and
a synchronize on both sides.  The decode kernel's roofline takes its average
launch duration from K back-to-back launches over the same rotating caches, and
counts the method's bytes only: the selected pages' valid K+V, q, the final O
and LSE, the lists and the page-table entries they resolve (not the split
partials, which are the kernel's choice).  Beside it: the same kernel launched
alone after an L2 flush, and the event-timed cost of a one-element launch.

The default run (--workload all, one GPU) adds the other four workloads in a
`workloads` object of the same line: the Llama-70B-shaped long decode (32
sequences of 64K-128K tokens; 256 MiB selected per step, one 12 GiB cache),
the FP8-page variant of the headline, the MLA + MTP tiered decode timed as a
CUDA graph of 61 back-to-back layer calls over 61 distinct latent caches (as a
61-layer model runs them), and the block-union chunked prefill.  Each has its
own value, step time, calls/s, roofline (HBM bytes or tensor FLOPs against the
measured peaks) and end-to-end figure.

End to end (`e2e`): the same steps through the public API with the step's
inputs (q, page table, sequence lengths) copied from pinned host memory and its
outputs (O, LSE) copied back inside the timed region, each side packed into one
buffer (one copy each way), the step itself one C call.

`cpu_baseline` (rank 0, one GPU): the float64 oracle, as it stands, on a
bounded sample of (sequence, kv head) units of the headline workload, timed on
the host cores (all of them, and one BLAS thread).  `--impl reference` times
the same oracle as this build's reference arm (there is no reference code to
run: the method comes from web pages) on the same workload and config.

With --gpus N (torchrun), every rank runs its own replica of the headline
workload (the path has no exchange step); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "selected-KV GB/s (fraction of HBM peak) and sparse-attn calls/sec at 1 B200"
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
GQA_LAYERS = 4          # distinct caches cycled by the Llama-8B-shaped steps
MLA_LAYERS = 61         # one latent cache per layer of a 61-layer model
L2_NOTE = ("inputs larger than L2: steps back to back, each on its own layer's cache "
           "({n} distinct caches cycled; one step touches {mb:.0f} MB, L2 is 126 MB)")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--splits", type=int, default=0, help="decode split count (0 = default)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--layers", type=int, default=0,
                    help="distinct layer caches the Llama-8B-shaped steps (0 = %d) and the MLA "
                         "graph (0 = %d) cycle; a small count keeps a profiler capture to a few "
                         "GB" % (GQA_LAYERS, MLA_LAYERS))
    ap.add_argument("--workload", default="all",
                    choices=["all", "llama8b", "llama70b", "mla", "prefill", "llama8b_fp8",
                             "dir_1m"],
                    help="all (default): the Llama-8B headline line with every other workload "
                         "in its `workloads` object; otherwise one workload's line alone")
    return ap.parse_args()


def gqa_layers(args):
    return args.layers if args.layers > 0 else GQA_LAYERS


def mla_layers(args):
    return args.layers if args.layers > 0 else MLA_LAYERS


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK}, "measured"
    return dict(FALLBACK), "fallback"


# ---------------------------------------------------------------------------
# clocks: nvidia-smi sampled in the background for the whole run
# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clock / throttle samples every 50 ms from before the first
    warm-up to after the last timed region; `windows` marks the GPU-busy spans
    (warm-up, graph capture, timed regions) whose samples the summary keeps."""

    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.samples = []          # (host time, line)
        self.windows = []
        self.proc = None

    def start(self, wait_s: float = 5.0):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True, bufsize=1)
        except Exception:
            self.proc = None
            return self
        threading.Thread(target=self._read, daemon=True).start()
        t0 = time.time()
        while not self.samples and time.time() - t0 < wait_s:   # first sample in
            time.sleep(0.01)
        return self

    def _read(self):
        for line in self.proc.stdout:
            if line.strip():
                self.samples.append((time.time(), line))

    def busy(self):
        """Context manager marking a GPU-busy span."""
        sampler = self

        class _W:
            def __enter__(self):
                self.t0 = time.time()

            def __exit__(self, *exc):
                sampler.windows.append((self.t0, time.time()))
        return _W()

    def stop(self):
        if self.proc is not None:
            time.sleep(0.06)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, mx, reasons, n_all = [], None, set(), 0
        for t, l in self.samples:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 7:
                continue
            n_all += 1
            if not any(a - 0.06 <= t <= b + 0.06 for a, b in self.windows):
                continue
            try:
                sm.append(float(f[0]))
                mx = float(f[1])
            except ValueError:
                continue
            for n, v in zip(names, f[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        out = {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm),
               "samples_whole_run": n_all,
               "window": "warm-up, graph capture and timed regions of every workload"}
        if sm:
            sm.sort()
            out["sm_mhz"] = sm[len(sm) // 2]
        return out


# ---------------------------------------------------------------------------
# shared helpers
# ---------------------------------------------------------------------------
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


class Flusher:
    """Evicts L2 before an isolated launch: writes a 256 MiB buffer, then reads
    another 256 MiB so the dirty lines are written back before the launch."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
        self.r = torch.ones(64 * 1024 * 1024, dtype=torch.int32, device=dev)
        self.sink = torch.empty((), dtype=torch.int64, device=dev)

    def __call__(self, i):
        import torch
        self.w.fill_(i & 0xFF)
        torch.sum(self.r, dim=0, dtype=torch.int64, out=self.sink)


def capture(fn):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def time_back_to_back(graphs, K, stream, world, dev):
    """Device seconds of K back-to-back graph replays cycling `graphs` (events at
    both ends, barrier + synchronize on both sides), max over ranks."""
    import torch
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(K):
        graphs[i % len(graphs)].replay()
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    return max_over_ranks(e0.elapsed_time(e1) / 1e3, world, dev)


def time_isolated(graph, n, flush, stream):
    """Mean device seconds of one replay of `graph` with L2 flushed before each."""
    import torch
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
    for i in range(n):
        flush(i)
        ev[i][0].record(stream)
        graph.replay()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in ev) / 1e3 / n


E2E_WHAT = ("every step: its inputs host->device from pinned memory (one packed copy), the "
            "step, its outputs device->host into pinned memory (one packed copy); copies on "
            "their own streams, so the upload of the next step and the download of the last "
            "overlap this step (a buffer is rewritten only after its last reader is done); "
            "device time from the first upload to the last download")


def time_e2e(items, K, stream, world, dev):
    """Device seconds of K end-to-end steps cycling `items` (each with h_in / d_in
    packed inputs, `call` launching the step on `stream`, d_out / h_out packed
    outputs), pipelined over an upload and a download stream; max over ranks."""
    import torch
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    n = len(items)
    ev_in = [torch.cuda.Event() for _ in range(n)]
    ev_done = [torch.cuda.Event() for _ in range(n)]
    ev_out = [torch.cuda.Event() for _ in range(n)]
    used = [False] * n
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    up.wait_event(e0)
    down.wait_event(e0)
    for k in range(K):
        i = k % n
        it = items[i]
        if used[i]:
            up.wait_event(ev_done[i])          # the last step reading d_in is done
            stream.wait_event(ev_out[i])       # d_out of its last use is downloaded
        with torch.cuda.stream(up):
            it["d_in"].copy_(it["h_in"], non_blocking=True)
        ev_in[i].record(up)
        stream.wait_event(ev_in[i])
        it["call"]()
        ev_done[i].record(stream)
        down.wait_event(ev_done[i])
        with torch.cuda.stream(down):
            it["h_out"].copy_(it["d_out"], non_blocking=True)
        ev_out[i].record(down)
        used[i] = True
    for i in range(n):
        if used[i]:
            stream.wait_event(ev_out[i])
    e1.record(stream)
    torch.cuda.synchronize()
    t = max_over_ranks(e0.elapsed_time(e1) / 1e3, world, dev)
    if world > 1:
        dist.barrier()
    return t


def launch_floor(flush, stream, dev, n=50):
    """Event-timed seconds of one flushed replay of a one-element kernel."""
    import torch
    x = torch.zeros(1, device=dev)
    g = capture(lambda: x.add_(1.0))
    for _ in range(3):
        g.replay()
    return time_isolated(g, n, flush, stream)


def selected_kv_bytes(counts, pages, seq_lens, P, D, elem_bytes=2):
    """K+V bytes of the valid tokens of every selected page; FP8 pages (elem_bytes
    1) add their two float32 scales per selected (page, kv head)."""
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


def gqa_config(cfg, n_splits, world, fp8=False, n_layers=GQA_LAYERS):
    """The `config` of a GQA decode line (both arms print the same one).  The
    bytes a step touches are the nominal ones of the workload (mean sequence
    length): the summaries it scores and the selected pages' K/V."""
    mean_pages = -(-((cfg.seq_len_lo + cfg.seq_len_hi) // 2) // cfg.page_size)
    budget_pages = cfg.budget_tokens // cfg.page_size
    elem = 1 if fp8 else 2
    step_mb = cfg.B * cfg.Hkv * (mean_pages * cfg.D * 2 +
                                 budget_pages * cfg.page_size * cfg.D * elem * 2) / 1e6
    c = {"workload": cfg.name + ("_fp8" if fp8 else ""), "B": cfg.B,
         "seq_len": (cfg.seq_len_lo if cfg.seq_len_lo == cfg.seq_len_hi
                     else f"U[{cfg.seq_len_lo},{cfg.seq_len_hi}]"),
         "Hq": cfg.Hq, "Hkv": cfg.Hkv, "D": cfg.D, "page_size": cfg.page_size,
         "kv_pages": "fp8 e4m3 + float32 scale per (page, kv head)" if fp8 else "bf16",
         "budget_tokens": cfg.budget_tokens, "sink_tokens": cfg.sink_tokens,
         "local_tokens": cfg.local_tokens, "n_splits": n_splits, "layer_caches": n_layers,
         "parallelism": f"replicas x{world}",
         "l2": L2_NOTE.format(n=n_layers, mb=step_mb)}
    return c


def gqa_splits(cfg, args):
    from paged_sparse_kv_sa_b200.pipeline import default_splits
    budget_pages = cfg.budget_tokens // cfg.page_size
    return args.splits or default_splits(cfg.B * cfg.Hkv, budget_pages)


# ---------------------------------------------------------------------------
# GQA decode workloads (Llama-8B, its FP8 pages, Llama-70B)
# ---------------------------------------------------------------------------
def run_gqa(cfg, args, dev, world, rank, clk, K, fp8=False, n_layers=GQA_LAYERS):
    import torch

    import paged_sparse_kv_sa_b200 as sa
    from paged_sparse_kv_sa_b200 import workloads as W

    sa.load()
    stream = torch.cuda.current_stream(dev)
    n_splits = gqa_splits(cfg, args)
    layers = []
    for l in range(n_layers):
        inp = W.gqa_decode_inputs(cfg, seed=args.seed + 1000 * rank + l, device=dev)
        if fp8:
            kc, ks = W.fp8_pages(inp.pop("k"))
            vc, vs = W.fp8_pages(inp.pop("v"))
            inp.update(kc=kc, ks=ks, vc=vc, vs=vs)
            sig = sa.sa_build_page_summaries_fp8(kc, ks, inp["page_table"], inp["seq_lens"])
        else:
            sig = sa.sa_build_page_summaries(inp["k"], inp["page_table"], inp["seq_lens"])
        step = sa.SparseDecodeStep(cfg.B, cfg.T, cfg.Hq, cfg.Hkv, cfg.D, cfg.page_size,
                                   inp["page_table"].shape[1], cfg.sink_tokens, cfg.local_tokens,
                                   cfg.budget_tokens, n_splits=n_splits, device=dev)
        torch.cuda.synchronize()
        layers.append(dict(inp=inp, sig=sig, step=step))

    def step_fn(L):
        i, s = L["inp"], L["step"]
        if fp8:
            s.run_fp8(i["q"], i["kc"], i["vc"], i["ks"], i["vs"], L["sig"], i["page_table"],
                      i["seq_lens"])
        else:
            s.run(i["q"], i["k"], i["v"], L["sig"], i["page_table"], i["seq_lens"])

    def decode_fn(L):
        i, s = L["inp"], L["step"]
        if fp8:
            s.decode_fp8(i["q"], i["kc"], i["vc"], i["ks"], i["vs"], i["page_table"],
                         i["seq_lens"])
        else:
            s.decode(i["q"], i["k"], i["v"], i["page_table"], i["seq_lens"])

    with clk.busy():
        for L in layers:
            L["step"].dev_error.zero_()
            for _ in range(max(args.warmup, 3)):
                step_fn(L)
        torch.cuda.synchronize()
        # algorithmic bytes of each layer's step (from the selection it made)
        for L in layers:
            s, i = L["step"], L["inp"]
            L["kv"] = selected_kv_bytes(s.counts, s.pages, i["seq_lens"], cfg.page_size, cfg.D,
                                        elem_bytes=1 if fp8 else 2)
            L["alg"] = (L["kv"] + i["q"].numel() * 2 + s.o.numel() * 4 + s.lse.numel() * 4 +
                        s.pages.numel() * 4 + s.counts.numel() * 4 +
                        int(s.counts.sum().item()) * 4)
            L["g_step"] = capture(lambda L=L: step_fn(L))
            L["g_dec"] = capture(lambda L=L: decode_fn(L))
        for L in layers:
            for _ in range(3):
                L["g_step"].replay()
                L["g_dec"].replay()
        torch.cuda.synchronize()
        t_step = time_back_to_back([L["g_step"] for L in layers], K, stream, world, dev)
        t_dec = time_back_to_back([L["g_dec"] for L in layers], K, stream, world, dev)
    kv_total = sum(layers[i % n_layers]["kv"] for i in range(K))
    alg_total = sum(layers[i % n_layers]["alg"] for i in range(K))
    for L in layers:
        assert int(L["step"].dev_error.item()) == 0, "device error flag set"
        assert torch.isfinite(L["step"].o).all().item(), "non-finite output"

    # the decode kernel alone after an L2 flush, and the cost of a launch itself
    flush = Flusher(dev)
    with clk.busy():
        n_iso = min(K, 50)
        t_iso = time_isolated(layers[0]["g_dec"], n_iso, flush, stream)
        t_floor = launch_floor(flush, stream, dev)
    del flush

    # end to end through the public API: the step's inputs from pinned host memory
    # (packed: one copy), the step's C calls (marshalled once: sa.bind), its
    # outputs back (packed: one copy); at least two buffer sets alternate
    items = []
    for idx in range(max(2, n_layers)):
        L = layers[idx % n_layers]
        i = L["inp"]
        s = L["step"] if idx < n_layers else sa.SparseDecodeStep(
            cfg.B, cfg.T, cfg.Hq, cfg.Hkv, cfg.D, cfg.page_size, i["page_table"].shape[1],
            cfg.sink_tokens, cfg.local_tokens, cfg.budget_tokens, n_splits=n_splits, device=dev)
        srcs = (i["q"], i["page_table"], i["seq_lens"])
        h_in, hv = _packed(srcs, "cpu")
        for h_, x in zip(hv, srcs):
            h_.copy_(x.cpu())
        d_in, (q_d, pt_d, sl_d) = _packed(srcs, dev)
        d_out, (s.o, s.lse) = _packed((s.o, s.lse), dev)   # the step writes these views
        h_out, _ = _packed((s.o, s.lse), "cpu")
        if fp8:
            call = sa.bind(lambda s=s, L=L, q_d=q_d, pt_d=pt_d, sl_d=sl_d: s.run_fp8(
                q_d, L["inp"]["kc"], L["inp"]["vc"], L["inp"]["ks"], L["inp"]["vs"], L["sig"],
                pt_d, sl_d))
        else:
            call = s.bind(q_d, i["k"], i["v"], L["sig"], pt_d, sl_d)
        items.append(dict(h_in=h_in, d_in=d_in, d_out=d_out, h_out=h_out, call=call))

    with clk.busy():
        time_e2e(items, max(args.warmup, 3) * len(items), stream, 1, dev)
        t_e2e = time_e2e(items, K, stream, world, dev)
    h2d = items[0]["h_in"].numel()
    d2h = items[0]["h_out"].numel()
    del items

    pk, peak_kind = peaks()
    hbm = pk["hbm_gbs"]
    dec_us = t_dec / K * 1e6
    achieved = alg_total / t_dec / 1e9
    traffic = None
    tp = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if os.path.exists(tp) and not fp8:
        with open(tp) as f:
            td = json.load(f)
        src = os.path.join(ROOT, "paged_sparse_kv_sa_b200", "csrc", "decode.cu")
        import hashlib
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if (td.get("workload") == cfg.name and td.get("splits") == n_splits
                and td.get("decode_cu_sha16") == sha):
            traffic = td.get("bytes_per_launch")
    kern = "decode_gqa_kernel" + ("<fp8>" if fp8 else "")
    return {
        "metric": METRIC, "value": round(world * kv_total / t_step / 1e9, 3), "unit": "GB/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": round(1e3 * t_step / K, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": gqa_config(cfg, n_splits, world, fp8, n_layers),
        "calls_per_sec": round(world * K / t_step, 2),
        "selected_kv_bytes_per_step": kv_total // K,
        "roofline": {"kernel": kern, "bound": "hbm", "achieved": round(achieved, 2),
                     "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                     "peak_kind": f"{peak_kind} (copy bandwidth)", "traffic": traffic,
                     "alg_bytes_per_launch": alg_total // K,
                     "alg_bytes_what": "selected valid K+V + q + final O and LSE (float32) + "
                                       "list entries + page-table entries",
                     "kernel_us": round(dec_us, 2),
                     "kernel_us_what": f"average launch duration over {K} back-to-back "
                                       f"launches cycling {n_layers} layer caches",
                     "isolated_us": round(1e6 * t_iso, 2),
                     "isolated_frac": round(alg_total / K / t_iso / 1e9 / hbm, 4),
                     "isolated_what": "one launch after an L2 flush, event-timed",
                     "launch_floor_us": round(1e6 * t_floor, 2),
                     "launch_floor_what": "one flushed, event-timed launch of a one-element "
                                          "kernel"},
        "e2e": {"value": round(world * kv_total / t_e2e / 1e9, 3), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(1e3 * t_e2e / K, 4),
                "what": E2E_WHAT + ("; the step: one C call (sa_sparse_step_fp8)" if fp8
                                    else "; the step: one C call (sa_sparse_step)")},
        "gpu_launches": 4 * K,
        "_layers": layers,
    }


# ---------------------------------------------------------------------------
# million-token page tables: the step over a two-level page map, and the same
# step over the flat table it stands for
# ---------------------------------------------------------------------------
def run_dir(args, dev, world, rank, clk, K):
    import torch

    import paged_sparse_kv_sa_b200 as sa
    from paged_sparse_kv_sa_b200 import workloads as W

    sa.load()
    cfg, shift = W.LLAMA8B_DIR_1M, W.DIR_BLOCK_SHIFT
    stream = torch.cuda.current_stream(dev)
    n_splits = gqa_splits(cfg, args)
    inp = W.gqa_decode_inputs(cfg, seed=args.seed + 1000 * rank, device=dev)
    page_dir, blocks = W.page_directory(inp["page_table"], inp["seq_lens"], cfg.page_size, shift,
                                        seed=args.seed + 1000 * rank)
    pt = inp["page_table"]
    q, k, v, sl = inp["q"], inp["k"], inp["v"], inp["seq_lens"]
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    sig = sa.sa_build_page_summaries_dir(k, page_dir, blocks, shift, sl, dev_error=err)
    scale = 1.0 / math.sqrt(cfg.D)
    bp = cfg.budget_tokens // cfg.page_size
    outs = {}
    for name in ("dir", "flat"):
        cap = sa.dir_capacity(page_dir, shift) if name == "dir" else pt.shape[1]
        n_ws = sa.sa_sparse_step_workspace_size(cfg.B, cfg.T, cfg.Hq, cfg.Hkv, cfg.D,
                                                cfg.page_size, cap, cfg.budget_tokens, n_splits)
        outs[name] = dict(
            pages=torch.empty((cfg.B, cfg.Hkv, bp), dtype=torch.int32, device=dev),
            counts=torch.empty((cfg.B, cfg.Hkv), dtype=torch.int32, device=dev),
            o=torch.empty((cfg.B, cfg.T, cfg.Hq, cfg.D), dtype=torch.float32, device=dev),
            lse=torch.empty((cfg.B, cfg.T, cfg.Hq), dtype=torch.float32, device=dev),
            ws=torch.empty(n_ws, dtype=torch.uint8, device=dev))

    def step(name):
        r = outs[name]
        common = dict(n_splits=n_splits, out_pages=r["pages"], out_counts=r["counts"],
                      o_out=r["o"], lse_out=r["lse"], workspace=r["ws"], dev_error=err)
        if name == "dir":
            sa.sa_sparse_step_dir(q, sig, k, v, page_dir, blocks, shift, sl, cfg.page_size,
                                  cfg.sink_tokens, cfg.local_tokens, cfg.budget_tokens, scale,
                                  **common)
        else:
            sa.sa_sparse_step(q, sig, k, v, pt, sl, cfg.page_size, cfg.sink_tokens,
                              cfg.local_tokens, cfg.budget_tokens, scale, **common)

    flush = Flusher(dev)
    with clk.busy():
        for _ in range(max(args.warmup, 3)):
            step("dir")
            step("flat")
        torch.cuda.synchronize()
        graphs = {n: capture(lambda n=n: step(n)) for n in ("dir", "flat")}
        for g in graphs.values():
            for _ in range(3):
                g.replay()
        t = {n: time_isolated(graphs[n], K, flush, stream) for n in ("dir", "flat")}
    del flush
    torch.cuda.synchronize()
    assert int(err.item()) == 0, "device error flag set"
    same = all(torch.equal(outs["dir"][x], outs["flat"][x]) for x in ("pages", "counts", "o",
                                                                       "lse"))
    r = outs["dir"]
    kv = selected_kv_bytes(r["counts"], r["pages"], sl, cfg.page_size, cfg.D)
    n_pages = ((sl.to(torch.int64) + cfg.page_size - 1) // cfg.page_size)
    tot_pages = int(n_pages.sum().item())
    sig_bytes = tot_pages * cfg.Hkv * cfg.D * 2
    map_bytes_dir = page_dir.numel() * 4 + blocks.numel() * 4
    map_bytes_flat = pt.numel() * 4
    alg = (sig_bytes + kv + q.numel() * 2 + r["o"].numel() * 4 + r["lse"].numel() * 4 +
           map_bytes_dir + r["pages"].numel() * 4 + r["counts"].numel() * 4)
    t_dir = max_over_ranks(t["dir"], world, dev)
    t_flat = max_over_ranks(t["flat"], world, dev)
    pk, peak_kind = peaks()
    hbm = pk["hbm_gbs"]
    achieved = alg / t_dir / 1e9
    return {
        "metric": "sparse-attn calls/sec over million-token page tables (two-level page map)",
        "value": round(world / t_dir, 2), "unit": "calls/s", "steps": K,
        "ms_per_step": round(1e3 * t_dir, 4),
        "config": {"workload": cfg.name, "B": cfg.B,
                   "seq_len": f"U[{cfg.seq_len_lo},{cfg.seq_len_hi}]",
                   "seq_lens": [int(x) for x in sl.tolist()], "Hq": cfg.Hq, "Hkv": cfg.Hkv,
                   "D": cfg.D, "page_size": cfg.page_size, "budget_tokens": cfg.budget_tokens,
                   "sink_tokens": cfg.sink_tokens, "local_tokens": cfg.local_tokens,
                   "n_splits": n_splits, "block_pages": 1 << shift,
                   "page_map_bytes": {"two_level": map_bytes_dir, "flat": map_bytes_flat},
                   "l2": "L2 flushed before every timed step (each step alone, event-timed)",
                   "parallelism": f"replicas x{world}"},
        "flat_table_ms_per_step": round(1e3 * t_flat, 4),
        "two_level_vs_flat": round(t_dir / t_flat, 4),
        "same_bits_as_flat": bool(same),
        "summary_bytes_scored_per_step": sig_bytes,
        "selected_kv_bytes_per_step": kv,
        "roofline": {"kernel": "whole step (score, choose, decode, combine)", "bound": "hbm",
                     "achieved": round(achieved, 2), "peak": hbm, "unit": "GB/s",
                     "frac": round(achieved / hbm, 4),
                     "peak_kind": f"{peak_kind} (copy bandwidth)", "traffic": None,
                     "alg_bytes_per_launch": alg,
                     "alg_bytes_what": "summaries of every page of every sequence + selected "
                                       "valid K+V + q + final O and LSE (float32) + directory "
                                       "and blocks + selection outputs",
                     "step_us": round(1e6 * t_dir, 2)},
        "gpu_launches": 4 * K * 2,
    }


# ---------------------------------------------------------------------------
# MLA + MTP tiered decode: a graph of 61 layer calls over distinct caches
# ---------------------------------------------------------------------------
def run_mla(args, dev, world, rank, clk, reps):
    import numpy as np
    import torch

    import paged_sparse_kv_sa_b200 as sa
    from paged_sparse_kv_sa_b200 import workloads as W

    lib = sa.load()
    cfg = W.MLA_MTP
    stream = torch.cuda.current_stream(dev)
    n_splits = args.splits or 8
    n_ml = mla_layers(args)
    cap = cfg.alpha + cfg.beta
    scale = 1.0 / math.sqrt(cfg.Dk)
    o = torch.empty((cfg.B, cfg.T, cfg.Hq, cfg.Dv), dtype=torch.float32, device=dev)
    lse = torch.empty((cfg.B, cfg.T, cfg.Hq), dtype=torch.float32, device=dev)
    o_p = torch.empty((n_splits, cfg.B, cfg.T, cfg.Hq, cfg.Dv), dtype=torch.float32, device=dev)
    l_p = torch.empty((n_splits, cfg.B, cfg.T, cfg.Hq), dtype=torch.float32, device=dev)
    aws = sa.attention_workspace(cfg.B, cfg.T, cfg.Hq, cfg.Dv, n_splits, dev)
    layers = []
    for l in range(n_ml):
        inp = W.mla_decode_inputs(cfg, seed=args.seed + 1000 * rank + l, device=dev)
        sig = sa.sa_build_page_summaries(inp["kv"], inp["page_table"], inp["seq_lens"])
        amb = set(int(h) for h in inp["ambient_heads"].tolist())
        ws = torch.empty(max(int(lib.sa_select_tiered_workspace_size(
            cfg.B, cfg.T, cfg.Hq, inp["page_table"].shape[1])), 16), dtype=torch.uint8, device=dev)
        layers.append(dict(inp=inp, sig=sig, ws=ws, h2l=[1 if h in amb else 0 for h in range(cfg.Hq)],
                           lists=torch.empty((cfg.B, 2, cap), dtype=torch.int32, device=dev),
                           counts=torch.empty((cfg.B, 2), dtype=torch.int32, device=dev)))
    torch.cuda.synchronize()

    def select(L, q, pt, sl):
        sa.sa_select_pages_tiered(q, L["sig"], pt, sl, cfg.page_size, cfg.alpha, cfg.beta,
                                  lists=L["lists"], list_counts=L["counts"], workspace=L["ws"])

    def attend(L, q, pt, sl, oo, ll):
        kv = L["inp"]["kv"]
        sa.sa_sparse_attention(q, kv, kv[..., :cfg.Dv], pt, sl, L["lists"], L["counts"], L["h2l"],
                               scale, n_splits, o_out=oo, lse_out=ll, workspace=aws)

    def step(L):
        i = L["inp"]
        select(L, i["q"], i["page_table"], i["seq_lens"])
        attend(L, i["q"], i["page_table"], i["seq_lens"], o, lse)

    def decode(L):
        i = L["inp"]
        kv = i["kv"]
        sa.sa_sparse_decode(i["q"], kv, kv[..., :cfg.Dv], i["page_table"], i["seq_lens"],
                            L["lists"], L["counts"], L["h2l"], scale, n_splits, o_partial=o_p,
                            lse_partial=l_p)

    with clk.busy():
        for _ in range(max(args.warmup, 3)):
            for L in layers:
                step(L)
        torch.cuda.synchronize()
        flops, kv_bytes = 0, 0
        for L in layers:
            Ls = L["inp"]["seq_lens"].cpu().numpy()
            ls, cs = L["lists"].cpu().numpy(), L["counts"].cpu().numpy()
            amb_n = sum(L["h2l"])
            for b in range(cfg.B):
                for t in range(cfg.T):
                    qpos = int(Ls[b]) - cfg.T + t
                    for li, nh in ((0, cfg.Hq - amb_n), (1, amb_n)):
                        pg = ls[b, li, :cs[b, li]].astype(np.int64)
                        keys = np.clip(np.minimum(qpos + 1, int(Ls[b])) - pg * cfg.page_size, 0,
                                       cfg.page_size).sum()
                        flops += 2 * nh * int(keys) * (cfg.Dk + cfg.Dv)
                pg = ls[b, 1, :cs[b, 1]].astype(np.int64)
                kv_bytes += int(np.clip(int(Ls[b]) - pg * cfg.page_size, 0,
                                        cfg.page_size).sum()) * cfg.Dk * 2
        g_step = capture(lambda: [step(L) for L in layers])
        g_dec = capture(lambda: [decode(L) for L in layers])
        for _ in range(2):
            g_step.replay()
            g_dec.replay()
        torch.cuda.synchronize()
        t_step = time_back_to_back([g_step], reps, stream, world, dev)
        t_dec = time_back_to_back([g_dec], reps, stream, world, dev)
    n = reps * n_ml
    assert torch.isfinite(o).all().item(), "non-finite output"

    # end to end through the public API over the first eight layers' caches (cycled):
    # a step's inputs from the host, select + attend, its outputs back
    items = []
    for L in layers[:8]:
        i0 = L["inp"]
        srcs = (i0["q"], i0["page_table"], i0["seq_lens"])
        h_in, hv = _packed(srcs, "cpu")
        for h_, x in zip(hv, srcs):
            h_.copy_(x.cpu())
        d_in, (q_d, pt_d, sl_d) = _packed(srcs, dev)
        d_out, (o_d, lse_d) = _packed((o, lse), dev)
        h_out, _ = _packed((o, lse), "cpu")

        call = sa.bind(lambda L=L, q_d=q_d, pt_d=pt_d, sl_d=sl_d, o_d=o_d, lse_d=lse_d: (
            select(L, q_d, pt_d, sl_d), attend(L, q_d, pt_d, sl_d, o_d, lse_d)))
        items.append(dict(h_in=h_in, d_in=d_in, d_out=d_out, h_out=h_out, call=call))
    K = max(args.steps, 20)
    with clk.busy():
        time_e2e(items, 3 * len(items), stream, 1, dev)
        t_e2e = time_e2e(items, K, stream, world, dev)
    h_in, h_out = items[0]["h_in"], items[0]["h_out"]
    pk, kind = peaks()
    per_call_flops = flops / n_ml
    per_call_bytes = kv_bytes / n_ml
    achieved = per_call_flops / (t_dec / n) / 1e12
    return {
        "value": round(world * kv_bytes * reps / t_step / 1e9, 3), "unit": "GB/s",
        "steps": n, "ms_per_step": round(1e3 * t_step / n, 4),
        "calls_per_sec": round(world * n / t_step, 2),
        "config": {"workload": cfg.name, "n_splits": n_splits, "layer_caches": n_ml,
                   "timing": f"CUDA graph of {n_ml} back-to-back layer calls over "
                             f"{n_ml} distinct latent caches, replayed {reps} times",
                   "l2": f"inputs larger than L2 ({n_ml} x 604 MB of caches cycled)"},
        "selected_kv_bytes_per_step": int(per_call_bytes), "flops_per_step": int(per_call_flops),
        "step_tflops": round(world * flops * reps / t_step / 1e12, 2),
        "roofline": {"kernel": "mla_kernel", "bound": "tensor", "achieved": round(achieved, 2),
                     "peak": pk["bf16_tflops_sustained"], "unit": "TFLOP/s",
                     "frac": round(achieved / pk["bf16_tflops_sustained"], 4),
                     "peak_kind": f"{kind} bf16 GEMM, sustained (a long loop of launches)",
                     "traffic": None,
                     "kernel_us": round(1e6 * t_dec / n, 2),
                     "kernel_us_what": f"average launch in a graph of {n_ml} "
                                       "back-to-back decode launches",
                     "hbm_achieved_gbs": round(per_call_bytes / (t_dec / n) / 1e9, 1),
                     "hbm_frac": round(per_call_bytes / (t_dec / n) / 1e9 / pk["hbm_gbs"], 4)},
        "e2e": {"value": round(world * (kv_bytes / n_ml) * K / t_e2e / 1e9, 3),
                "unit": "GB/s", "h2d_bytes_per_step": h_in.numel(),
                "d2h_bytes_per_step": h_out.numel(), "ms_per_step": round(1e3 * t_e2e / K, 4),
                "what": E2E_WHAT + "; the step: select and attend (two C calls), eight layer "
                                   "caches cycled"},
        "gpu_launches": 4 * n,
    }


# ---------------------------------------------------------------------------
# block-union chunked prefill
# ---------------------------------------------------------------------------
def run_prefill(args, dev, world, rank, clk, K):
    import numpy as np
    import torch

    import paged_sparse_kv_sa_b200 as sa
    from paged_sparse_kv_sa_b200 import workloads as W

    sa.load()
    cfg = W.UNION_PREFILL
    stream = torch.cuda.current_stream(dev)
    inp = W.prefill_inputs(cfg, seed=args.seed + rank, device=dev)
    q, kk, vv, pt, sl = inp["q"], inp["k"], inp["v"], inp["page_table"], inp["seq_lens"]
    scores = W.block_union_scores(cfg, seed=args.seed + rank, device=dev)
    off = cfg.q_offset // cfg.block
    tables = torch.empty((cfg.Hkv, cfg.n_kv_blocks), dtype=torch.int32, device=dev)
    tcounts = torch.empty((cfg.Hkv,), dtype=torch.int32, device=dev)
    h2l = [h // (cfg.Hq // cfg.Hkv) for h in range(cfg.Hq)]
    n_splits = args.splits or 4
    o = torch.empty((1, cfg.chunk, cfg.Hq, cfg.D), dtype=torch.float32, device=dev)
    lse = torch.empty((1, cfg.chunk, cfg.Hq), dtype=torch.float32, device=dev)
    o_p = torch.empty((n_splits, 1, cfg.chunk, cfg.Hq, cfg.D), dtype=torch.float32, device=dev)
    l_p = torch.empty((n_splits, 1, cfg.chunk, cfg.Hq), dtype=torch.float32, device=dev)
    aws = sa.attention_workspace(1, cfg.chunk, cfg.Hq, cfg.D, n_splits, dev)
    scale = 1.0 / math.sqrt(cfg.D)

    def step(sc, qq, ptt, sll, oo, ll):
        sa.sa_block_union(sc, cfg.Hkv, off, cfg.top_k, cfg.n_sink_blocks, tables=tables,
                          counts=tcounts)
        sa.sa_sparse_attention(qq, kk, vv, ptt, sll, tables.view(1, cfg.Hkv, -1),
                               tcounts.view(1, cfg.Hkv), h2l, scale, n_splits, o_out=oo,
                               lse_out=ll, workspace=aws)

    def decode():
        sa.sa_sparse_decode(q, kk, vv, pt, sl, tables.view(1, cfg.Hkv, -1),
                            tcounts.view(1, cfg.Hkv), h2l, scale, n_splits, o_partial=o_p,
                            lse_partial=l_p)

    with clk.busy():
        for _ in range(max(args.warmup, 3)):
            step(scores, q, pt, sl, o, lse)
        torch.cuda.synchronize()
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
        g_step = capture(lambda: step(scores, q, pt, sl, o, lse))
        g_dec = capture(decode)
        for _ in range(2):
            g_step.replay()
            g_dec.replay()
        torch.cuda.synchronize()
        t_step = time_back_to_back([g_step], K, stream, world, dev)
        t_dec = time_back_to_back([g_dec], K, stream, world, dev)
    assert torch.isfinite(o).all().item(), "non-finite output"

    # end to end: two input / output buffer sets alternate (double buffering)
    srcs = (scores, pt, sl, q)
    items = []
    for _ in range(2):
        h_in, hv = _packed(srcs, "cpu")
        for h_, x in zip(hv, srcs):
            h_.copy_(x.cpu())
        d_in, (sc_d, pt_d, sl_d, q_d) = _packed(srcs, dev)
        d_out, (o_d, lse_d) = _packed((o, lse), dev)
        h_out, _ = _packed((o, lse), "cpu")
        items.append(dict(h_in=h_in, d_in=d_in, d_out=d_out, h_out=h_out,
                          call=sa.bind(lambda a=(sc_d, q_d, pt_d, sl_d, o_d, lse_d): step(*a))))
    with clk.busy():
        time_e2e(items, 2, stream, 1, dev)
        t_e2e = time_e2e(items, K, stream, world, dev)
    h_in, h_out = items[0]["h_in"], items[0]["h_out"]
    pk, kind = peaks()
    achieved = flops / (t_dec / K) / 1e12
    traffic = None
    tp = os.path.join(ROOT, "profiles", "prefill_traffic.json")
    if os.path.exists(tp):
        with open(tp) as f:
            td = json.load(f)
        src = os.path.join(ROOT, "paged_sparse_kv_sa_b200", "csrc", "prefill.cu")
        import hashlib
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if (td.get("workload") == cfg.name and td.get("splits") == n_splits
                and td.get("prefill_cu_sha16") == sha):
            traffic = td.get("bytes_per_launch")
    return {
        "value": round(world * kv_bytes * K / t_step / 1e9, 3), "unit": "GB/s", "steps": K,
        "ms_per_step": round(1e3 * t_step / K, 4), "calls_per_sec": round(world * K / t_step, 2),
        "config": {"workload": cfg.name, "n_splits": n_splits,
                   "l2": "inputs larger than L2 (529 MB K/V pool, 217 MB selected per step), "
                         "steps back to back"},
        "selected_kv_bytes_per_step": kv_bytes, "flops_per_step": flops,
        "step_tflops": round(world * flops * K / t_step / 1e12, 2),
        "roofline": {"kernel": "prefill_kernel", "bound": "tensor", "achieved": round(achieved, 2),
                     "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(achieved / pk["bf16_tflops"], 4),
                     "peak_kind": f"{kind} bf16 GEMM, burst", "traffic": traffic,
                     "traffic_what": "DRAM bytes read + written per launch (ncu, one launch of "
                                     "this kernel at this workload and split count), or null",
                     "kernel_ms": round(1e3 * t_dec / K, 4),
                     "kernel_ms_what": f"average over {K} back-to-back launches"},
        "e2e": {"value": round(world * kv_bytes * K / t_e2e / 1e9, 3), "unit": "GB/s",
                "h2d_bytes_per_step": h_in.numel(), "d2h_bytes_per_step": h_out.numel(),
                "ms_per_step": round(1e3 * t_e2e / K, 4),
                "what": E2E_WHAT + "; inputs: block scores, page table, lengths and queries; "
                                   "the step: union + attend (two C calls)"},
        "gpu_launches": 5 * K,
    }


# ---------------------------------------------------------------------------
# the float64 oracle on the host cores (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------
def oracle_units(cfg, inp, units, fp8):
    """Each sampled (b, kv head) unit as a local problem the oracle can run alone
    (its query rows, its pages, an identity page table), with its summaries
    computed by the oracle (not part of a step) and its selected KV bytes."""
    import numpy as np
    import torch

    import oracle as O
    from paged_sparse_kv_sa_b200 import workloads as W

    G = cfg.Hq // cfg.Hkv
    out = []
    for b, kvh in units:
        L = int(inp["seq_lens"][b].item())
        N = -(-L // cfg.page_size)
        phys = inp["page_table"][b, :N].to(torch.int64)
        pt = np.arange(N, dtype=np.int32).reshape(1, N)
        sl = np.array([L], dtype=np.int32)
        u = dict(q=W.bf16_bits(inp["q"][b:b + 1, :, kvh * G:(kvh + 1) * G]), pt=pt, sl=sl, G=G)
        if fp8:
            u["kc"] = inp["kc"][phys, kvh].unsqueeze(1).cpu().numpy()
            u["vc"] = inp["vc"][phys, kvh].unsqueeze(1).cpu().numpy()
            u["ks"] = inp["ks"][phys, kvh].unsqueeze(1).cpu().numpy()
            u["vs"] = inp["vs"][phys, kvh].unsqueeze(1).cpu().numpy()
            u["sig"] = O.page_summaries_fp8(u["kc"], u["ks"], pt, sl, cfg.page_size)
        else:
            u["k"] = W.bf16_bits(inp["k"][phys, kvh].unsqueeze(1))
            u["v"] = W.bf16_bits(inp["v"][phys, kvh].unsqueeze(1))
            u["sig"] = O.page_summaries(u["k"], pt, sl, cfg.page_size)
        out.append(u)
    return out


def oracle_step(cfg, u, fp8):
    """One unit of the step on the oracle: selection, then attention over it.
    Returns the selected valid K+V bytes."""
    import numpy as np

    import oracle as O

    pages, counts = O.select_pages(u["q"], u["sig"], u["pt"], u["sl"], cfg.page_size,
                                   cfg.sink_tokens, cfg.local_tokens, cfg.budget_tokens)
    h2l = np.zeros(u["G"], np.int64)
    scale = 1.0 / math.sqrt(cfg.D)
    if fp8:
        O.sparse_attention_fp8(u["q"], u["kc"], u["ks"], u["vc"], u["vs"], u["pt"], u["sl"],
                               pages, counts, h2l, scale, cfg.page_size)
    else:
        O.sparse_attention(u["q"], u["k"], u["v"], u["pt"], u["sl"], pages, counts, h2l, scale,
                           cfg.page_size)
    L = int(u["sl"][0])
    lst = pages[0, 0, :counts[0, 0]]
    toks = sum(min(cfg.page_size, L - int(p) * cfg.page_size) for p in lst)
    return toks * cfg.D * 2 * (1 if fp8 else 2) + (len(lst) * 8 if fp8 else 0)


def time_oracle(cfg, prepared, fp8, min_s, max_s=60.0, n_steps=None):
    """GB/s of the oracle over the prepared units (cycled): either until min_s
    seconds have passed and every unit ran once, or exactly n_steps units."""
    t0 = time.perf_counter()
    done, nbytes = 0, 0
    while True:
        nbytes += oracle_step(cfg, prepared[done % len(prepared)], fp8)
        done += 1
        el = time.perf_counter() - t0
        if n_steps is not None:
            if done >= n_steps:
                break
        elif (el >= min_s and done >= len(prepared)) or el > max_s:
            break
    dt = time.perf_counter() - t0
    return nbytes / dt / 1e9, done, dt


def blas_threads(n):
    from threadpoolctl import threadpool_limits
    return threadpool_limits(limits=n)


def oracle_sample_units(cfg, n, seed=7):
    import numpy as np
    rng = np.random.default_rng(seed)
    units = set()
    while len(units) < min(n, cfg.B * cfg.Hkv):
        units.add((int(rng.integers(cfg.B)), int(rng.integers(cfg.Hkv))))
    return sorted(units)


def cpu_baseline(cfg, inp, fp8, cores):
    prepared = oracle_units(cfg, inp, oracle_sample_units(cfg, 16), fp8)
    gbs, n, dt = time_oracle(cfg, prepared, fp8, min_s=10.0)
    with blas_threads(1):
        gbs1, n1, dt1 = time_oracle(cfg, prepared, fp8, min_s=4.0)
    return {"value": round(gbs, 6), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} (sequence, kv head) units of select + attention (a fixed sample of "
                      f"16 units of layer 0, cycled) in {dt:.1f} s; summaries computed beforehand",
            "value_1_thread": round(gbs1, 6),
            "sample_1_thread": f"{n1} units in {dt1:.1f} s, BLAS limited to one thread"}


def run_reference(args, dev, cores):
    """The oracle arm: the float64 oracle times K steps (one (sequence, kv head)
    unit of select + attention each) of the headline workload on the host cores."""
    import torch

    from paged_sparse_kv_sa_b200 import workloads as W

    fp8 = args.workload == "llama8b_fp8"
    cfg = {"llama70b": W.LLAMA70B_LONG}.get(args.workload, W.LLAMA8B_DECODE)
    inp = W.gqa_decode_inputs(cfg, seed=args.seed, device=dev)   # layer 0 of rank 0
    if fp8:
        kc, ks = W.fp8_pages(inp.pop("k"))
        vc, vs = W.fp8_pages(inp.pop("v"))
        inp.update(kc=kc, ks=ks, vc=vc, vs=vs)
    prepared = oracle_units(cfg, inp, oracle_sample_units(cfg, 16), fp8)
    del inp
    torch.cuda.empty_cache()
    for i in range(args.warmup):
        oracle_step(cfg, prepared[i % len(prepared)], fp8)
    gbs, n, dt = time_oracle(cfg, prepared, fp8, 0.0, n_steps=args.steps)
    with blas_threads(1):
        gbs1, n1, dt1 = time_oracle(cfg, prepared, fp8, 0.0, n_steps=min(args.steps, 16))
    n_layers = gqa_layers(args) if cfg is W.LLAMA8B_DECODE else 1
    line = {"metric": METRIC, "value": round(gbs, 6), "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1000 * dt / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": gqa_config(cfg, gqa_splits(cfg, args), args.gpus, fp8, n_layers),
            "cpu_baseline": {"value": round(gbs, 6), "unit": "GB/s", "cores": cores,
                             "kind": "oracle",
                             "sample": f"{n} steps, each one (sequence, kv head) unit of select "
                                       f"+ attention from a fixed sample of 16 units, {dt:.1f} s",
                             "value_1_thread": round(gbs1, 6),
                             "sample_1_thread": f"{n1} units in {dt1:.1f} s, one BLAS thread"},
            "e2e": {"value": round(gbs, 6), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def main():
    args = parse()
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    cores = len(os.sched_getaffinity(0))
    if args.impl == "reference":
        if rank != 0:
            return                  # the oracle arm runs on rank 0 only
        dev = torch.device("cuda", local)
        torch.cuda.set_device(dev)
        if args.workload in ("mla", "prefill", "dir_1m"):
            print(json.dumps({"impl": "reference", "unavailable":
                              "the oracle arm is timed on the GQA decode workloads"}))
            return
        return run_reference(args, dev, cores)
    if world > 1:
        torch.cuda.set_device(local)
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    from paged_sparse_kv_sa_b200 import workloads as W

    clk = ClockSampler(local).start()
    K = args.steps
    wl = args.workload
    try:
        if wl in ("mla", "prefill", "dir_1m"):
            sub = (run_mla(args, dev, world, rank, clk, reps=max(1, -(-K // mla_layers(args))))
                   if wl == "mla" else run_prefill(args, dev, world, rank, clk, K)
                   if wl == "prefill" else run_dir(args, dev, world, rank, clk, K))
            line = {"metric": METRIC, "n_gpus": world, "warmup": args.warmup,
                    "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                    "dtype": "bf16", "data": "synthetic", **sub}
        else:
            cfg = {"llama70b": W.LLAMA70B_LONG}.get(wl, W.LLAMA8B_DECODE)
            fp8 = wl == "llama8b_fp8"
            line = run_gqa(cfg, args, dev, world, rank, clk, K, fp8=fp8,
                           n_layers=gqa_layers(args) if cfg is W.LLAMA8B_DECODE else 1)
            layers = line.pop("_layers")
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline(cfg, layers[0]["inp"], fp8, cores)
            del layers
            torch.cuda.empty_cache()
            if wl == "all" and world == 1:
                subs = {}
                k_long = min(K, 100)
                r = run_gqa(W.LLAMA70B_LONG, args, dev, world, rank, clk, k_long, n_layers=1)
                r.pop("_layers")
                subs["llama70b"] = r
                torch.cuda.empty_cache()
                r = run_gqa(W.LLAMA8B_DECODE, args, dev, world, rank, clk, K, fp8=True)
                r.pop("_layers")
                subs["llama8b_fp8"] = r
                torch.cuda.empty_cache()
                subs["mla"] = run_mla(args, dev, world, rank, clk,
                                      reps=max(2, -(-K // mla_layers(args))))
                torch.cuda.empty_cache()
                subs["prefill"] = run_prefill(args, dev, world, rank, clk, min(K, 20))
                torch.cuda.empty_cache()
                subs["dir_1m"] = run_dir(args, dev, world, rank, clk, min(K, 20))
                for s in subs.values():
                    for k_ in ("metric", "n_gpus", "warmup", "higher_is_better", "scaling",
                               "vs_baseline", "dtype", "data"):
                        s.pop(k_, None)
                line["workloads"] = subs
    finally:
        clk.stop()
    line["clocks"] = clk.summary()
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
