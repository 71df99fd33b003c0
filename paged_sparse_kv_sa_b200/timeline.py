"""Per-warp timeline of the decode kernel at the Llama-8B-shaped decode workload.

    python -m paged_sparse_kv_sa_b200.timeline [--splits N] [--reps R] [--seed S] [--fp8]
    python -m paged_sparse_kv_sa_b200.timeline --prefill [--reps R]

Builds a diagnostic copy of the library (``_build/timeline/libsa_timeline.so``,
compiled with ``-DSA_DECODE_TIMELINE=1``: each decode warp records
``%globaltimer`` stamps for its first work item), selects the pages of the
workload once (``--fp8``: the same pages stored as FP8 E4M3 codes with
per-(page, kv head) scales), then times R decode launches, each after an L2
flush (a 256 MiB write, then a 256 MiB read), and prints where a launch's time
goes:

* the phases of the warps (when they start, have read their list entries,
  have resolved their pages, see their first and last unit's data, and have
  stored their partial; and how long the arithmetic on the first unit takes),
  as percentiles over the warps;
* the bytes that arrive in each microsecond (K + V of every unit whose data
  has landed), i.e. the aggregate rate at which the launch moves its bytes;
* how many warps are still running in each microsecond.

Times are microseconds from the first warp's start, for the launch whose
span (first start to last partial stored) is the median of the R launches.
The CUDA-event time of each launch is printed beside its span.

``--prefill``: the block-union chunked prefill instead (the tcgen05 many-row
kernel, built with ``-DSA_PREFILL_TIMELINE=1``): the first CTAs of a launch
stamp the SM clock per key tile -- the MMA thread's waits (K tile in, P of
each row tile in) and issues, and the softmax warps' phases (scores in, row
maxima exchanged and done, each half of the probabilities written) -- and the
tool prints the median cycles of each step of a key tile's round trip.  GPU only; the library proper
(``libsa.so``) has no timeline code.
"""
from __future__ import annotations

import argparse
import ctypes
import os

import numpy as np

from . import _lib
from .build import OBJ, build

TL_WARPS, TL_SLOTS = 8192, 16


PT_CTAS, PT_ITERS, PT_SLOTS = 4, 256, 16


def _build_timeline_lib() -> str:
    obj_dir = os.path.join(OBJ, "timeline")
    out = os.path.join(obj_dir, "libsa_timeline.so")
    return build(defines=("SA_DECODE_TIMELINE=1", "SA_PREFILL_TIMELINE=1"), out=out,
                 obj_dir=obj_dir)


def analyse_prefill(stamps: np.ndarray):
    """Median cycles of each step of a key tile's round trip, per CTA, from the
    [CTAs, iterations, 16] clock stamps of one launch (tiles 2.. n-2: steady state)."""
    out = []
    for c in range(stamps.shape[0]):
        st = stamps[c].astype(np.int64)
        n = int(st[0, 11])
        n_rec = min(n, st.shape[0])          # tiles past the record's end are not stamped
        if n_rec < 6 or st[0, 10] == 0:
            continue
        j = np.arange(2, n_rec - 3)
        med = lambda v: float(np.median(v))   # noqa: E731
        row = {
            "tiles": n,
            "per tile (K in to next K in, MMA thread)": med(st[j + 1, 0] - st[j, 0]),
            "softmax A: S in -> partial maxima exchanged": med(st[j, 12] - st[j, 4]),
            "softmax A: -> row max (and O rescale) done": med(st[j, 13] - st[j, 12]),
            "softmax A: -> P of keys 0-63 written": med(st[j, 5] - st[j, 13]),
            "softmax A: S in -> P of keys 64-127 written": med(st[j, 6] - st[j, 4]),
            "softmax B: S in -> row max done": med(st[j, 15] - st[j, 7]),
            "softmax B: row max done -> P of keys 0-63 written": med(st[j, 8] - st[j, 15]),
            "P_A (second half) in at the MMA thread after S_A in": med(st[j, 2] - st[j, 4]),
            "MMA thread: P_A(j) in -> K(j+1) in": med(st[j + 1, 0] - st[j, 2]),
            "MMA thread: K(j+1) in -> P_B(j) in": med(st[j, 3] - st[j + 1, 0]),
            "MMA thread: P_B(j) in -> QK_B(j+1) issued": med(st[j + 1, 1] - st[j, 3]),
            "MMA thread: QK_B(j+1) issued -> P_A(j+1) in": med(st[j + 1, 2] - st[j + 1, 1]),
            "softmax A: P(j) written -> S(j+1) in (PV + QK round trip)":
                med(st[j + 1, 4] - st[j, 5]),
            "softmax A: S(j) in -> S(j+1) in": med(st[j + 1, 4] - st[j, 4]),
            "launch to first tile (cycles)": float(st[0, 0] - st[0, 10]),
        }
        out.append(row)
    return out


PT_ALL = 8192


def analyse_prefill_grid(cta: np.ndarray, n_sm: int):
    """Whole-launch figures from the per-CTA [n, 4] records (entry ns, exit ns,
    active tiles, SM id; rows of CTAs that never ran are 0)."""
    c = cta[cta[:, 0] > 0].astype(np.int64)
    if len(c) == 0:
        return None
    t0 = c[:, 0].min()
    start, end, tiles = c[:, 0] - t0, c[:, 1] - t0, c[:, 2]
    dur = end - start
    span = float(end.max())
    work = tiles > 0
    # per-CTA duration = fixed + per_tile * tiles (least squares over CTAs with tiles)
    if work.sum() >= 2 and np.ptp(tiles[work]) > 0:
        per_tile, fixed = np.polyfit(tiles[work], dur[work], 1)
    else:
        per_tile, fixed = float("nan"), float("nan")
    # SMs busy over time, in 2% steps of the span
    grid = np.linspace(0, span, 51)
    busy = [int(((start <= g) & (end > g)).sum()) for g in grid[:-1]]
    return {
        "ctas": int(len(c)), "ctas with tiles": int(work.sum()),
        "tiles": int(tiles.sum()), "span_us": span / 1e3,
        "sm utilisation": float(dur.sum()) / (span * n_sm),
        "per tile ns (fit)": float(per_tile), "per CTA fixed ns (fit)": float(fixed),
        "CTA duration us p50 / p90 / max": (float(np.median(dur)) / 1e3,
                                            float(np.percentile(dur, 90)) / 1e3,
                                            float(dur.max()) / 1e3),
        "tiles per CTA p50 / p90 / max": (float(np.median(tiles[work])) if work.any() else 0.0,
                                          float(np.percentile(tiles[work], 90)) if work.any()
                                          else 0.0, int(tiles.max())),
        "last CTA start us": float(start.max()) / 1e3,
        "busy SMs over the span (2% steps)": busy,
    }


def main_prefill(lib, reps):
    import math

    import torch

    from . import workloads as W
    from ._lib import sa_block_union, sa_sparse_decode

    lib.sa_prefill_timeline.restype = ctypes.c_int
    lib.sa_prefill_timeline.argtypes = [ctypes.c_void_p, ctypes.c_int]
    lib.sa_prefill_cta_timeline.restype = ctypes.c_int
    lib.sa_prefill_cta_timeline.argtypes = [ctypes.c_void_p, ctypes.c_int]
    cbuf = np.zeros(PT_ALL * 4, dtype=np.int64)
    grids = []
    dev = torch.device("cuda", 0)
    cfg = W.UNION_PREFILL
    inp = W.prefill_inputs(cfg, seed=0, device=dev)
    scores = W.block_union_scores(cfg, seed=0, device=dev)
    tables, counts = sa_block_union(scores, cfg.Hkv, cfg.q_offset // cfg.block, cfg.top_k,
                                    cfg.n_sink_blocks)
    h2l = [h // (cfg.Hq // cfg.Hkv) for h in range(cfg.Hq)]
    buf = np.zeros(PT_CTAS * PT_ITERS * PT_SLOTS, dtype=np.int64)
    rows = []
    for r in range(reps + 1):
        lib.sa_prefill_timeline(buf.ctypes.data, buf.size)    # clears the stamps
        lib.sa_prefill_cta_timeline(cbuf.ctypes.data, cbuf.size)
        sa_sparse_decode(inp["q"], inp["k"], inp["v"], inp["page_table"], inp["seq_lens"],
                         tables.view(1, cfg.Hkv, -1), counts.view(1, cfg.Hkv), h2l,
                         1.0 / math.sqrt(cfg.D), 4)
        torch.cuda.synchronize()
        if lib.sa_prefill_timeline(buf.ctypes.data, buf.size) != 0:
            raise RuntimeError("sa_prefill_timeline failed")
        if lib.sa_prefill_cta_timeline(cbuf.ctypes.data, cbuf.size) != 0:
            raise RuntimeError("sa_prefill_cta_timeline failed")
        if r >= 1:
            rows += analyse_prefill(buf.reshape(PT_CTAS, PT_ITERS, PT_SLOTS).copy())
            n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
            grids.append(analyse_prefill_grid(cbuf.reshape(PT_ALL, 4).copy(), n_sm))
    print(f"workload {cfg.name}, 4 splits: {len(rows)} CTA records over {reps} launches "
          f"(the first {PT_CTAS} CTAs of each)")
    keys = [k for k in rows[0] if k != "tiles"]
    print(f"key tiles per CTA: {int(np.median([r_['tiles'] for r_ in rows]))} (median)\n")
    print("| step of a key tile (SM clock cycles, median over tiles, then over CTAs) | cycles |")
    print("|---|---:|")
    for k in keys:
        print(f"| {k} | {np.median([r_[k] for r_ in rows]):.0f} |")
    g = [x for x in grids if x is not None]
    if g:
        mid = sorted(g, key=lambda x: x["span_us"])[len(g) // 2]
        print(f"\nwhole launch (the launch of median span of {len(g)}):")
        for k, v in mid.items():
            print(f"  {k}: {v}")


def _pct(x, q):
    return float(np.percentile(x, q)) if len(x) else float("nan")


def analyse(stamps: np.ndarray, unit_bytes: int):
    """Per-launch tables from the [warps, 16] stamps of one launch."""
    rows = stamps[stamps[:, 0] != 0]
    t0 = rows[:, 0].min()
    us = lambda v: (v.astype(np.int64) - np.int64(t0)) / 1e3   # noqa: E731
    meta = rows[:, 15]
    n_units = ((meta >> 16) & 0xFFFF).astype(np.int64)
    start, ents, pages, end = us(rows[:, 0]), us(rows[:, 1]), us(rows[:, 2]), us(rows[:, 12])
    c0 = rows[:, 3] != 0
    comp0 = us(rows[c0, 3]) - us(rows[c0, 4])    # first unit: data in -> arithmetic done
    arr = []
    first, last = [], []
    for i in range(len(rows)):
        k = int(min(n_units[i], 8))
        a = us(rows[i, 4:4 + k]) if k else np.array([])
        arr.append(a)
        if k:
            first.append(a[0])
            last.append(a[-1])
    phases = [("warp start", start), ("list entries read", ents), ("pages resolved", pages),
              ("first unit's data in", np.array(first)), ("last unit's data in", np.array(last)),
              ("partial stored", end), ("first unit's arithmetic (duration)", comp0)]
    span = float(end.max())
    n_b = int(np.ceil(span)) + 1
    got = np.zeros(n_b)
    for a in arr:
        for v in a:
            got[min(int(v), n_b - 1)] += unit_bytes
    running = np.array([int(((start <= t + 1) & (end > t)).sum()) for t in range(n_b)])
    return dict(phases=phases, span=span, bytes_per_us=got, running=running, n_warps=len(rows),
                n_units=int(n_units.sum()), units_recorded=int(sum(len(a) for a in arr)))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--splits", type=int, default=0)
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--fp8", action="store_true")
    ap.add_argument("--prefill", action="store_true")
    args = ap.parse_args()
    path = _build_timeline_lib()
    lib = _lib.load(path)               # every wrapper below now calls this copy
    if args.prefill:
        return main_prefill(lib, args.reps)
    lib.sa_decode_timeline.restype = ctypes.c_int
    lib.sa_decode_timeline.argtypes = [ctypes.c_void_p, ctypes.c_int]

    import torch

    from . import workloads as W
    from .pipeline import SparseDecodeStep, default_splits
    from ._lib import sa_build_page_summaries, sa_build_page_summaries_fp8

    dev = torch.device("cuda", 0)
    cfg = W.LLAMA8B_DECODE
    inp = W.gqa_decode_inputs(cfg, seed=args.seed, device=dev)
    if args.fp8:
        kc, ks = W.fp8_pages(inp.pop("k"))
        vc, vs = W.fp8_pages(inp.pop("v"))
        sig = sa_build_page_summaries_fp8(kc, ks, inp["page_table"], inp["seq_lens"])
    else:
        sig = sa_build_page_summaries(inp["k"], inp["page_table"], inp["seq_lens"])
    bp = cfg.budget_tokens // cfg.page_size
    n_splits = args.splits or default_splits(cfg.B * cfg.Hkv, bp)
    step = SparseDecodeStep(cfg.B, cfg.T, cfg.Hq, cfg.Hkv, cfg.D, cfg.page_size,
                            inp["page_table"].shape[1], cfg.sink_tokens, cfg.local_tokens,
                            cfg.budget_tokens, n_splits=n_splits, device=dev)
    step.select(inp["q"], sig, inp["page_table"], inp["seq_lens"])
    torch.cuda.synchronize()
    buf = np.zeros(TL_WARPS * TL_SLOTS, dtype=np.uint64)
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(64 << 20, dtype=torch.int32, device=dev)
    unit_bytes = 16 * cfg.D * 2 * (1 if args.fp8 else 2)
    runs = []
    for r in range(args.reps + 3):
        flush_w.fill_(r & 0xFF)
        flush_r.sum()
        lib.sa_decode_timeline(buf.ctypes.data, buf.size)   # clears the stamps
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        if args.fp8:
            step.decode_fp8(inp["q"], kc, vc, ks, vs, inp["page_table"], inp["seq_lens"])
        else:
            step.decode(inp["q"], inp["k"], inp["v"], inp["page_table"], inp["seq_lens"])
        e1.record()
        torch.cuda.synchronize()
        st = lib.sa_decode_timeline(buf.ctypes.data, buf.size)
        if st != 0:
            raise RuntimeError(f"sa_decode_timeline: status {st}")
        if r >= 3:
            res = analyse(buf.reshape(TL_WARPS, TL_SLOTS).copy(), unit_bytes)
            res["event_us"] = e0.elapsed_time(e1) * 1e3
            runs.append(res)
    assert int(step.dev_error.item()) == 0
    runs.sort(key=lambda x: x["span"])
    med = runs[len(runs) // 2]
    kind = " (FP8 pages)" if args.fp8 else ""
    print(f"workload {cfg.name}{kind}, {n_splits} splits, {med['n_warps']} warps with an item, "
          f"{med['n_units']} units of {unit_bytes} B ({med['units_recorded']} stamped)")
    print("launches (span first start -> last partial stored / CUDA-event time), us: " +
          ", ".join(f"{x['span']:.1f}/{x['event_us']:.1f}" for x in runs))
    print(f"\nmedian launch: span {med['span']:.2f} us, event {med['event_us']:.2f} us\n")
    print("| phase (us from the first warp's start) | min | p10 | p50 | p90 | max |")
    print("|---|---:|---:|---:|---:|---:|")
    for name, v in med["phases"]:
        print(f"| {name} | {_pct(v, 0):.2f} | {_pct(v, 10):.2f} | {_pct(v, 50):.2f} | "
              f"{_pct(v, 90):.2f} | {_pct(v, 100):.2f} |")
    print("\n| us | data in (MB) | rate (TB/s) | warps running |")
    print("|---:|---:|---:|---:|")
    for t, (b, n) in enumerate(zip(med["bytes_per_us"], med["running"])):
        print(f"| {t}-{t + 1} | {b / 1e6:.2f} | {b / 1e6:.2f} | {n} |")


if __name__ == "__main__":
    main()
