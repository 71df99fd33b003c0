"""Per-warp timeline of the decode kernel at the Llama-8B-shaped decode workload.

    python -m paged_sparse_kv_sa_b200.timeline [--splits N] [--reps R] [--seed S] [--fp8]

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
The CUDA-event time of each launch is printed beside its span.  GPU only; the
library proper (``libsa.so``) has no timeline code.
"""
from __future__ import annotations

import argparse
import ctypes
import os

import numpy as np

from . import _lib
from .build import OBJ, build

TL_WARPS, TL_SLOTS = 8192, 16


def _build_timeline_lib() -> str:
    obj_dir = os.path.join(OBJ, "timeline")
    out = os.path.join(obj_dir, "libsa_timeline.so")
    return build(defines=("SA_DECODE_TIMELINE=1",), out=out, obj_dir=obj_dir)


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
    args = ap.parse_args()
    path = _build_timeline_lib()
    lib = _lib.load(path)               # every wrapper below now calls this copy
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
