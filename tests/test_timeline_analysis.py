"""The timeline tool's analysis of recorded stamps, decode and prefill (CPU only: the stamps
here are written by hand, the GPU build that records them is not involved)."""
import numpy as np

from paged_sparse_kv_sa_b200 import timeline as T


def _stamps():
    s = np.zeros((T.TL_WARPS, T.TL_SLOTS), dtype=np.uint64)
    # warp 0: two units; warp 1: one unit; warp 2 recorded nothing
    s[0, [0, 1, 2, 3, 4, 5, 12]] = [1000, 2000, 2500, 4500, 4000, 5000, 6000]
    s[0, 15] = 7 | (2 << 16) | (0 << 32)
    s[1, [0, 1, 2, 3, 4, 12]] = [1200, 2100, 2600, 5200, 4800, 7000]
    s[1, 15] = 9 | (1 << 16) | (1 << 32)
    return s


def test_phases_span_and_bytes():
    r = T.analyse(_stamps(), unit_bytes=8192)
    assert r["n_warps"] == 2 and r["n_units"] == 3 and r["units_recorded"] == 3
    assert abs(r["span"] - 6.0) < 1e-9                     # last partial at 7000 ns, first start 1000
    ph = dict(r["phases"])
    assert np.allclose(np.sort(ph["warp start"]), [0.0, 0.2])
    assert np.allclose(np.sort(ph["pages resolved"]), [1.5, 1.6])
    assert np.allclose(np.sort(ph["first unit's data in"]), [3.0, 3.8])
    assert np.allclose(np.sort(ph["last unit's data in"]), [3.8, 4.0])
    assert np.allclose(np.sort(ph["first unit's arithmetic (duration)"]), [0.4, 0.5])
    # units land at 3.0 us and 3.8 us (bucket 3) and 4.0 us (bucket 4)
    got = r["bytes_per_us"]
    assert got[3] == 2 * 8192 and got[4] == 8192 and got.sum() == 3 * 8192
    assert r["running"][0] == 2 and r["running"][5] == 1 and r["running"][6] == 0


def test_prefill_grid_analysis_recovers_per_tile_cost():
    # CTAs of 5 us fixed cost + 100 ns per tile, started 50 ns apart: the fit
    # recovers both, and utilisation / busy counts follow from the intervals
    from paged_sparse_kv_sa_b200.timeline import analyse_prefill_grid
    rng = np.random.default_rng(0)
    c = np.zeros((8192, 4), dtype=np.int64)
    for i in range(300):
        t = int(rng.integers(1, 100))
        s = 1000 + 50 * i
        c[i] = [s, s + 5000 + 100 * t, t, i % 148]
    g = analyse_prefill_grid(c, 148)
    assert g["ctas"] == 300 and g["tiles"] == int(c[:300, 2].sum())
    assert abs(g["per tile ns (fit)"] - 100.0) < 1e-6
    assert abs(g["per CTA fixed ns (fit)"] - 5000.0) < 1e-3
    dur = (c[:300, 1] - c[:300, 0]).sum()
    assert abs(g["sm utilisation"] - dur / (g["span_us"] * 1e3 * 148)) < 1e-12
    assert max(g["busy SMs over the span (2% steps)"]) <= 300
