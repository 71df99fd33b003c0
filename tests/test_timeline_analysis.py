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


def test_prefill_tile_analysis_reads_the_slots():
    # one CTA of 40 tiles with a period of 5000 cycles: K in at 5000 j, QK_B
    # issued 600 later, S_A in at +1000, P of A's halves at +3000 / +3200, P_A at
    # the MMA thread at +3300; the medians come back as those differences
    from paged_sparse_kv_sa_b200.timeline import analyse_prefill
    st = np.zeros((1, 256, 16), dtype=np.int64)
    n = 40
    for j in range(n):
        b = 100000 + 5000 * j
        st[0, j, 0], st[0, j, 1] = b, b + 600
        st[0, j, 4], st[0, j, 12], st[0, j, 13] = b + 1000, b + 1400, b + 1500
        st[0, j, 5], st[0, j, 6], st[0, j, 2] = b + 3000, b + 3200, b + 3300
        st[0, j, 7], st[0, j, 15], st[0, j, 8], st[0, j, 3] = b + 3500, b + 3900, b + 5400, b + 5600
    st[0, 0, 10], st[0, 0, 11] = 90000, n
    (row,) = analyse_prefill(st)
    assert row["tiles"] == n
    assert row["per tile (K in to next K in, MMA thread)"] == 5000
    assert row["softmax A: S in -> partial maxima exchanged"] == 400
    assert row["softmax A: -> P of keys 0-63 written"] == 1500
    assert row["softmax A: S in -> P of keys 64-127 written"] == 2200
    assert row["softmax A: P(j) written -> S(j+1) in (PV + QK round trip)"] == 3000
    assert row["MMA thread: P_A(j) in -> K(j+1) in"] == 1700
    assert row["launch to first tile (cycles)"] == 10000
