"""The trace summary (attention_jvp_fwd_b200.trace) on synthetic stamps with
known gaps, on the CPU."""
import math

import numpy as np
import pytest

from attention_jvp_fwd_b200 import trace as T


def _synthetic(ctas=2, tiles=12, period=2400, alt=False):
    t = np.zeros((ctas, tiles, T.EVENTS), np.int64)
    for c in range(ctas):
        base = 1000 + 77 * c
        for i in range(tiles):
            s0 = base + i * period
            t[c, i, T.K_LOAD] = s0 - 3000
            t[c, i, T.V_LOAD] = s0 - 2500
            t[c, i, T.S_ISSUE] = s0 - 1200
            gs = [i % 2] if alt else [0, 1]
            for g in gs:
                t[c, i, T.SM_S + 3 * g] = s0 + 10 * g
                t[c, i, T.SM_P + 3 * g] = s0 + 1300 + 10 * g
                t[c, i, T.SM_PD + 3 * g] = s0 + 2000 + 10 * g
            t[c, i, T.PA_ISSUE] = s0 + 1310 + 40
            t[c, i, T.PB_ISSUE] = s0 + 2010 + 25
    return t


def test_summary_recovers_known_gaps():
    s = T.summarize(_synthetic())
    assert s["period"] == 2400
    assert s["softmax_p"] == 1300 and s["softmax_pd"] == 700 and s["softmax_tile"] == 2000
    assert s["pa_after_p"] == 40 and s["pb_after_pd"] == 25
    assert s["k_lead"] == 1800
    assert s["s_wait"] == 1205  # median over both warpgroups (1200 and 1210)


def test_summary_of_tile_split_stamps():
    """d = 64: each warpgroup stamps only its own (alternate) key tiles, so
    its period is two key tiles."""
    s = T.summarize(_synthetic(alt=True))
    assert s["period"] == 4800
    # even tiles: P of warpgroup 0 (1300) -> 50; odd tiles: warpgroup 1 (1310) -> 40
    assert s["pa_after_p"] == 45


def test_missing_stamps_and_shape_check():
    t = np.zeros((1, 4, T.EVENTS), np.int64)
    s = T.summarize(t)
    assert all(math.isnan(v) for v in s.values())
    with pytest.raises(ValueError):
        T.summarize(np.zeros((1, 4, 5), np.int64))


@pytest.mark.parametrize("B,H,Lq,Lk,kv,grid", [
    (2, 1, 256, 100, [0, 100], 3),
    (4, 3, 1000, 512, [421, 81, 0, 600], 7),
    (1, 24, 4099, 4099, None, 148),
])
def test_query_tile_starts_follow_the_kernel_walk(B, H, Lq, Lk, kv, grid):
    """Every query tile in launch order goes to CTA w % grid; a CTA's key tiles
    are counted over its own query tiles, skipping those without keys."""
    nqt = -(-Lq // 128)
    expect = {c: [] for c in range(grid)}
    count = {c: 0 for c in range(grid)}
    for w in range(nqt * B * H):
        b = w // (nqt * H)
        nb = Lk if kv is None else min(max(kv[b], 0), Lk)
        nt = -(-nb // 64)
        if nt:
            expect[w % grid].append((count[w % grid], nt))
            count[w % grid] += nt
    for c in range(grid):
        assert T.query_tile_starts(B, H, Lq, Lk, kv, grid, c) == expect[c]


@pytest.mark.parametrize("alt", [False, True])
def test_boundary_gap(alt):
    """Query tiles of 3, 2 and 4 key tiles on one CTA; the gaps from the last
    P (sS' - c) of one query tile to the first S seen of the next are 900 and
    1500, so the median of the two is 1200."""
    starts = [[(0, 3), (3, 2), (5, 4)]]
    t = np.zeros((1, 9, T.EVENTS), np.int64)
    clock = 1000
    for i in range(9):
        if i == 3:
            clock += 900
        if i == 5:
            clock += 1500
        gs = [i % 2] if alt else [0, 1]
        for g in gs:
            t[0, i, T.SM_S + 3 * g] = clock
            t[0, i, T.SM_PD + 3 * g] = clock + 2000 - 5 * g
        clock += 2000
    r = T.summarize_boundaries(t, starts)
    assert r["boundaries"] == 2 and r["epilogue_gap"] == 1200


def test_boundary_gap_outside_the_stamped_range():
    starts = [[(0, 3), (3, 2)]]
    t = np.zeros((1, 3, T.EVENTS), np.int64)  # only the first query tile is stamped
    r = T.summarize_boundaries(t, starts)
    assert r["boundaries"] == 0 and math.isnan(r["epilogue_gap"])
