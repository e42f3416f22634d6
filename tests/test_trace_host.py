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
