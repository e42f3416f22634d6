"""Helpers shared by the GPU tests: move generator output to the device, run
the CUDA path, and compare against the oracle with the parity metrics."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from attention_jvp_fwd_b200 import attn_jvp_fwd

# Tolerances for O, O' (max|err| / max|ref| over the compared outputs) and lse
# (absolute), as the parity bar states them.  The O and O' bars hold twice:
# over the whole compared tensor, and over every (b, h) slice against that
# slice's own max|ref|.  The second matters where tangents are scaled per
# head (the stress sweeps draw 10^u, u in [-3, 1]): there the largest heads
# set the whole-tensor denominator, and a wrong small-tangent head would hide
# under it.
TOL_O = 1e-2
TOL_OD = 2e-2
TOL_LSE = 1e-3


def to_dev(bits: np.ndarray, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device).view(torch.bfloat16)


def run_gpu(w, device="cuda", kv_len=None, scale=None):
    ins = [to_dev(x, device) for x in w.inputs()]
    kv = w.kv_len if kv_len is None else kv_len
    kvt = torch.from_numpy(np.asarray(kv, np.int32)).to(device) if kv is not None else None
    o, od, lse = attn_jvp_fwd(*ins, scale=w.scale if scale is None else scale, kv_len=kvt)
    torch.cuda.synchronize()
    return o, od, lse


def gpu_rows(o, od, lse, rows=None):
    """(o, od, lse, heads) as fp64 numpy, flattened to rows; `heads` is the
    flat (b, h) index of every returned row, for the per-head gate."""
    d = o.shape[-1]
    Lq = o.shape[-2]
    o = o.float().reshape(-1, d)
    od = od.float().reshape(-1, d)
    lse = lse.reshape(-1)
    if rows is not None:
        r = torch.from_numpy(np.asarray(rows, np.int64)).to(o.device)
        o, od, lse = o[r], od[r], lse[r]
        heads = np.asarray(rows, np.int64) // Lq
    else:
        heads = np.arange(o.shape[0], dtype=np.int64) // Lq
    return (o.cpu().numpy().astype(np.float64), od.cpu().numpy().astype(np.float64),
            lse.cpu().numpy().astype(np.float64), heads)


def ratio(err_max, ref_max):
    return err_max / ref_max if ref_max > 0 else err_max


def per_head_ratios(g, r, heads):
    """max|err| / max|ref| of every (b, h) slice: {head: ratio}."""
    out = {}
    for h in np.unique(heads):
        sel = heads == h
        out[int(h)] = float(ratio(np.max(np.abs(g[sel] - r[sel])), np.max(np.abs(r[sel]))))
    return out


def compare(g, ref, what=""):
    """Returns a dict of metrics; asserts the parity bar over the whole
    compared tensor and over every (b, h) slice (when `g` carries the head
    index of its rows, as gpu_rows returns it)."""
    d = g[0].shape[-1]
    go, god, gl = tuple(np.asarray(x).reshape(-1, d) for x in g[:2]) + (np.asarray(g[2]).reshape(-1),)
    ro, rod, rl = tuple(np.asarray(x).reshape(-1, d) for x in ref[:2]) + (np.asarray(ref[2]).reshape(-1),)
    eo = ratio(np.max(np.abs(go - ro)), np.max(np.abs(ro)))
    eod = ratio(np.max(np.abs(god - rod)), np.max(np.abs(rod)))
    fin = np.isfinite(rl)
    assert np.array_equal(np.isneginf(gl), np.isneginf(rl)), f"{what}: lse -inf pattern"
    el = float(np.max(np.abs(gl[fin] - rl[fin]))) if fin.any() else 0.0
    m = {"o": float(eo), "o_dot": float(eod), "lse": el}
    assert np.all(np.isfinite(go)) and np.all(np.isfinite(god)), f"{what}: non-finite output"
    assert eo <= TOL_O, f"{what}: O error {eo:.3e} > {TOL_O}"
    assert eod <= TOL_OD, f"{what}: O' error {eod:.3e} > {TOL_OD}"
    assert el <= TOL_LSE, f"{what}: lse error {el:.3e} > {TOL_LSE}"
    if len(g) > 3 and g[3] is not None:
        heads = np.asarray(g[3]).reshape(-1)
        ho = per_head_ratios(go, ro, heads)
        hod = per_head_ratios(god, rod, heads)
        worst_o = max(ho, key=ho.get)
        worst_od = max(hod, key=hod.get)
        m["o_head_max"] = ho[worst_o]
        m["o_dot_head_max"] = hod[worst_od]
        assert ho[worst_o] <= TOL_O, f"{what}: O error {ho[worst_o]:.3e} > {TOL_O} in head {worst_o}"
        assert hod[worst_od] <= TOL_OD, f"{what}: O' error {hod[worst_od]:.3e} > {TOL_OD} in head {worst_od}"
    return m


def oracle_ref(w, rows=None, kv_len=None, scale=None):
    kv = w.kv_len if kv_len is None else kv_len
    return oracle.attn_jvp(*w.inputs(), w.scale if scale is None else scale, kv_len=kv, rows=rows)
