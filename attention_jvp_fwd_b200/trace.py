"""Summaries of the stamps that ``attn_jvp_fwd_trace`` records.

For every CTA and key tile the trace build writes SM clock stamps (cycles) of
these pipeline events; a stamp that was not taken stays 0:

    0 K_LOAD     TMA warp issued the K/K' loads
    1 V_LOAD     TMA warp issued the V/V' loads
    2 S_ISSUE    MMA warp issued S = Q[K;K']^T and S' += Q'K^T
    3 PA_ISSUE   MMA warp issued O += P V (and O' += P V')
    4 PB_ISSUE   MMA warp issued O' += P (sS' - c) V
    5 + 3g       softmax warpgroup g saw S in TMEM
    6 + 3g       softmax warpgroup g signalled bf16 P
    7 + 3g       softmax warpgroup g signalled bf16 P (sS' - c)

Stamps compare only within a CTA (each SM has its own clock).  The summary
takes medians over key tiles, so the rare epilogue gap between query tiles
does not dominate; ``summarize_boundaries`` measures that gap on its own.
"""
import numpy as np

BM, BN = 128, 64  # query rows and keys per tile

K_LOAD, V_LOAD, S_ISSUE, PA_ISSUE, PB_ISSUE = 0, 1, 2, 3, 4
SM_S, SM_P, SM_PD = 5, 6, 7
EVENTS = 11


def _sm(g, ev):
    return ev + 3 * g


def summarize(trace, skip: int = 2) -> dict:
    """Median durations in cycles, from an int64 array [ctas, tiles, 11].

    The first ``skip`` key tiles of each CTA (pipeline fill) are left out.
    Keys of the result:
      period        S seen by a softmax warpgroup, from one of its key tiles to its next
      s_wait        S MMAs issued -> S seen (queue ahead of S plus the S MMAs)
      softmax_p     S seen -> P signalled
      softmax_pd    P signalled -> P (sS' - c) signalled
      softmax_tile  S seen -> P (sS' - c) signalled
      pa_after_p    last P signal of the tile -> P V MMAs issued
      pb_after_pd   last P (sS' - c) signal -> P (sS' - c) V MMAs issued
      k_lead        K loads issued -> S MMAs issued
    """
    t = np.asarray(trace, dtype=np.int64)
    if t.ndim != 3 or t.shape[2] != EVENTS:
        raise ValueError(f"expected [ctas, tiles, {EVENTS}], got {t.shape}")
    t = t[:, skip:, :]
    out = {k: [] for k in ("period", "s_wait", "softmax_p", "softmax_pd", "softmax_tile",
                           "pa_after_p", "pb_after_pd", "k_lead")}
    for c in range(t.shape[0]):
        tc = t[c]
        for g in (0, 1):
            seen = tc[:, _sm(g, SM_S)]
            idx = np.nonzero(seen)[0]
            if len(idx) >= 2:
                out["period"].extend(np.diff(seen[idx]).tolist())
            for i in idx:
                row = tc[i]
                if row[S_ISSUE]:
                    out["s_wait"].append(row[_sm(g, SM_S)] - row[S_ISSUE])
                if row[_sm(g, SM_P)]:
                    out["softmax_p"].append(row[_sm(g, SM_P)] - row[_sm(g, SM_S)])
                if row[_sm(g, SM_PD)] and row[_sm(g, SM_P)]:
                    out["softmax_pd"].append(row[_sm(g, SM_PD)] - row[_sm(g, SM_P)])
                    out["softmax_tile"].append(row[_sm(g, SM_PD)] - row[_sm(g, SM_S)])
        for i in range(tc.shape[0]):
            row = tc[i]
            p = [row[_sm(g, SM_P)] for g in (0, 1) if row[_sm(g, SM_P)]]
            pd = [row[_sm(g, SM_PD)] for g in (0, 1) if row[_sm(g, SM_PD)]]
            if p and row[PA_ISSUE]:
                out["pa_after_p"].append(row[PA_ISSUE] - max(p))
            if pd and row[PB_ISSUE]:
                out["pb_after_pd"].append(row[PB_ISSUE] - max(pd))
            if row[K_LOAD] and row[S_ISSUE]:
                out["k_lead"].append(row[S_ISSUE] - row[K_LOAD])
    return {k: float(np.median(v)) if v else float("nan") for k, v in out.items()}


def query_tile_starts(B: int, H: int, Lq: int, Lk: int, kv_len, grid: int, cta: int) -> list:
    """(first key tile, key tiles) of each query tile that CTA ``cta`` walks,
    in its own key-tile count, the way the kernel walks them: query tiles
    w = cta, cta + grid, ... of the ceil(Lq / 128) * B * H tiles, the query
    tile varying fastest, tiles without keys skipped.  ``kv_len`` is None or a
    sequence of B key lengths (clamped to [0, Lk])."""
    nqt = (Lq + BM - 1) // BM
    starts, gk = [], 0
    for w in range(cta, nqt * B * H, grid):
        b = (w // nqt) // H
        nb = Lk if kv_len is None else min(max(int(kv_len[b]), 0), Lk)
        nt = (nb + BN - 1) // BN
        if nt == 0:
            continue
        starts.append((gk, nt))
        gk += nt
    return starts


def summarize_boundaries(trace, starts_per_cta) -> dict:
    """Median clocks from the last P (sS' - c) signal of a query tile to the
    first S seen of the CTA's next query tile (the epilogue and the refill
    between them), over the boundaries whose stamps are in the trace.
    ``starts_per_cta[c]`` is ``query_tile_starts`` for CTA c."""
    t = np.asarray(trace, dtype=np.int64)
    gaps = []
    for c, starts in enumerate(starts_per_cta[: t.shape[0]]):
        tc = t[c]
        for (g0, n0), (g1, _) in zip(starts, starts[1:]):
            last = g0 + n0 - 1
            if g1 >= tc.shape[0]:
                break
            pd = [tc[last, _sm(g, SM_PD)] for g in (0, 1) if tc[last, _sm(g, SM_PD)]]
            seen = [tc[g1, _sm(g, SM_S)] for g in (0, 1) if tc[g1, _sm(g, SM_S)]]
            if pd and seen:
                gaps.append(min(seen) - max(pd))
    return {"boundaries": len(gaps),
            "epilogue_gap": float(np.median(gaps)) if gaps else float("nan")}


def format_summary(s: dict) -> str:
    return "\n".join(f"{k:14s} {v:10.0f} cycles" for k, v in s.items())


def main(argv=None):
    """``python -m attention_jvp_fwd_b200.trace [--workload NAME] [--tiles N]``:
    trace one launch on a named synthetic workload (after warm-up launches)
    and print the summary."""
    import argparse

    import torch

    from . import api
    from . import workloads as W
    from .build import build

    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="t2i_self")
    ap.add_argument("--tiles", type=int, default=128)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--seed", type=int, default=0)
    args = ap.parse_args(argv)
    build()
    w = W.make(args.workload, seed=args.seed)
    if w.zero_kv_dot:
        raise SystemExit("the trace build takes all six inputs; pick a workload with K', V'")
    dev = torch.device("cuda", 0)
    ins = [torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16) for x in w.inputs()]
    kv = torch.from_numpy(w.kv_len).to(dev) if w.kv_len is not None else None
    for _ in range(args.warmup):
        api.attn_jvp_fwd(*ins, scale=w.scale, kv_len=kv)
    *_, tr = api.attn_jvp_fwd_trace(*ins, scale=w.scale, kv_len=kv, tiles=args.tiles)
    torch.cuda.synchronize(dev)
    st, site = api.attn_jvp_check()
    if st != 0:
        raise SystemExit(f"device status {st} at site {site}")
    print(f"{w.name}: B={w.B} H={w.H} Lq={w.Lq} Lk={w.Lk} d={w.d}; {tr.shape[0]} CTAs x "
          f"{tr.shape[1]} key tiles stamped")
    t = tr.cpu().numpy()
    print(format_summary(summarize(t)))
    n_tiles = ((w.Lq + BM - 1) // BM) * w.B * w.H
    grid = min(n_tiles, torch.cuda.get_device_properties(dev).multi_processor_count)
    starts = [query_tile_starts(w.B, w.H, w.Lq, w.Lk, w.kv_len, grid, c) for c in range(t.shape[0])]
    bs = summarize_boundaries(t, starts)
    if bs["boundaries"]:
        print(f"{'epilogue_gap':14s} {bs['epilogue_gap']:10.0f} cycles  (last P(sS'-c) of a query "
              f"tile -> first S seen of the next; {bs['boundaries']} boundaries)")
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
