"""bench.py's multi-rank bookkeeping on CPU: two gloo ranks, max of the
per-rank times and sum of the per-rank work, as the GPU run does over NCCL."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ws, r, local = bench.dist_setup()
        assert (ws, r, local) == (world, rank, rank)
        ms, flops = bench.aggregate(10.0 + 5.0 * rank, 1e12 * (rank + 1), True, "cpu")
        out[rank] = (ms, flops)
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation():
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    for r in range(2):
        ms, flops = res[r]
        assert ms == 15.0
        assert flops == 3e12


def test_single_rank_aggregation_is_identity():
    assert bench.aggregate(3.5, 7.0, False) == (3.5, 7.0)


def test_algorithmic_bytes_and_flops():
    from attention_jvp_fwd_b200 import workloads as W
    w = W.make_custom(2, 3, 100, 50, 64, seed=0, kv_len=[50, 10])
    assert w.flops_nominal() == 12 * 100 * 50 * 64 * 6
    assert w.flops_valid() == 12 * 100 * 64 * 3 * (50 + 10)
    rows = np.arange(2 * 3 * 100)
    assert bench.row_flops(w, rows) == w.flops_valid()
    b = bench.algorithmic_bytes(w)
    assert b == 2 * 64 * (2 * 600 + 4 * 3 * 60) + 4 * 600 * 64 + 4 * 600


def test_reference_arm_runs_on_cpu(capsys):
    import json
    rc = bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "3",
                     "--warmup", "1"])
    assert rc == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
