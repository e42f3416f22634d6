"""CUDA path against the fp64 oracle, element by element on seeded inputs.

Small cases compare every output; the full-size workloads compare a seeded
row subset (first/last rows, tile edges, random rows of every head), which is
exact parity for those rows since rows are independent."""
import math

import numpy as np
import pytest
import torch

from attention_jvp_fwd_b200 import workloads as W
from gpu_util import compare, gpu_rows, oracle_ref, run_gpu, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from attention_jvp_fwd_b200.build import build
    build()


def test_tiny_full():
    w = W.make("tiny", seed=0)
    m = compare(gpu_rows(*run_gpu(w)), oracle_ref(w), "tiny")
    print("tiny", m)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Lq,Lk", [(1, 1), (1, 64), (128, 64), (127, 129), (129, 63),
                                   (200, 1000), (64, 4099), (300, 65)])
def test_shapes_full(d, Lq, Lk):
    w = W.make_custom(2, 2, Lq, Lk, d, seed=Lq * 7 + Lk)
    compare(gpu_rows(*run_gpu(w)), oracle_ref(w), f"d{d} Lq{Lq} Lk{Lk}")


@pytest.mark.parametrize("d", [64, 128])
def test_kv_len_and_nan_padding(d):
    """Per-batch key lengths, including 0, 1, tile edges and > Lk; padded keys
    filled with NaN must not reach any output."""
    B, H, Lq, Lk = 8, 2, 130, 200
    kv = np.array([0, 1, 63, 64, 65, 128, 199, 500], np.int32)
    w = W.make_custom(B, H, Lq, Lk, d, seed=5, kv_len=kv)
    nan_bits = np.uint16(0x7FC0)
    for t in (w.k, w.v, w.k_dot, w.v_dot):
        for b in range(B):
            t[b, :, max(int(kv[b]), 0):] = nan_bits
    compare(gpu_rows(*run_gpu(w)), oracle_ref(w), f"kv_len d{d}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("scale", [-0.3, 0.0, 2.0])
def test_scale_values(scale, d):
    """A negative scale turns the row max into a row min; scale 0 makes P
    uniform."""
    w = W.make_custom(1, 3, 150, 300, d, seed=9)
    compare(gpu_rows(*run_gpu(w, scale=scale)), oracle_ref(w, scale=scale), f"scale {scale} d{d}")


@pytest.mark.parametrize("d", [64, 128])
def test_large_tangent_mean(d):
    """Tangent logits with a large common row mean (K' = K + 50): the
    centring constant keeps O' accurate (at d = 64 each softmax warpgroup
    has its own, merged in the epilogue)."""
    w = W.make_custom(1, 2, 256, 512, d, seed=10)
    kd = W.bf16_bits_to_f32(w.k_dot) + 50.0 * W.bf16_bits_to_f32(w.k)
    w.k_dot = W.bf16_round_bits(kd)
    qd = W.bf16_bits_to_f32(w.q_dot) + 20.0
    w.q_dot = W.bf16_round_bits(qd)
    compare(gpu_rows(*run_gpu(w)), oracle_ref(w), f"large tangent mean d{d}")


def test_deterministic_and_streams():
    w = W.make_custom(2, 4, 333, 777, 128, seed=11)
    a = run_gpu(w)
    s = torch.cuda.Stream()
    ins = [to_dev(x) for x in w.inputs()]
    with torch.cuda.stream(s):
        b = __import__("attention_jvp_fwd_b200").attn_jvp_fwd(*ins, scale=w.scale)
    s.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y), "same inputs must give bitwise equal outputs"


NAMED_FULL = ["t2i_self", "cross", "t2v_self"] + W._stress_names() + W._stress_sharp_names()


@pytest.mark.parametrize("name", NAMED_FULL)
def test_named_workload_rows(name):
    w = W.make(name, seed=0)
    per_head = 48 if w.Lk <= 4099 else 12
    rows = W.sample_rows(w, per_head=per_head)
    g = gpu_rows(*run_gpu(w), rows=rows)
    m = compare(g, oracle_ref(w, rows=rows), name)
    print(name, m)


@pytest.mark.parametrize("d", [64, 128])
def test_persistent_tile_walk(d):
    """More query tiles (288) than SMs, so every CTA walks several of them and
    the K/V rings, the S buffers and the barrier phases carry on from one
    query tile to the next; batches without keys (which every role skips)
    sit between ones with full, tail and single-key lengths, and padded keys
    hold NaN."""
    B, H, Lq, Lk = 6, 8, 700, 333
    kv = np.array([333, 0, 65, 1, 0, 200], np.int32)
    w = W.make_custom(B, H, Lq, Lk, d, seed=12, kv_len=kv)
    nan_bits = np.uint16(0x7FC0)
    for t in (w.k, w.v, w.k_dot, w.v_dot):
        for b in range(B):
            t[b, :, int(kv[b]):] = nan_bits
    compare(gpu_rows(*run_gpu(w)), oracle_ref(w), f"tile walk d{d}")


@pytest.mark.parametrize("d", [64, 128])
def test_all_keys_masked(d):
    """kv_len = 0 for every batch: no CTA has a key tile, so the loads, the
    MMAs and the softmax loops all skip every query tile; O = O' = 0 and
    lse = -inf everywhere."""
    B, H, Lq, Lk = 3, 2, 200, 100
    kv = np.zeros(B, np.int32)
    w = W.make_custom(B, H, Lq, Lk, d, seed=14, kv_len=kv)
    o, od, lse = run_gpu(w)
    assert not torch.any(o.float() != 0) and not torch.any(od.float() != 0)
    assert bool(torch.all(torch.isneginf(lse)))
    compare(gpu_rows(o, od, lse), oracle_ref(w), f"all masked d{d}")


@pytest.mark.parametrize("d", [64, 128])
def test_many_one_row_query_tiles(d):
    """300 query tiles of 3 rows each (Lq = 3, 150 heads per batch): every
    CTA walks two or three nearly empty query tiles."""
    w = W.make_custom(2, 150, 3, 700, d, seed=15)
    compare(gpu_rows(*run_gpu(w)), oracle_ref(w), f"one-row tiles d{d}")


@pytest.mark.parametrize("d", [64, 128])
def test_outputs_16_byte_aligned(d):
    """Output buffers that are 16-byte but not 32-byte aligned take the
    16-byte store path of the epilogue; the results must not change."""
    w = W.make_custom(2, 2, 200, 300, d, seed=31)
    ins = [to_dev(x) for x in w.inputs()]
    n = 2 * 2 * 200 * d
    base_o = torch.empty(n + 16, dtype=torch.bfloat16, device="cuda")
    base_od = torch.empty(n + 16, dtype=torch.bfloat16, device="cuda")
    o = base_o[8:8 + n].view(2, 2, 200, d)     # 8 bf16 = 16 bytes past a 256-byte boundary
    od = base_od[8:8 + n].view(2, 2, 200, d)
    assert o.data_ptr() % 32 == 16 and od.data_ptr() % 32 == 16
    lse = torch.empty((2, 2, 200), dtype=torch.float32, device="cuda")
    from attention_jvp_fwd_b200 import attn_jvp_fwd
    attn_jvp_fwd(*ins, scale=w.scale, out=(o, od, lse))
    torch.cuda.synchronize()
    compare(gpu_rows(o, od, lse), oracle_ref(w), f"16-byte aligned outputs d{d}")
    ref = [t.clone() for t in attn_jvp_fwd(*ins, scale=w.scale)]
    torch.cuda.synchronize()
    assert torch.equal(o, ref[0]) and torch.equal(od, ref[1]) and torch.equal(lse, ref[2])


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("masked", [False, True])
def test_centring_window_underflow(d, masked):
    """One dominant key at index 40 and keys 0..31 about 120 logits below it:
    in the first key tile every p of keys 0..31 underflows to exactly 0, so
    the p-weighted centring window has zero weight.  The outputs must stay
    finite and match the oracle (the centring constant cancels in exact
    arithmetic, so the kernel may take any finite value there)."""
    B, H, Lq, Lk = 2, 2, 130, 200
    w = W.make_custom(B, H, Lq, Lk, d, seed=41,
                      kv_len=np.array([41, 200], np.int32) if masked else None)
    q = 0.1 * W.bf16_bits_to_f32(w.q)
    k = 0.1 * W.bf16_bits_to_f32(w.k)
    q[..., 0] = 10.0
    k[..., :32, 0] = -10.0   # keys 0..31: logit about -100 at scale 1
    k[..., 40, 0] = 2.0      # key 40: about +20
    w.q = W.bf16_round_bits(q)
    w.k = W.bf16_round_bits(k)
    o, od, lse = run_gpu(w, scale=1.0)
    assert bool(torch.all(torch.isfinite(o.float()))) and bool(torch.all(torch.isfinite(od.float())))
    assert bool(torch.all(torch.isfinite(lse)))
    compare(gpu_rows(o, od, lse), oracle_ref(w, scale=1.0), f"centring underflow d{d} masked={masked}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("split", [
    pytest.param(False, marks=pytest.mark.xfail(
        strict=True,
        reason="known limit: the centring constant comes from a query tile's first key tile; with sS' "
               "drifting by about 40 along the keys the bf16 P (sS' - c) of the dominant keys carry "
               "rounding about 40 * 2^-9, and O' misses the 2e-2 bar (6.1e-2 at d = 64, 8.1e-2 at d = 128)")),
    True])
def test_rescale_every_key_tile(d, split):
    """Logits and tangent logits that grow along the key axis (0.1 per key
    at scale 1, about 9 log2 units per 64-key tile): the row max passes the
    lazy-rescale threshold (2^4) in every key tile, so O and O'_acc are
    rescaled every tile, each time after the previous tile's PV MMAs are
    done.  With the split, the 4 query tiles are cut into key ranges with a
    centring constant each, merged at the end: within the bar.  Without it,
    each query tile walks all 7 key tiles (a ragged last one of 17 keys) with
    the first tile's centring constant, and O' misses the bar."""
    from attention_jvp_fwd_b200 import api, attn_jvp_fwd
    B, H, Lq, Lk = 1, 2, 200, 6 * 64 + 17
    w = W.make_custom(B, H, Lq, Lk, d, seed=77)
    q = 0.1 * W.bf16_bits_to_f32(w.q)
    k = 0.1 * W.bf16_bits_to_f32(w.k)
    q[..., 0] = 1.0
    k[..., :, 0] = 0.1 * np.arange(Lk, dtype=np.float32)
    w.q = W.bf16_round_bits(q)
    w.k = W.bf16_round_bits(k)
    ins = [to_dev(x) for x in w.inputs()]
    o, od, lse = attn_jvp_fwd(*ins, scale=1.0, split=split)
    torch.cuda.synchronize()
    st, site = api.attn_jvp_check()
    assert st == 0, f"device status {st} at site {site}"
    compare(gpu_rows(o, od, lse), oracle_ref(w, scale=1.0), f"rescale every tile d{d} split={split}")
