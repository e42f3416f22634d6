"""Pins for the fp64 oracle: checks against facts fixed by the mathematics,
not against the oracle itself.

Every pin takes a loaded oracle library (so the mutation test can run the same
battery against deliberately broken copies) and raises AssertionError when the
oracle disagrees.  Kinds of evidence used:

- central finite differences of the oracle's own forward (eps = 1e-6), per
  tangent component, so the JVP terms are checked against the forward;
- ``torch.func.jvp`` and ``torch.logsumexp`` of a plain fp64 attention written
  with library calls (a routine independent of the C code);
- an explicitly materialised Jacobian built from the partial derivatives of
  softmax attention, checked column by column against finite differences;
- closed forms (V' = V with Q' = K' = 0; equal keys; one key; zero scale;
  equal values), linearity, key-permutation invariance, masking;
- hand-derived examples stored under tests/golden/.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "hand_examples.json")


def run(lib, q, k, v, qd, kd, vd, scale, kv_len=None, rows=None):
    return oracle.attn_jvp(q, k, v, qd, kd, vd, scale, kv_len=kv_len, rows=rows,
                           lib=lib, n_threads=2)


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(float(np.max(np.abs(b))), 1e-300))


def _rand(seed, B, H, Lq, Lk, d):
    r = np.random.default_rng(seed)
    return (r.standard_normal((B, H, Lq, d)), r.standard_normal((B, H, Lk, d)),
            r.standard_normal((B, H, Lk, d)), r.standard_normal((B, H, Lq, d)),
            r.standard_normal((B, H, Lk, d)), r.standard_normal((B, H, Lk, d)))


def _np_softmax_rows(S):
    m = S.max(axis=-1, keepdims=True)
    e = np.exp(S - m)
    return e / e.sum(axis=-1, keepdims=True)


# ---------------------------------------------------------------------------

def pin_finite_difference(lib):
    """O' against (O(x + eps x') - O(x - eps x')) / (2 eps), eps = 1e-6, with
    each tangent component alone and all together."""
    q, k, v, qd, kd, vd = _rand(11, 1, 2, 5, 7, 4)
    s = 0.7
    eps = 1e-6
    z = np.zeros_like
    for tq, tk, tv in [(qd, kd, vd), (qd, z(kd), z(vd)), (z(qd), kd, z(vd)), (z(qd), z(kd), vd)]:
        _, od, _ = run(lib, q, k, v, tq, tk, tv, s)
        op, _, _ = run(lib, q + eps * tq, k + eps * tk, v + eps * tv, tq, tk, tv, s)
        om, _, _ = run(lib, q - eps * tq, k - eps * tk, v - eps * tv, tq, tk, tv, s)
        fd = (op - om) / (2 * eps)
        assert rel(od, fd) < 1e-7, f"finite difference mismatch {rel(od, fd)}"


def _torch_attn(q, k, v, s):
    S = s * q @ k.transpose(-1, -2)
    return torch.softmax(S, dim=-1) @ v


def pin_torch_jvp(lib):
    """O, O' against torch.func.jvp of a plain fp64 attention and lse against
    torch.logsumexp, with and without a key mask."""
    B, H, Lq, Lk, d = 2, 3, 6, 9, 5
    q, k, v, qd, kd, vd = _rand(12, B, H, Lq, Lk, d)
    s = 0.45
    for kv_len in (None, np.array([5, 9], np.int32)):
        o, od, lse = run(lib, q, k, v, qd, kd, vd, s, kv_len=kv_len)
        for b in range(B):
            n = Lk if kv_len is None else int(kv_len[b])
            t = [torch.from_numpy(np.ascontiguousarray(x[b, :, :n] if x.shape[2] == Lk else x[b]))
                 for x in (q, k, v, qd, kd, vd)]
            ro, rod = torch.func.jvp(lambda a, bb, c: _torch_attn(a, bb, c, s),
                                     (t[0], t[1], t[2]), (t[3], t[4], t[5]))
            rl = torch.logsumexp(s * t[0] @ t[1].transpose(-1, -2), dim=-1)
            assert rel(o[b], ro.numpy()) < 1e-12, "O vs torch"
            assert rel(od[b], rod.numpy()) < 1e-12, "O' vs torch.func.jvp"
            assert np.max(np.abs(lse[b] - rl.numpy())) < 1e-12, "lse vs torch.logsumexp"


def pin_explicit_jacobian(lib):
    """Materialise dO/d(q, k, v) for Lq=3, Lk=4, d=2 from the partials
    dO_i/dS_ij = P_ij (v_j - O_i), dS_ij/dq_i = s k_j, dS_ij/dk_j = s q_i,
    dO_i/dv_j = P_ij I.  Check J x' against O' and every column of J against
    a central finite difference of the oracle's O."""
    Lq, Lk, d = 3, 4, 2
    q, k, v, qd, kd, vd = _rand(13, 1, 1, Lq, Lk, d)
    s = 0.9
    Q, K, V = q[0, 0], k[0, 0], v[0, 0]
    P = _np_softmax_rows(s * Q @ K.T)
    O = P @ V
    nq, nk = Lq * d, Lk * d
    J = np.zeros((Lq * d, nq + 2 * nk))
    for i in range(Lq):
        for c in range(d):
            row = i * d + c
            for j in range(Lk):
                g = P[i, j] * (V[j, c] - O[i, c])  # dO_ic / dS_ij
                for e in range(d):
                    J[row, i * d + e] += g * s * K[j, e]          # via q_i
                    J[row, nq + j * d + e] += g * s * Q[i, e]     # via k_j
                J[row, nq + nk + j * d + c] += P[i, j]            # via v_j
    t = np.concatenate([qd[0, 0].ravel(), kd[0, 0].ravel(), vd[0, 0].ravel()])
    _, od, _ = run(lib, q, k, v, qd, kd, vd, s)
    assert rel(od[0, 0].ravel(), J @ t) < 1e-12, "J x' vs O'"
    eps = 1e-6
    x0 = np.concatenate([q.ravel(), k.ravel(), v.ravel()])
    zq, zk = np.zeros_like(q), np.zeros_like(k)
    for col in range(J.shape[1]):
        xp = x0.copy(); xp[col] += eps
        xm = x0.copy(); xm[col] -= eps
        def split(x):
            return (x[:nq].reshape(q.shape), x[nq:nq + nk].reshape(k.shape),
                    x[nq + nk:].reshape(v.shape))
        op, _, _ = run(lib, *split(xp), zq, zk, zk, s)
        om, _, _ = run(lib, *split(xm), zq, zk, zk, s)
        fd = ((op - om) / (2 * eps)).ravel()
        assert np.max(np.abs(fd - J[:, col])) < 1e-7, f"Jacobian column {col}"


def pin_vdot_equals_v(lib):
    """Q' = K' = 0 and V' = V give S' = 0, so O' = P V = O exactly."""
    q, k, v, _, _, _ = _rand(14, 2, 2, 7, 11, 8)
    z = np.zeros_like
    o, od, _ = run(lib, q, k, v, z(q), z(k), v, 0.3)
    assert np.array_equal(o, od), "O' must equal O bit for bit"


def pin_equal_keys(lib):
    """All keys equal: P is uniform, O = mean V, lse = s q.k + ln n.  With
    K' = 0, O' = mean V' for any Q'; with K' != 0,
    O' = mean V' + (s/n) sum_j (q . (k'_j - mean k')) v_j."""
    B, H, Lq, Lk, d = 1, 2, 4, 6, 3
    q, k, v, qd, kd, vd = _rand(15, B, H, Lq, Lk, d)
    k[:] = k[:, :, :1, :]
    s = 0.8
    o, od, lse = run(lib, q, k, v, qd, np.zeros_like(kd), vd, s)
    assert rel(o, np.broadcast_to(v.mean(axis=2, keepdims=True), o.shape)) < 1e-14
    ref_lse = s * np.einsum("bhic,bhc->bhi", q, k[:, :, 0]) + math.log(Lk)
    assert np.max(np.abs(lse - ref_lse)) < 1e-13, "lse equal keys"
    assert rel(od, np.broadcast_to(vd.mean(axis=2, keepdims=True), od.shape)) < 1e-13
    _, od2, _ = run(lib, q, k, v, qd, kd, vd, s)
    kdc = kd - kd.mean(axis=2, keepdims=True)
    ref = vd.mean(axis=2, keepdims=True) + (s / Lk) * np.einsum(
        "bhij,bhjc->bhic", np.einsum("bhic,bhjc->bhij", q, kdc), v)
    assert rel(od2, ref) < 1e-12, "equal keys with K' != 0"


def pin_linearity(lib):
    """O' is linear in the tangent (Q', K', V')."""
    q, k, v, qd, kd, vd = _rand(16, 1, 3, 6, 10, 4)
    r = np.random.default_rng(17)
    qe, ke, ve = (r.standard_normal(x.shape) for x in (qd, kd, vd))
    a, b = 1.7, -0.6
    s = 0.5
    _, o1, _ = run(lib, q, k, v, qd, kd, vd, s)
    _, o2, _ = run(lib, q, k, v, qe, ke, ve, s)
    _, o3, _ = run(lib, q, k, v, a * qd + b * qe, a * kd + b * ke, a * vd + b * ve, s)
    assert rel(o3, a * o1 + b * o2) < 1e-13, "linearity"


def pin_single_key(lib):
    """Lk = 1: O = V, O' = V', lse = S."""
    q, k, v, qd, kd, vd = _rand(18, 2, 2, 5, 1, 4)
    s = 1.3
    o, od, lse = run(lib, q, k, v, qd, kd, vd, s)
    assert np.array_equal(o, np.broadcast_to(v, o.shape))
    assert np.array_equal(od, np.broadcast_to(vd, od.shape))
    assert rel(lse, s * np.einsum("bhic,bhc->bhi", q, k[:, :, 0])) < 1e-15


def pin_zero_scale(lib):
    """s = 0: uniform P, O = mean V, S' = 0 so O' = mean V', lse = ln Lk."""
    q, k, v, qd, kd, vd = _rand(19, 1, 2, 3, 9, 5)
    o, od, lse = run(lib, q, k, v, qd, kd, vd, 0.0)
    assert rel(o, np.broadcast_to(v.mean(axis=2, keepdims=True), o.shape)) < 1e-14
    assert rel(od, np.broadcast_to(vd.mean(axis=2, keepdims=True), od.shape)) < 1e-14
    assert np.max(np.abs(lse - math.log(9))) < 1e-14


def pin_equal_values(lib):
    """All V rows equal: sum_j P'_ij = 0 kills P' V, so O' = P V'."""
    q, k, v, qd, kd, vd = _rand(20, 1, 2, 5, 8, 3)
    v[:] = v[:, :, :1, :]
    s = 0.6
    _, od, _ = run(lib, q, k, v, qd, kd, vd, s)
    P = _np_softmax_rows(s * np.einsum("bhic,bhjc->bhij", q, k))
    assert rel(od, np.einsum("bhij,bhjc->bhic", P, vd)) < 1e-13


def pin_key_permutation(lib):
    """Permuting keys (with their values and tangents) changes nothing."""
    q, k, v, qd, kd, vd = _rand(21, 1, 2, 4, 9, 4)
    perm = np.random.default_rng(22).permutation(9)
    s = 0.7
    a = run(lib, q, k, v, qd, kd, vd, s)
    b = run(lib, q, k[:, :, perm], v[:, :, perm], qd, kd[:, :, perm], vd[:, :, perm], s)
    for x, y in zip(a, b):
        assert rel(y, x) < 1e-13, "key permutation"


def pin_masking(lib):
    """kv_len: padded keys (NaN here) never matter; 0 gives O = O' = 0 and
    lse = -inf; values above Lk clamp to Lk; negative values act as 0."""
    B, H, Lq, Lk, d = 3, 2, 4, 10, 4
    q, k, v, qd, kd, vd = _rand(23, B, H, Lq, Lk, d)
    s = 0.5
    n = [6, 1, 10]
    pk, pv, pkd, pvd = (x.copy() for x in (k, v, kd, vd))
    for b in range(B):
        for x in (pk, pv, pkd, pvd):
            x[b, :, n[b]:] = np.nan
    o, od, lse = run(lib, q, pk, pv, qd, pkd, pvd, s, kv_len=np.array(n, np.int32))
    for b in range(B):
        sl = lambda x: np.ascontiguousarray(x[b:b + 1, :, :n[b]])
        ro, rod, rl = run(lib, q[b:b + 1], sl(k), sl(v), qd[b:b + 1], sl(kd), sl(vd), s)
        assert np.array_equal(o[b:b + 1], ro) and np.array_equal(od[b:b + 1], rod)
        assert np.array_equal(lse[b:b + 1], rl)
    o, od, lse = run(lib, q, k, v, qd, kd, vd, s, kv_len=np.array([0, -3, 99], np.int32))
    assert np.all(o[:2] == 0) and np.all(od[:2] == 0) and np.all(np.isneginf(lse[:2]))
    full = run(lib, q[2:], k[2:], v[2:], qd[2:], kd[2:], vd[2:], s)
    assert np.array_equal(o[2:], full[0]) and np.array_equal(od[2:], full[1])


def pin_large_logits(lib):
    """Equal keys with s q.k near 1000: lse = s q.k + ln n and O = mean V stay
    finite (the softmax must subtract the row max)."""
    q = np.full((1, 1, 2, 2), 10.0)
    k = np.full((1, 1, 5, 2), 50.0)
    r = np.random.default_rng(24)
    v = r.standard_normal((1, 1, 5, 2))
    s = 1.0
    o, od, lse = run(lib, q, k, v, np.zeros_like(q), np.zeros_like(k), v, s)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    assert np.max(np.abs(lse - (1000.0 + math.log(5)))) < 1e-12
    assert rel(o, np.broadcast_to(v.mean(axis=2, keepdims=True), o.shape)) < 1e-14


def pin_row_subset(lib):
    """A row subset returns exactly the full result at those rows."""
    q, k, v, qd, kd, vd = _rand(25, 2, 2, 6, 7, 3)
    s = 0.4
    o, od, lse = run(lib, q, k, v, qd, kd, vd, s)
    rows = np.array([0, 5, 7, 13, 23], np.int64)
    so, sod, sl = run(lib, q, k, v, qd, kd, vd, s, rows=rows)
    assert np.array_equal(so, o.reshape(-1, 3)[rows])
    assert np.array_equal(sod, od.reshape(-1, 3)[rows])
    assert np.array_equal(sl, lse.reshape(-1)[rows])


def pin_bf16_inputs(lib):
    """bf16 bit patterns are widened exactly: same result as fp64 inputs."""
    from attention_jvp_fwd_b200.workloads import bf16_bits_to_f32, make_custom
    w = make_custom(1, 2, 9, 13, 8, seed=26)
    a = run(lib, *w.inputs(), w.scale)
    wide = [bf16_bits_to_f32(x).astype(np.float64) for x in w.inputs()]
    b = run(lib, *wide, w.scale)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def _golden_array(x):
    return np.array(x, dtype=object).astype(np.float64)


def pin_hand_examples(lib):
    """Cases worked out by hand (tests/golden/hand_examples.json)."""
    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        ins = [_golden_array(c[n]) for n in ("q", "k", "v", "q_dot", "k_dot", "v_dot")]
        kv = np.array(c["kv_len"], np.int32) if "kv_len" in c else None
        o, od, lse = run(lib, *ins, c["scale"], kv_len=kv)
        eo, eod, el = (_golden_array(c[n]) for n in ("o", "o_dot", "lse"))
        assert np.allclose(o, eo, rtol=1e-14, atol=1e-14), c["name"]
        assert np.allclose(od, eod, rtol=1e-14, atol=1e-14), c["name"]
        assert np.array_equal(np.isneginf(lse), np.isneginf(el)), c["name"]
        fin = np.isfinite(el)
        assert np.allclose(lse[fin], el[fin], rtol=1e-14, atol=1e-14), c["name"]
        if "lse_dot" in c:  # lse' = sum_j P_j S'_j, worked out by hand as well
            mu = run_mu(lib, *ins, c["scale"], kv_len=kv)[3]
            assert np.allclose(mu, _golden_array(c["lse_dot"]), rtol=1e-14, atol=1e-14), c["name"]


def run_mu(lib, q, k, v, qd, kd, vd, scale, kv_len=None, rows=None):
    return oracle.attn_jvp(q, k, v, qd, kd, vd, scale, kv_len=kv_len, rows=rows,
                           lib=lib, n_threads=2, lse_dot=True)


def pin_lse_dot_finite_difference(lib):
    """lse' against (lse(x + eps x') - lse(x - eps x')) / (2 eps), eps = 1e-6,
    for Q' and K' alone and together; V' must not move it."""
    q, k, v, qd, kd, vd = _rand(23, 1, 2, 5, 7, 4)
    s = 0.9
    eps = 1e-6
    z = np.zeros_like
    for tq, tk in [(qd, kd), (qd, z(kd)), (z(qd), kd)]:
        _, _, _, mu = run_mu(lib, q, k, v, tq, tk, vd, s)
        _, _, lp = run(lib, q + eps * tq, k + eps * tk, v, tq, tk, vd, s)
        _, _, lm = run(lib, q - eps * tq, k - eps * tk, v, tq, tk, vd, s)
        fd = (lp - lm) / (2 * eps)
        assert rel(mu, fd) < 1e-7, f"lse' finite difference mismatch {rel(mu, fd)}"
        _, _, _, mu0 = run_mu(lib, q, k, v, tq, tk, z(vd), s)
        assert np.array_equal(mu, mu0), "V' changed lse'"


def pin_lse_dot_torch_jvp(lib):
    """lse' against torch.func.jvp of torch.logsumexp over plain fp64 logits."""
    q, k, v, qd, kd, vd = _rand(29, 2, 2, 6, 9, 8)
    s = 0.35
    _, _, _, mu = run_mu(lib, q, k, v, qd, kd, vd, s)
    f = lambda qq, kk: torch.logsumexp(s * qq @ kk.transpose(-1, -2), dim=-1)
    _, ref = torch.func.jvp(f, (torch.from_numpy(q), torch.from_numpy(k)),
                            (torch.from_numpy(qd), torch.from_numpy(kd)))
    assert rel(mu, ref.numpy()) < 1e-12, f"lse' vs torch.func.jvp {rel(mu, ref.numpy())}"


def pin_lse_dot_closed_forms(lib):
    """One key: lse' = s (q'.k + q.k').  Equal keys with K' = 0: lse' = s q'.k.
    No valid key: lse' = 0.  Padded keys (NaN) do not reach it."""
    q, k, v, qd, kd, vd = _rand(31, 1, 1, 4, 1, 5)
    s = 1.3
    _, _, _, mu = run_mu(lib, q, k, v, qd, kd, vd, s)
    ref = s * (np.einsum("bhid,bhd->bhi", qd, k[:, :, 0]) + np.einsum("bhid,bhd->bhi", q, kd[:, :, 0]))
    assert rel(mu, ref) < 1e-13, "single-key lse'"
    q, k, v, qd, kd, vd = _rand(37, 1, 1, 3, 6, 4)
    k[:] = k[:, :, :1]
    _, _, _, mu = run_mu(lib, q, k, v, qd, np.zeros_like(kd), vd, s)
    ref = s * np.einsum("bhid,bhd->bhi", qd, k[:, :, 0])
    assert rel(mu, ref) < 1e-13, "equal-keys lse'"
    q, k, v, qd, kd, vd = _rand(41, 2, 1, 3, 8, 4)
    kv = np.array([0, 5], np.int32)
    _, _, _, mu = run_mu(lib, q, k, v, qd, kd, vd, s, kv_len=kv)
    assert np.all(mu[0] == 0.0), "lse' of a row without keys"
    k2, kd2 = k.copy(), kd.copy()
    k2[1, :, 5:] = np.nan
    kd2[1, :, 5:] = np.nan
    _, _, _, mu2 = run_mu(lib, q, k2, v, qd, kd2, vd, s, kv_len=kv)
    assert np.array_equal(mu[1], mu2[1]), "padded keys reached lse'"


PINS = [pin_finite_difference, pin_torch_jvp, pin_explicit_jacobian, pin_vdot_equals_v,
        pin_equal_keys, pin_linearity, pin_single_key, pin_zero_scale, pin_equal_values,
        pin_key_permutation, pin_masking, pin_large_logits, pin_row_subset,
        pin_bf16_inputs, pin_hand_examples, pin_lse_dot_finite_difference,
        pin_lse_dot_torch_jvp, pin_lse_dot_closed_forms]
