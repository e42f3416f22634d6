"""Pins for the QKV projection + RMSNorm prologue oracle
(oracle/qkv_prologue.py): finite differences, torch.func.jvp of an
independent torch routine (F.rms_norm), invariants of RMSNorm, linearity,
head locality; plus planted mistakes that the pins must catch."""
import os
import types

import numpy as np
import pytest
import torch

from oracle import qkv_prologue

SRC = os.path.abspath(qkv_prologue.__file__)


def _inputs(seed, B=2, L=5, H=3, d=8, D=12):
    r = np.random.default_rng(seed)
    return (r.standard_normal((B * L, D)), r.standard_normal((B * L, D)),
            r.standard_normal((3 * H * d, D)) / np.sqrt(D), 1 + 0.2 * r.standard_normal(d),
            1 + 0.2 * r.standard_normal(d), (B, L, H, d))


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def pin_finite_difference(m):
    x, xd, w, gq, gk, (B, L, H, d) = _inputs(1)
    eps = 1e-6
    out = m.qkv_rmsnorm_jvp(x, xd, w, gq, gk, B, L, H, d)
    plus = m.qkv_rmsnorm_jvp(x + eps * xd, xd, w, gq, gk, B, L, H, d)
    minus = m.qkv_rmsnorm_jvp(x - eps * xd, xd, w, gq, gk, B, L, H, d)
    for i in range(3):
        fd = (plus[i] - minus[i]) / (2 * eps)
        assert _rel(out[3 + i], fd) < 1e-7, f"tangent {i}: {_rel(out[3 + i], fd)}"


def pin_torch_jvp(m):
    """Against torch.func.jvp of a torch fp64 prologue built on F.rms_norm."""
    x, xd, w, gq, gk, (B, L, H, d) = _inputs(2)
    out = m.qkv_rmsnorm_jvp(x, xd, w, gq, gk, B, L, H, d, eps=1e-6)
    W = torch.from_numpy(w)
    Gq, Gk = torch.from_numpy(gq), torch.from_numpy(gk)

    def f(xx):
        y = xx @ W.T
        parts = [y[:, i * H * d:(i + 1) * H * d].reshape(B, L, H, d).transpose(1, 2) for i in range(3)]
        q = torch.nn.functional.rms_norm(parts[0], (d,), weight=Gq, eps=1e-6)
        k = torch.nn.functional.rms_norm(parts[1], (d,), weight=Gk, eps=1e-6)
        return q, k, parts[2]
    prim, tang = torch.func.jvp(f, (torch.from_numpy(x),), (torch.from_numpy(xd),))
    for i in range(3):
        assert _rel(out[i], prim[i].numpy()) < 1e-12, f"primal {i}"
        assert _rel(out[3 + i], tang[i].numpy()) < 1e-12, f"tangent {i}"


def pin_scale_invariance(m):
    """RMSNorm (eps = 0) is homogeneous of degree 0: along x' = x, q' = k' = 0
    while the linear v' = v."""
    x, _, w, gq, gk, (B, L, H, d) = _inputs(3)
    q, k, v, qd, kd, vd = m.qkv_rmsnorm_jvp(x, x, w, gq, gk, B, L, H, d, eps=0.0)
    assert np.max(np.abs(qd)) < 1e-12 and np.max(np.abs(kd)) < 1e-12
    assert _rel(vd, v) < 1e-14


def pin_unit_rms_and_orthogonal_tangent(m):
    """gamma = 1, eps = 0: every q row has unit RMS, and its tangent is
    orthogonal to it (d/de of a constant norm)."""
    x, xd, w, _, _, (B, L, H, d) = _inputs(4)
    one = np.ones(d)
    q, k, v, qd, kd, vd = m.qkv_rmsnorm_jvp(x, xd, w, one, one, B, L, H, d, eps=0.0)
    for a, ad in ((q, qd), (k, kd)):
        assert np.allclose(np.mean(a * a, axis=-1), 1.0, rtol=0, atol=1e-13)
        assert np.max(np.abs(np.sum(a * ad, axis=-1))) < 1e-12


def pin_linearity(m):
    x, xd, w, gq, gk, (B, L, H, d) = _inputs(5)
    xe = np.random.default_rng(6).standard_normal(x.shape)
    a = m.qkv_rmsnorm_jvp(x, xd, w, gq, gk, B, L, H, d)
    b = m.qkv_rmsnorm_jvp(x, xe, w, gq, gk, B, L, H, d)
    c = m.qkv_rmsnorm_jvp(x, 2 * xd - 3 * xe, w, gq, gk, B, L, H, d)
    for i in range(3, 6):
        assert _rel(c[i], 2 * a[i] - 3 * b[i]) < 1e-12


def pin_head_locality(m):
    """Changing the weight rows of q-head 1 changes q/q' of head 1 only, in
    the [B, H, L, d] layout."""
    x, xd, w, gq, gk, (B, L, H, d) = _inputs(7)
    a = m.qkv_rmsnorm_jvp(x, xd, w, gq, gk, B, L, H, d)
    w2 = w.copy()
    w2[1 * d:2 * d] *= 1.7
    w2[1 * d] += 0.3
    b = m.qkv_rmsnorm_jvp(x, xd, w2, gq, gk, B, L, H, d)
    for i in (0, 3):
        diff = np.abs(a[i] - b[i]).max(axis=(0, 2, 3))
        assert diff[1] > 1e-3 and diff[0] == 0 and diff[2] == 0
    for i in (1, 2, 4, 5):
        assert np.array_equal(a[i], b[i])


def pin_token_layout(m):
    """Token t = b L + l lands at [b, :, l, :]: a single token's change moves
    only that position."""
    x, xd, w, gq, gk, (B, L, H, d) = _inputs(8)
    a = m.qkv_rmsnorm_jvp(x, xd, w, gq, gk, B, L, H, d)
    x2, xd2 = x.copy(), xd.copy()
    x2[1 * L + 3] += 1.0
    xd2[1 * L + 3] -= 0.5
    b = m.qkv_rmsnorm_jvp(x2, xd2, w, gq, gk, B, L, H, d)
    for i in range(6):
        diff = np.abs(a[i] - b[i]).max(axis=(1, 3))  # [B, L]
        changed = np.argwhere(diff > 0)
        assert changed.tolist() == [[1, 3]], f"output {i}: {changed.tolist()}"


PINS = [pin_finite_difference, pin_torch_jvp, pin_scale_invariance,
        pin_unit_rms_and_orthogonal_tangent, pin_linearity, pin_head_locality, pin_token_layout]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(qkv_prologue)


MUTANTS = [
    ("drop_cubic_term", "return gamma * y * r, gamma * (yd * r - y * r ** 3 * m)",
     "return gamma * y * r, gamma * (yd * r)"),
    ("tangent_without_gamma", "return gamma * y * r, gamma * (yd * r - y * r ** 3 * m)",
     "return gamma * y * r, (yd * r - y * r ** 3 * m)"),
    ("rms_over_tokens", "r = 1.0 / np.sqrt(np.mean(y * y, axis=-1, keepdims=True) + eps)",
     "r = 1.0 / np.sqrt(np.mean(y * y, axis=-2, keepdims=True) + eps)"),
    ("eps_outside_sqrt", "r = 1.0 / np.sqrt(np.mean(y * y, axis=-1, keepdims=True) + eps)",
     "r = 1.0 / (np.sqrt(np.mean(y * y, axis=-1, keepdims=True)) + eps)"),
    ("tangent_square_term", "m = np.mean(y * yd, axis=-1, keepdims=True)",
     "m = np.mean(yd * yd, axis=-1, keepdims=True)"),
    ("v_normalised", "v, vd = heads(y, 2), heads(yd, 2)",
     "v, vd = _rmsnorm_jvp(heads(y, 2), heads(yd, 2), 1.0, eps)"),
    ("q_gamma_for_k", "k, kd = _rmsnorm_jvp(heads(y, 1), heads(yd, 1), gk, eps)",
     "k, kd = _rmsnorm_jvp(heads(y, 1), heads(yd, 1), gq, eps)"),
    ("heads_tokens_swapped", "reshape(B, L, H, d).transpose(0, 2, 1, 3)",
     "reshape(B, H, L, d)"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, name
    mod = types.ModuleType(f"qkv_mutant_{name}")
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), mod.__dict__)
    caught = []
    for pin in PINS:
        try:
            pin(mod)
        except Exception:  # noqa: BLE001 - any failure counts
            caught.append(pin.__name__)
    assert caught, f"no pin caught {name}"
