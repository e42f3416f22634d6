"""Pins for the sCM tangent-normalised loss oracle (oracle/scm_loss.py):
closed forms, exact rational arithmetic, finite differences and invariances,
plus planted mistakes in copies of its source that the pins must catch."""
import os
import types
from fractions import Fraction

import numpy as np
import pytest

from oracle import scm_loss

SRC = os.path.abspath(scm_loss.__file__)


def _rand(seed, B, N):
    r = np.random.default_rng(seed)
    return r.standard_normal((B, N)), r.standard_normal((B, N)), r.standard_normal((B, N))


def pin_zero_tangent(m):
    """g = 0: the target is F- itself."""
    f, fe, _ = _rand(1, 3, 17)
    loss, grad = m.scm_tangent_loss(f, fe, np.zeros_like(f))
    assert np.allclose(loss, np.sum((f - fe) ** 2, axis=1), rtol=1e-14, atol=0)
    assert np.allclose(grad, 2 * (f - fe), rtol=1e-14, atol=0)


def pin_exact_rationals(m):
    """Small integer inputs against exact rational arithmetic."""
    f = np.array([[1.0, 0.0, 2.0], [0.5, -1.0, 0.25]])
    fe = np.array([[0.0, 0.0, 1.0], [0.0, 0.5, 0.0]])
    g = np.array([[3.0, 4.0, 0.0], [1.0, -2.0, 2.0]])
    c = Fraction(1, 10)
    loss, grad = m.scm_tangent_loss(f, fe, g, c=0.1)
    for b in range(2):
        n = sum(Fraction(x) ** 2 for x in g[b])
        r = [Fraction(f[b, i]) - Fraction(fe[b, i]) - Fraction(g[b, i]) / (n + c) for i in range(3)]
        assert abs(loss[b] - float(sum(x * x for x in r))) <= 1e-15 * max(1.0, loss[b])
        for i in range(3):
            assert abs(grad[b, i] - float(2 * r[i])) <= 1e-15


def pin_finite_difference(m):
    """grad = d loss / dF by central differences (g and F- fixed)."""
    f, fe, g = _rand(3, 2, 6)
    loss, grad = m.scm_tangent_loss(f, fe, g)
    eps = 1e-6
    for b in range(2):
        for i in range(6):
            fp, fm = f.copy(), f.copy()
            fp[b, i] += eps
            fm[b, i] -= eps
            fd = (m.scm_tangent_loss(fp, fe, g)[0][b] - m.scm_tangent_loss(fm, fe, g)[0][b]) / (2 * eps)
            assert abs(fd - grad[b, i]) < 1e-7 * max(1.0, abs(grad[b, i]))


def pin_shift_invariance(m):
    """Adding the same field to F and F- changes nothing."""
    f, fe, g = _rand(4, 2, 9)
    d = np.random.default_rng(5).standard_normal(f.shape)
    a = m.scm_tangent_loss(f, fe, g)
    b = m.scm_tangent_loss(f + d, fe + d, g)
    assert np.allclose(a[0], b[0], rtol=1e-12, atol=1e-12)


def pin_projection_target(m):
    """With c = 0 the target step is g / |g|^2: F = F- + g / |g|^2 gives loss 0."""
    _, fe, g = _rand(6, 3, 11)
    f = fe + g / np.sum(g * g, axis=1, keepdims=True)
    loss, _ = m.scm_tangent_loss(f, fe, g, c=0.0)
    assert np.all(loss < 1e-28)


def pin_samples_independent(m):
    """Each sample's loss depends on that sample only."""
    f, fe, g = _rand(7, 4, 5)
    full, _ = m.scm_tangent_loss(f, fe, g)
    for b in range(4):
        one, _ = m.scm_tangent_loss(f[b:b + 1], fe[b:b + 1], g[b:b + 1])
        assert one[0] == full[b]


def pin_bf16_widening(m):
    """bf16 bit patterns widen exactly: 1.5 = 0x3FC0, -2 = 0xC000, 0.25 = 0x3E80."""
    bits = np.array([[0x3FC0, 0xC000, 0x3E80]], np.uint16)
    vals = np.array([[1.5, -2.0, 0.25]])
    a = m.scm_tangent_loss(bits, bits * 0, bits)
    b = m.scm_tangent_loss(vals, vals * 0, vals)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


PINS = [pin_zero_tangent, pin_exact_rationals, pin_finite_difference, pin_shift_invariance,
        pin_projection_target, pin_samples_independent, pin_bf16_widening]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(scm_loss)


MUTANTS = [
    ("norm_not_squared", "n = np.sum(g * g, axis=1)", "n = np.sqrt(np.sum(g * g, axis=1))"),
    ("c_dropped", "r = f - fe - g / (n + c)[:, None]", "r = f - fe - g / n[:, None]"),
    ("tangent_sign", "r = f - fe - g / (n + c)[:, None]", "r = f - fe + g / (n + c)[:, None]"),
    ("grad_factor", "return loss, 2.0 * r", "return loss, r"),
    ("loss_not_squared", "loss = np.sum(r * r, axis=1)", "loss = np.sum(np.abs(r), axis=1)"),
    ("norm_over_batch", "n = np.sum(g * g, axis=1)", "n = np.sum(g * g)"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, name
    mod = types.ModuleType(f"scm_loss_mutant_{name}")
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), mod.__dict__)
    caught = []
    for pin in PINS:
        try:
            pin(mod)
        except Exception:  # noqa: BLE001 - any failure counts
            caught.append(pin.__name__)
    assert caught, f"no pin caught {name}"
