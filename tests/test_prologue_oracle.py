"""Pins of the oracle's input prologue (oracle/prologue.py): the L2 normalisation
of q and k and the gate activations.

Each pin compares with something other than the prologue's own formula: values
the closed forms fix at chosen points, an independently written expression of
the same function, the algebraic identities of the functions, and one property
of the recurrence itself (the exact write-over S_t k_t = v_t holds for raw keys
once they are normalised and beta -> 1).  A last group feeds plausible wrong
versions of the prologue through the same pins and checks each is rejected.
"""
import math

import numpy as np
import pytest

from oracle import oracle as O
from oracle import prologue as P


# ---------------------------------------------------------------- pins ----

def pin_softplus_points(f=P.log_alpha_from_logit):
    # -softplus at points where it has a closed form: ln 2 at 0, ln 4 at ln 3,
    # ln(1 + 1/3) at -ln 3
    np.testing.assert_allclose(f(0.0), -math.log(2.0), rtol=0, atol=1e-15)
    np.testing.assert_allclose(f(math.log(3.0)), -math.log(4.0), rtol=0, atol=1e-15)
    np.testing.assert_allclose(f(-math.log(3.0)), -math.log(4.0 / 3.0), rtol=0, atol=1e-15)
    # alpha = exp(log alpha) = 1 / (1 + e^x), written independently
    x = np.linspace(-30.0, 30.0, 121)
    np.testing.assert_allclose(np.exp(f(x)), 1.0 / (1.0 + np.exp(x)), rtol=1e-13, atol=0)
    # no overflow far out: -softplus(x) -> -x for large x, -> -e^x for very negative x
    np.testing.assert_allclose(f(800.0), -800.0, rtol=1e-15)
    np.testing.assert_allclose(f(-50.0), -math.exp(-50.0), rtol=1e-12)
    assert np.all(f(x) < 0)


def pin_sigmoid_points(f=P.beta_from_logit):
    np.testing.assert_allclose(f(0.0), 0.5, rtol=0, atol=1e-16)
    np.testing.assert_allclose(f(math.log(3.0)), 0.75, rtol=0, atol=1e-15)
    y = np.linspace(-40.0, 40.0, 161)
    np.testing.assert_allclose(f(-y), 1.0 - f(y), rtol=0, atol=1e-15)   # symmetry
    np.testing.assert_allclose(f(y) / f(-y), np.exp(y), rtol=1e-12)  # odds = e^y
    assert f(1000.0) == 1.0 and 0.0 <= f(-1000.0) < 1e-300 + 1e-400
    assert np.all((f(y) > 0) & (f(y) <= 1))


def pin_l2_normalise(f=P.l2_normalise):
    # (3, 4) has norm 5
    np.testing.assert_allclose(f([3.0, 4.0]), np.array([3.0, 4.0]) / math.sqrt(25.0 + P.EPS),
                               rtol=0, atol=1e-16)
    rng = np.random.default_rng(7)
    x = rng.standard_normal((5, 3, 16))
    n = f(x)
    # unit norm (up to EPS) along the last axis only, direction kept
    np.testing.assert_allclose(np.linalg.norm(n, axis=-1),
                               np.linalg.norm(x, axis=-1) / np.sqrt(
                                   np.linalg.norm(x, axis=-1) ** 2 + P.EPS), rtol=1e-14)
    np.testing.assert_allclose(np.sum(n * x, axis=-1),
                               np.linalg.norm(n, axis=-1) * np.linalg.norm(x, axis=-1),
                               rtol=1e-13)
    # scale invariance for a positive factor per row (exact up to EPS)
    s = rng.uniform(0.5, 4.0, size=(5, 3, 1))
    np.testing.assert_allclose(f(s * x), n, rtol=1e-6)
    # the zero vector stays zero (no division by zero)
    assert np.all(f(np.zeros(8)) == 0.0)


def pin_write_over_with_raw_inputs(apply=P.apply):
    """Raw, non-unit keys and gate logits: after the prologue, with beta -> 1 (a
    large write logit) the state writes over exactly: S_t k_hat_t = v_t."""
    rng = np.random.default_rng(11)
    B, T, H, Dk, Dv = 1, 6, 2, 8, 5
    q = 3.0 * rng.standard_normal((B, T, H, Dk))
    k = 5.0 * rng.standard_normal((B, T, H, Dk))
    v = rng.standard_normal((B, T, H, Dv))
    x = rng.standard_normal((B, T, H))
    y = np.full((B, T, H), 60.0)            # sigmoid(60) = 1 - 9e-27
    qh, kh, la, be = apply(q, k, x, y, True, True)
    for t in range(1, T + 1):
        _, S = O.forward(qh[:, :t], kh[:, :t], v[:, :t], la[:, :t], be[:, :t], None)
        for h in range(H):
            # |k_hat|^2 = |k|^2 / (|k|^2 + EPS): write-over to that precision
            np.testing.assert_allclose(S[0, h] @ kh[0, t - 1, h], v[0, t - 1, h], rtol=0,
                                       atol=1e-6)
    # and the read-out used the normalised query: o_t = S_t q_hat_t
    o, S = O.forward(qh, kh, v, la, be, None)
    np.testing.assert_allclose(o[0, -1, 0], S[0, 0] @ qh[0, -1, 0], rtol=1e-12)


PINS = [pin_softplus_points, pin_sigmoid_points, pin_l2_normalise, pin_write_over_with_raw_inputs]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_prologue_pin(pin):
    pin()


def test_apply_leaves_inputs_alone_without_flags():
    rng = np.random.default_rng(3)
    q, k = rng.standard_normal((2, 3, 4)), rng.standard_normal((2, 3, 4))
    la, be = -rng.uniform(size=(2, 3)), rng.uniform(size=(2, 3))
    out = P.apply(q, k, la, be, False, False)
    for a, b in zip(out, (q, k, la, be)):
        assert np.array_equal(a, b)


# ------------------------------------------------- planted mistakes ----
def _softplus_no_max(x):           # drops the max(x, 0) term
    x = np.asarray(x, float)
    return -np.log1p(np.exp(-np.abs(x)))


def _softplus_sign(x):             # log alpha = +softplus
    return -P.log_alpha_from_logit(x)


def _sigmoid_flipped(y):           # sigmoid(-y)
    return P.beta_from_logit(-np.asarray(y, float))


def _l2_wrong_axis(x):             # normalises over the first axis
    x = np.asarray(x, float)
    return x / np.sqrt(np.sum(x * x, axis=0, keepdims=True) + P.EPS)


def _l2_no_sqrt(x):                # divides by the squared norm
    x = np.asarray(x, float)
    return x / (np.sum(x * x, axis=-1, keepdims=True) + P.EPS)


def _apply_swapped_gates(q, k, la, be, l2, gl):   # beta from the decay logit
    q2, k2, _, _ = P.apply(q, k, la, be, l2, False)
    return q2, k2, P.log_alpha_from_logit(be), P.beta_from_logit(la)


MISTAKES = {
    "softplus_no_max": (pin_softplus_points, _softplus_no_max),
    "softplus_sign": (pin_softplus_points, _softplus_sign),
    "sigmoid_flipped": (pin_sigmoid_points, _sigmoid_flipped),
    "l2_wrong_axis": (pin_l2_normalise, _l2_wrong_axis),
    "l2_no_sqrt": (pin_l2_normalise, _l2_no_sqrt),
    "gates_swapped": (pin_write_over_with_raw_inputs, _apply_swapped_gates),
}


@pytest.mark.parametrize("name", sorted(MISTAKES))
def test_prologue_pins_reject_planted_mistake(name):
    pin, wrong = MISTAKES[name]
    with pytest.raises(AssertionError):
        pin(wrong)
