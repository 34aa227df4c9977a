"""Pins of the oracle's channel-wise-gate rule (oracle.forward_cw, the Gated
DeltaNet-2 reading S_t = S_{t-1} Diag(alpha_t)(I - (b_t o k_t) k_t^T) + (w_t o v_t) k_t^T).

Each pin compares with something fixed independently of that code: the scalar
collapse the pages state (it must equal the separately pinned Gated DeltaNet
oracle), the pure channel-wise decay when nothing is erased or written (a
closed form), the per-column closed form for keys that are basis vectors
(which isolates the decay of each key channel and the erase gate), and the
exact write-over of a unit key with a full erase gate.  A last group plants
plausible mistakes into a copy of the source and checks each is rejected.
"""
import subprocess

import numpy as np
import pytest

from oracle import oracle as O


def _rand(seed, B, T, H, Dk, Dv):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, Dk))
    k = rng.standard_normal((B, T, H, Dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, Dv))
    la = -np.log1p(np.exp(rng.standard_normal((B, T, H, Dk))))
    b = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H, Dk))))
    w = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H, Dv))))
    S0 = 0.3 * rng.standard_normal((B, H, Dv, Dk))
    return q, k, v, la, b, w, S0, rng


def _rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


def pin_scalar_collapse_is_gated_deltanet(lib=None):
    q, k, v, la, b, w, S0, rng = _rand(1, 2, 23, 2, 5, 4)
    a = la[..., 0]                          # one decay per token and head
    be = b[..., 0]                          # one gate for erase and write
    o1, S1 = O.forward(q, k, v, a, be, S0)
    o2, S2 = O.forward_cw(q, k, v, np.repeat(a[..., None], 5, -1), np.repeat(be[..., None], 5, -1),
                          np.repeat(be[..., None], 4, -1), S0, lib=lib)
    assert _rel(o2, o1) < 1e-13 and _rel(S2, S1) < 1e-13


def pin_decay_only(lib=None):
    """b = w = 0: S_t = S0 Diag(prod_{s<=t} alpha_s), o_t = S_t q_t."""
    q, k, v, la, b, w, S0, rng = _rand(2, 1, 9, 1, 4, 3)
    o, S = O.forward_cw(q, k, v, la, np.zeros_like(b), np.zeros_like(w), S0, lib=lib)
    cum = np.exp(np.cumsum(la[0, :, 0], axis=0))       # [T, Dk]
    for t in range(9):
        St = S0[0, 0] * cum[t][None, :]
        np.testing.assert_allclose(o[0, t, 0], St @ q[0, t, 0], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(S[0, 0], S0[0, 0] * cum[-1][None, :], rtol=1e-13)


def pin_basis_keys(lib=None):
    """k_t = e_{j(t)}: column j(t) becomes alpha_j (1 - b_j) S[:, j] + w o v, every
    other column m is scaled by alpha_m."""
    q, k, v, la, b, w, S0, rng = _rand(3, 1, 12, 1, 4, 3)
    js = rng.integers(0, 4, size=12)
    k = np.zeros_like(k)
    k[0, np.arange(12), 0, js] = 1.0
    o, S = O.forward_cw(q, k, v, la, b, w, S0, lib=lib)
    ref = S0[0, 0].copy()
    for t in range(12):
        j = js[t]
        alpha = np.exp(la[0, t, 0])
        new = ref * alpha[None, :]
        new[:, j] = alpha[j] * (1.0 - b[0, t, 0, j]) * ref[:, j] + w[0, t, 0] * v[0, t, 0]
        ref = new
        np.testing.assert_allclose(o[0, t, 0], ref @ q[0, t, 0], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(S[0, 0], ref, rtol=1e-12, atol=1e-14)


def pin_write_over(lib=None):
    """A full erase gate (b = 1) and a unit key: S_t k_t = w_t o v_t, whatever the decay."""
    q, k, v, la, b, w, S0, rng = _rand(4, 1, 10, 2, 6, 3)
    for t in range(1, 11):
        _, S = O.forward_cw(q[:, :t], k[:, :t], v[:, :t], la[:, :t], np.ones_like(b[:, :t]),
                            w[:, :t], S0, lib=lib)
        for h in range(2):
            np.testing.assert_allclose(S[0, h] @ k[0, t - 1, h], w[0, t - 1, h] * v[0, t - 1, h],
                                       rtol=0, atol=1e-12)


PINS = [pin_scalar_collapse_is_gated_deltanet, pin_decay_only, pin_basis_keys, pin_write_over]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_cw_pin(pin):
    pin()


def test_cw_units_subset_matches_full():
    q, k, v, la, b, w, S0, _ = _rand(5, 2, 30, 3, 4, 5)
    of, Sf = O.forward_cw(q, k, v, la, b, w, S0)
    op, Sp = O.forward_cw(q, k, v, la, b, w, S0, units=[2, 3])
    for u in (2, 3):
        bb, h = divmod(u, 3)
        np.testing.assert_array_equal(op[bb, :, h], of[bb, :, h])
        np.testing.assert_array_equal(Sp[bb, h], Sf[bb, h])


MUTATIONS = {
    "erase_gate_dropped": ("e += row[j] * b[j] * k[j];", "e += row[j] * k[j];"),
    "decay_on_value_axis": ("row[j] = exp(log_alpha[j]) * row[j];",
                            "row[j] = exp(log_alpha[i % Dk]) * row[j];"),
    "erase_reads_undecayed": ("row[j] = exp(log_alpha[j]) * row[j];\n            e += row[j] * b[j] * k[j];",
                              "e += row[j] * b[j] * k[j];\n            row[j] = exp(log_alpha[j]) * row[j];"),
    "write_gate_on_key_axis": ("w[i] * v[i] * k[j]", "w[j % Dv] * v[i] * k[j]"),
    "erase_sign": ("row[j] - e * k[j] + w[i]", "row[j] + e * k[j] + w[i]"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_cw_pins_reject_planted_mistake(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(O.SOURCE).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    mpath = tmp_path / "mutant.c"
    mpath.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-shared", "-fPIC", "-pthread", str(mpath), "-o",
                           str(so), "-lm"])
    lib = O.load_variant(str(so))
    failed = []
    for pin in PINS:
        try:
            pin(lib)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"no pin rejects the planted mistake {name}"
