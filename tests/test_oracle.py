"""Pins of the float64 oracle against what the pages and the mathematics fix.

Every check here is independent of the oracle's own code path: a hand-expanded
worked example, the two reductions the pages name (gating alone, the delta rule
alone), the write-over property of the online-regression view, a closed form for
orthonormal keys, and an explicit transition-matrix brute force.  The last group
plants plausible mistakes into a copy of the oracle's source and checks that at
least one pin rejects each of them.
"""
import json
import os
import subprocess

import numpy as np
import pytest

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "gdn_t2_d2.json")


def _rand(rng, B, T, H, Dk, Dv, unit_keys=True):
    q = rng.standard_normal((B, T, H, Dk))
    k = rng.standard_normal((B, T, H, Dk))
    if unit_keys:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, Dv))
    la = -np.log1p(np.exp(rng.standard_normal((B, T, H))))
    be = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    return q, k, v, la, be


def _rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


# ---------------------------------------------------------------- pins ----
# Each pin takes an oracle library handle (None = the real oracle) so the
# planted-mistake checks below can rerun the same pins on a mutated build.

def pin_golden(lib=None):
    """Hand-expanded T=2, Dk=Dv=2 case (tests/golden/gdn_t2_d2.json)."""
    g = json.load(open(GOLDEN))
    inp = g["inputs"]
    k = np.array(inp["k"], float).reshape(1, 2, 1, 2)
    v = np.array(inp["v"], float).reshape(1, 2, 1, 2)
    q = np.array(inp["q"], float).reshape(1, 2, 1, 2)
    la = np.log(np.array(inp["alpha"], float)).reshape(1, 2, 1)
    be = np.array(inp["beta"], float).reshape(1, 2, 1)
    for case in g["cases"]:
        S0 = np.array(case["S0"], float).reshape(1, 1, 2, 2)
        o1, S1 = O.forward(q[:, :1], k[:, :1], v[:, :1], la[:, :1], be[:, :1], S0, lib=lib)
        o, S2 = O.forward(q, k, v, la, be, S0, lib=lib)
        np.testing.assert_allclose(S1[0, 0], case["S1"], rtol=0, atol=1e-14)
        np.testing.assert_allclose(o1[0, 0, 0], case["o1"], rtol=0, atol=1e-14)
        np.testing.assert_allclose(o[0, 0, 0], case["o1"], rtol=0, atol=1e-14)
        np.testing.assert_allclose(S2[0, 0], case["S2"], rtol=0, atol=1e-14)
        np.testing.assert_allclose(o[0, 1, 0], case["o2"], rtol=0, atol=1e-14)
        # write-over of the second token (beta = 1, unit key): S_2 k_2 = v_2
        np.testing.assert_allclose(S2[0, 0] @ k[0, 1, 0], v[0, 1, 0], rtol=0, atol=1e-14)


def pin_deltanet(lib=None):
    """alpha == 1 reduces the rule to DeltaNet, S <- S + beta (v - S k) k^T
    (gating removed; 'Gated DeltaNet: Harmonizing Gating and the Delta Rule for
    Superior Linear RNNs', section 'Problem & Motivation', item 2)."""
    rng = np.random.default_rng(11)
    B, T, H, Dk, Dv = 2, 9, 3, 5, 4
    q, k, v, _, be = _rand(rng, B, T, H, Dk, Dv)
    la = np.zeros((B, T, H))
    S0 = rng.standard_normal((B, H, Dv, Dk))
    o, ST = O.forward(q, k, v, la, be, S0, lib=lib)
    for b in range(B):
        for h in range(H):
            S = S0[b, h].copy()
            for t in range(T):
                kt, vt = k[b, t, h], v[b, t, h]
                S = S + be[b, t, h] * np.outer(vt - S @ kt, kt)
                assert _rel(o[b, t, h], S @ q[b, t, h]) < 1e-12
            assert _rel(ST[b, h], S) < 1e-12


def pin_gating_only(lib=None):
    """beta == 0 leaves only the scalar decay (Mamba2-style gating,
    'Gated DeltaNet: Harmonizing Gating ...', section 'Problem & Motivation',
    item 1): S_t = (prod_{i<=t} alpha_i) S_0 in closed form."""
    rng = np.random.default_rng(12)
    B, T, H, Dk, Dv = 2, 13, 2, 6, 3
    q, k, v, la, _ = _rand(rng, B, T, H, Dk, Dv)
    be = np.zeros((B, T, H))
    S0 = rng.standard_normal((B, H, Dv, Dk))
    o, ST = O.forward(q, k, v, la, be, S0, lib=lib)
    g = np.cumsum(la, axis=1)  # log prod alpha
    for b in range(B):
        for h in range(H):
            for t in range(T):
                ref = np.exp(g[b, t, h]) * (S0[b, h] @ q[b, t, h])
                assert _rel(o[b, t, h], ref) < 1e-12
            assert _rel(ST[b, h], np.exp(g[b, -1, h]) * S0[b, h]) < 1e-12


def pin_write_over(lib=None):
    """Online-regression view ('Critical Insight': S_t k_t ~ v_t), exact when
    beta_t = 1 and |k_t| = 1, for any gate and any previous state.  Reading the
    state with q_t = k_t therefore returns v_t."""
    rng = np.random.default_rng(13)
    B, T, H, Dk, Dv = 1, 17, 2, 8, 5
    _, k, v, la, _ = _rand(rng, B, T, H, Dk, Dv)
    be = np.ones((B, T, H))
    S0 = rng.standard_normal((B, H, Dv, Dk))
    o, ST = O.forward(k, k, v, la, be, S0, lib=lib)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-12)
    np.testing.assert_allclose(np.einsum("bhvk,bhk->bhv", ST, k[:, -1]), v[:, -1], atol=1e-12)


def pin_orthonormal(lib=None):
    """alpha = beta = 1, S0 = 0, orthonormal keys: the delta rule never collides,
    so S_T = sum_i v_i k_i^T and querying with k_j returns v_j."""
    rng = np.random.default_rng(14)
    Dk, Dv, T = 8, 3, 6
    Qm, _ = np.linalg.qr(rng.standard_normal((Dk, Dk)))
    k = Qm[:T].reshape(1, T, 1, Dk)              # rows are orthonormal
    v = rng.standard_normal((1, T, 1, Dv))
    perm = [0, 0, 1, 3, 2, 5]                    # q_t = k_perm[t], perm[t] <= t
    q = k[:, perm]
    la = np.zeros((1, T, 1))
    be = np.ones((1, T, 1))
    o, ST = O.forward(q, k, v, la, be, None, lib=lib)
    np.testing.assert_allclose(ST[0, 0], np.einsum("tv,tk->vk", v[0, :, 0], k[0, :, 0]),
                               atol=1e-13)
    np.testing.assert_allclose(o[0, :, 0], v[0, perm, 0], atol=1e-13)


def pin_transition_matrices(lib=None):
    """Brute force with explicit transition matrices M_t = alpha_t (I - beta_t k_t k_t^T):
    S_T = S_0 M_1 ... M_T + sum_t beta_t v_t k_t^T M_{t+1} ... M_T, and
    o_t = S_t q_t with S_t from the same unrolled sum (no recurrence)."""
    rng = np.random.default_rng(15)
    B, T, H, Dk, Dv = 1, 7, 2, 4, 3
    q, k, v, la, be = _rand(rng, B, T, H, Dk, Dv, unit_keys=False)
    S0 = rng.standard_normal((B, H, Dv, Dk))
    o, ST = O.forward(q, k, v, la, be, S0, lib=lib)
    I = np.eye(Dk)
    for h in range(H):
        M = [np.exp(la[0, t, h]) * (I - be[0, t, h] * np.outer(k[0, t, h], k[0, t, h]))
             for t in range(T)]

        def prod(a, b_):  # M_a ... M_{b_-1}
            P = I.copy()
            for s in range(a, b_):
                P = P @ M[s]
            return P

        for t in range(T):
            St = S0[0, h] @ prod(0, t + 1)
            for i in range(t + 1):
                St = St + be[0, i, h] * np.outer(v[0, i, h], k[0, i, h]) @ prod(i + 1, t + 1)
            assert _rel(o[0, t, h], St @ q[0, t, h]) < 1e-12
            if t == T - 1:
                assert _rel(ST[0, h], St) < 1e-12


def pin_split(lib=None):
    """State passing: one pass over T tokens equals T1 tokens then T - T1 tokens
    started from the state the first call returned."""
    rng = np.random.default_rng(16)
    B, T, H, Dk, Dv = 2, 20, 2, 6, 5
    q, k, v, la, be = _rand(rng, B, T, H, Dk, Dv)
    S0 = rng.standard_normal((B, H, Dv, Dk))
    o, ST = O.forward(q, k, v, la, be, S0, lib=lib)
    T1 = 7
    oa, Sa = O.forward(q[:, :T1], k[:, :T1], v[:, :T1], la[:, :T1], be[:, :T1], S0, lib=lib)
    ob, Sb = O.forward(q[:, T1:], k[:, T1:], v[:, T1:], la[:, T1:], be[:, T1:], Sa, lib=lib)
    np.testing.assert_allclose(np.concatenate([oa, ob], axis=1), o, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(Sb, ST, rtol=1e-13, atol=1e-13)


PINS = [pin_golden, pin_deltanet, pin_gating_only, pin_write_over, pin_orthonormal,
        pin_transition_matrices, pin_split]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    pin()


def test_units_subset_matches_full():
    rng = np.random.default_rng(17)
    B, T, H, Dk, Dv = 3, 11, 4, 5, 6
    q, k, v, la, be = _rand(rng, B, T, H, Dk, Dv)
    S0 = rng.standard_normal((B, H, Dv, Dk))
    o, ST = O.forward(q, k, v, la, be, S0)
    units = [0, 5, 11]
    os_, Ss = O.forward(q, k, v, la, be, S0, units=units)
    for u in units:
        b, h = divmod(u, H)
        np.testing.assert_array_equal(os_[b, :, h], o[b, :, h])
        np.testing.assert_array_equal(Ss[b, h], ST[b, h])
    assert np.isnan(os_[0, :, 1]).all()


def test_decode_matches_forward():
    """The decode entry is the same rule with a [steps,B,H,*] layout."""
    rng = np.random.default_rng(18)
    B, T, H, Dk, Dv = 2, 10, 3, 4, 7
    q, k, v, la, be = _rand(rng, B, T, H, Dk, Dv)
    S0 = rng.standard_normal((B, H, Dv, Dk))
    o, ST = O.forward(q, k, v, la, be, S0)
    sw = lambda x: np.ascontiguousarray(np.swapaxes(x, 0, 1))
    od, Sd = O.decode(sw(q), sw(k), sw(v), sw(la), sw(be), S0)
    np.testing.assert_array_equal(sw(od), o)
    np.testing.assert_array_equal(Sd, ST)


def test_thread_count_does_not_change_result():
    rng = np.random.default_rng(19)
    q, k, v, la, be = _rand(rng, 2, 9, 5, 4, 3)
    a = O.forward(q, k, v, la, be, nthreads=1)
    b = O.forward(q, k, v, la, be, nthreads=7)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_bad_arguments_rejected():
    with pytest.raises(ValueError):
        O.forward(np.zeros((1, 2, 1, 3)), np.zeros((1, 2, 1, 3)), np.zeros((1, 2, 1, 2)),
                  np.zeros((1, 2, 1)), np.zeros((1, 3, 1)))
    with pytest.raises(ValueError):
        O.forward(np.zeros((1, 2, 1, 3)), np.zeros((1, 2, 1, 3)), np.zeros((1, 2, 1, 2)),
                  np.zeros((1, 2, 1)), np.zeros((1, 2, 1)), units=[5])


# ------------------------------------------------- planted mistakes -------
MUTATIONS = {
    "gate_dropped_on_state": ("alpha * row[j] - alpha", "row[j] - alpha"),
    "erase_sign_flipped": ("- alpha * beta * sk * k[j]", "+ alpha * beta * sk * k[j]"),
    "erase_without_gate": ("- alpha * beta * sk * k[j]", "- beta * sk * k[j]"),
    "erase_reads_query": ("sk += row[m] * k[m]", "sk += row[m] * q[m]"),
    "write_transposed": ("beta * v[i] * k[j]", "beta * v[j % Dv] * k[i % Dk]"),
    "readout_with_key": ("oi += row[j] * q[j]", "oi += row[j] * k[j]"),
    "gate_linearised": ("exp(log_alpha)", "(1.0 + log_alpha)"),
    "beta_squared": ("beta * v[i] * k[j]", "beta * beta * v[i] * k[j]"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_reject_planted_mistake(name, tmp_path):
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
