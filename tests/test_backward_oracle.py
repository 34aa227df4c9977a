"""Pins of the oracle's backward (oracle.backward, the exact gradient of the token
recurrence taken token by token in reverse).

Each pin compares with something computed another way: central finite
differences of the (separately pinned) forward oracle, reverse-mode automatic
differentiation of an independently written float64 PyTorch loop of the same
recurrence, and a closed form for the gating-only case (beta = 0).  The last
group plants plausible mistakes into a copy of the oracle's source and checks
that at least one pin rejects each of them.
"""
import subprocess

import numpy as np
import pytest
import torch

from oracle import oracle as O


def _case(seed, B, T, H, Dk, Dv, beta_zero=False):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, Dk))
    k = rng.standard_normal((B, T, H, Dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, Dv))
    la = -np.log1p(np.exp(rng.standard_normal((B, T, H))))
    be = np.zeros((B, T, H)) if beta_zero else 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    S0 = 0.5 * rng.standard_normal((B, H, Dv, Dk))
    do = rng.standard_normal((B, T, H, Dv))
    dS = rng.standard_normal((B, H, Dv, Dk))
    return [q, k, v, la, be, S0], do, dS


def _loss(lib, args, do, dS):
    o, S = O.forward(*args, lib=lib)
    return float(np.sum(o * do) + np.sum(S * dS))


def _rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


# ---------------------------------------------------------------- pins ----

def pin_finite_differences(lib=None):
    """Every gradient against central differences of the forward, on a sequence
    that crosses the backward's checkpoint blocks (T = 70)."""
    args, do, dS = _case(1, 1, 70, 2, 3, 2)
    grads = O.backward(*args, do, dS, lib=lib)
    eps = 1e-6
    for ai, (a, g) in enumerate(zip(args, grads)):
        num = np.zeros_like(a)
        for idx in np.ndindex(a.shape):
            ap = [x.copy() for x in args]
            am = [x.copy() for x in args]
            ap[ai][idx] += eps
            am[ai][idx] -= eps
            num[idx] = (_loss(lib, ap, do, dS) - _loss(lib, am, do, dS)) / (2 * eps)
        assert _rel(g, num) < 1e-7, f"input {ai}: rel {_rel(g, num):.2e}"


def _torch_forward(q, k, v, la, be, S0):
    """The recurrence written independently, one token at a time, in torch."""
    B, T, H, Dk = q.shape
    outs, finals = [], []
    for b in range(B):
        ob, sb = [], []
        for h in range(H):
            S = S0[b, h]
            ot = []
            for t in range(T):
                kt, vt = k[b, t, h], v[b, t, h]
                a = torch.exp(la[b, t, h])
                E = torch.eye(Dk, dtype=q.dtype) - be[b, t, h] * torch.outer(kt, kt)
                S = S @ (a * E) + be[b, t, h] * torch.outer(vt, kt)
                ot.append(S @ q[b, t, h])
            ob.append(torch.stack(ot))
            sb.append(S)
        outs.append(torch.stack(ob, dim=1))
        finals.append(torch.stack(sb))
    return torch.stack(outs), torch.stack(finals)


def pin_autograd(lib=None):
    args, do, dS = _case(2, 2, 19, 2, 4, 3)
    ts = [torch.tensor(a, requires_grad=True) for a in args]
    o, S = _torch_forward(*ts)
    (torch.sum(o * torch.tensor(do)) + torch.sum(S * torch.tensor(dS))).backward()
    grads = O.backward(*args, do, dS, lib=lib)
    for i, (t, g) in enumerate(zip(ts, grads)):
        assert _rel(g, t.grad.numpy()) < 1e-12, f"input {i}: rel {_rel(g, t.grad.numpy()):.2e}"


def pin_gating_only(lib=None):
    """beta = 0: S_t = c_t S0 with c_t = exp(sum_{s<=t} log alpha_s), o_t = c_t S0 q_t.
    Then dS0 = sum_t c_t do_t q_t^T + c_T dS_T, dq_t = c_t S0^T do_t, dk = dv = 0,
    dlog_alpha_s = sum_{t>=s} c_t do_t.(S0 q_t) + c_T <dS_T, S0>."""
    args, do, dS = _case(3, 1, 9, 1, 3, 2, beta_zero=True)
    q, k, v, la, be, S0 = args
    c = np.exp(np.cumsum(la[0, :, 0]))
    s0 = S0[0, 0]
    dq, dk, dv, dla, dbe, dS0 = O.backward(*args, do, dS, lib=lib)
    ref_dS0 = sum(c[t] * np.outer(do[0, t, 0], q[0, t, 0]) for t in range(9)) + c[-1] * dS[0, 0]
    np.testing.assert_allclose(dS0[0, 0], ref_dS0, rtol=1e-13, atol=1e-14)
    for t in range(9):
        np.testing.assert_allclose(dq[0, t, 0], c[t] * s0.T @ do[0, t, 0], rtol=1e-13, atol=1e-14)
    assert np.all(dk == 0) and np.all(dv == 0)
    per_t = np.array([c[t] * do[0, t, 0] @ (s0 @ q[0, t, 0]) for t in range(9)])
    ref_dla = np.cumsum(per_t[::-1])[::-1] + c[-1] * np.sum(dS[0, 0] * s0)
    np.testing.assert_allclose(dla[0, :, 0], ref_dla, rtol=1e-12, atol=1e-14)


PINS = [pin_finite_differences, pin_autograd, pin_gating_only]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_backward_pin(pin):
    pin()


def test_backward_units_subset_matches_full():
    args, do, dS = _case(4, 2, 80, 3, 5, 4)
    full = O.backward(*args, do, dS)
    units = [1, 4]
    part = O.backward(*args, do, dS, units=units)
    for f, p in zip(full, part):
        for u in units:
            b, h = divmod(u, 3)
            if f.ndim == 4 and f.shape[:2] == (2, 3):      # dS0 [B,H,Dv,Dk]
                np.testing.assert_array_equal(p[b, h], f[b, h])
            else:                                          # [B,T,H,...]
                np.testing.assert_array_equal(p[b, :, h], f[b, :, h])


def test_backward_without_final_state_gradient():
    args, do, _ = _case(5, 1, 12, 2, 3, 3)
    a = O.backward(*args, do, None)
    b = O.backward(*args, do, np.zeros((1, 2, 3, 3)))
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


# ------------------------------------------------- planted mistakes -------
MUTATIONS = {
    "dv_without_beta": ("dv[i] = beta * c;", "dv[i] = c;"),
    "dk_cross_sign": ("beta * gv - alpha * beta * (gs + sg)", "beta * gv + alpha * beta * (gs + sg)"),
    "dk_one_sided": ("(gs + sg)", "(2.0 * sg)"),
    "dlog_alpha_is_dalpha": ("j->dla[GG(t)] = alpha * dalpha;", "j->dla[GG(t)] = dalpha;"),
    "state_grad_ungated": ("G[i * Dk + m] = alpha * (G[i * Dk + m] - beta * Gk[i] * k[m]);",
                           "G[i * Dk + m] = G[i * Dk + m] - beta * Gk[i] * k[m];"),
    "dq_from_previous_state": ("a += Sc[i * Dk + m] * dout[i];", "a += Sp[i * Dk + m] * dout[i];"),
    "dbeta_erase_ungated": ("(v[i] - alpha * a) * c", "(v[i] - a) * c"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_backward_pins_reject_planted_mistake(name, tmp_path):
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
