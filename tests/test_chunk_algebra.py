"""The chunk algebra the kernels implement, written out in float64 numpy from the
formulas in their source headers, against the oracle's token recurrence: the
gated WY/UT forward, its chunkwise backward, and the channel-wise (Gated
DeltaNet-2) chunk form.  A wrong term in any of those formulas fails here,
independently of the GPU; it is also a second check that the chunked form
computes what the recurrence computes.  CPU only; nothing here is imported by
the library or the oracle.
"""
import numpy as np
import pytest

from oracle import oracle as O


def _pad(x, C):
    pad = (-x.shape[0]) % C
    return np.concatenate([x, np.zeros((pad,) + x.shape[1:])]) if pad else x


def _head(seed, T, Dk, Dv, channel_wise=False):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, Dk))
    k = rng.standard_normal((T, Dk))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, Dv))
    shape = (T, Dk) if channel_wise else (T,)
    la = -np.log1p(np.exp(rng.standard_normal(shape)))
    be = 1.0 / (1.0 + np.exp(-rng.standard_normal(shape)))
    w = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, Dv))))
    S0 = 0.3 * rng.standard_normal((Dv, Dk))
    return q, k, v, la, be, w, S0, rng


def _chunk_pieces(Q, K, V, a, b):
    C = Q.shape[0]
    g = np.cumsum(a)
    gam = np.exp(g)
    Gm = np.exp(g[:, None] - g[None, :]) * np.tri(C)
    A = np.tril(b[:, None] * Gm * (K @ K.T), -1)
    Tm = np.linalg.inv(np.eye(C) + A)
    W = Tm @ ((b * gam)[:, None] * K)
    U = Tm @ (b[:, None] * V)
    P = (Q @ K.T) * Gm
    D = np.exp(g[-1] - g)
    return g, gam, Gm, A, Tm, W, U, P, D


def chunk_forward(q, k, v, la, be, S0, C):
    T = q.shape[0]
    q, k, v, la, be = (_pad(x, C) for x in (q, k, v, la, be))
    S, o = S0.copy(), np.zeros_like(v)
    for c in range(q.shape[0] // C):
        sl = slice(c * C, (c + 1) * C)
        g, gam, Gm, A, Tm, W, U, P, D = _chunk_pieces(q[sl], k[sl], v[sl], la[sl], be[sl])
        Up = U - W @ S.T
        o[sl] = gam[:, None] * (q[sl] @ S.T) + P @ Up
        S = np.exp(g[-1]) * S + Up.T @ (D[:, None] * k[sl])
    return o[:T], S


def chunk_backward(q, k, v, la, be, S0, do, dS_T, C, drop=None):
    """The per-chunk adjoint of the chunk form (the formulas of csrc/chunk_bwd.cu).
    ``drop`` names one term to leave out (the harness's own check)."""
    on = lambda name: 0.0 if drop == name else 1.0
    T = q.shape[0]
    q, k, v, la, be, do = (_pad(x, C) for x in (q, k, v, la, be, do))
    NT = q.shape[0] // C
    S, states, pieces = S0.copy(), [], []
    for c in range(NT):
        sl = slice(c * C, (c + 1) * C)
        pc = _chunk_pieces(q[sl], k[sl], v[sl], la[sl], be[sl])
        g, gam, Gm, A, Tm, W, U, P, D = pc
        states.append(S.copy())
        pieces.append(pc)
        S = np.exp(g[-1]) * S + (U - W @ S.T).T @ (D[:, None] * k[sl])
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dla, dbe = np.zeros_like(la), np.zeros_like(be)
    dS = dS_T.copy()
    for c in reversed(range(NT)):
        sl = slice(c * C, (c + 1) * C)
        Q, K, V, b, dO = q[sl], k[sl], v[sl], be[sl], do[sl]
        g, gam, Gm, A, Tm, W, U, P, D = pieces[c]
        S, dSn = states[c], dS
        Up = U - W @ S.T
        KdS = K @ dSn.T
        dUp = P.T @ dO + D[:, None] * KdS
        Z = Tm.T @ dUp
        dP = (dO @ Up.T) * np.tri(C)
        dQ1 = gam[:, None] * (dO @ S)
        Y = Tm.T @ (-dUp @ S)
        dA = np.tril(-(Y @ W.T + Z @ U.T), -1)
        E = b[:, None] * dA * Gm
        dq[sl] = dQ1 + (dP * Gm) @ K
        dk[sl] = ((dP * Gm).T @ Q + D[:, None] * (Up @ dSn) + (b * gam)[:, None] * Y
                  + E @ K + on("EtK") * (E.T @ K))
        dv[sl] = b[:, None] * Z
        dbe[sl] = gam * np.sum(Y * K, 1) + np.sum(Z * V, 1) + np.sum(dA * Gm * (K @ K.T), 1)
        dG = dP * P
        dAA = dA * A
        h = D * np.sum(Up * KdS, 1)
        dg = (np.sum(dQ1 * Q, 1) + dG.sum(1) - dG.sum(0) + b * gam * np.sum(Y * K, 1)
              + on("dAA") * (dAA.sum(1) - dAA.sum(0)) - on("h") * h)
        dg[-1] += np.exp(g[-1]) * np.sum(dSn * S) + h.sum()
        dla[sl] = np.cumsum(dg[::-1])[::-1]
        dS = (np.exp(g[-1]) * dSn + dO.T @ (gam[:, None] * Q)
              - on("ZK") * (Z.T @ ((b * gam)[:, None] * K)))
    return dq[:T], dk[:T], dv[:T], dla[:T], dbe[:T], dS


def chunk_forward_cw(q, k, v, la, b, w, S0, C):
    """The channel-wise chunk form (the formulas of csrc/chunk_cw.cu)."""
    T = q.shape[0]
    q, k, v, la, b, w = (_pad(x, C) for x in (q, k, v, la, b, w))
    S, o = S0.copy(), np.zeros_like(v)
    for c in range(q.shape[0] // C):
        sl = slice(c * C, (c + 1) * C)
        Q, K, V, L, Bg, Wg = q[sl], k[sl], v[sl], la[sl], b[sl], w[sl]
        Lam = np.cumsum(L, 0)
        E = np.exp(Lam[:, None, :] - Lam[None, :, :])       # [r, i, j]
        A = np.einsum('rj,ij,rij->ri', Bg * K, K, E) * np.tri(C, k=-1)
        P = np.einsum('rj,ij,rij->ri', Q, K, E) * np.tri(C)
        Tm = np.linalg.inv(np.eye(C) + A)
        lam = np.exp(Lam)
        R = Wg * V - (Bg * K * lam) @ S.T
        U = Tm @ R
        o[sl] = (Q * lam) @ S.T + P @ U
        S = S * lam[-1][None, :] + U.T @ (K * np.exp(Lam[-1][None, :] - Lam))
    return o[:T], S


def _rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


def _b(x):   # one head -> [1, T, 1, ...]
    return x[None, :, None]


@pytest.mark.parametrize("C", [16, 64])
def test_chunk_forward_equals_the_recurrence(C):
    q, k, v, la, be, _, S0, _ = _head(1, 150, 8, 6)
    o, S = chunk_forward(q, k, v, la, be, S0, C)
    o_ref, S_ref = O.forward(_b(q), _b(k), _b(v), _b(la), _b(be), S0[None, None])
    assert _rel(o, o_ref[0, :, 0]) < 1e-13 and _rel(S, S_ref[0, 0]) < 1e-13


@pytest.mark.parametrize("C", [16, 64])
def test_chunk_backward_equals_the_exact_gradient(C):
    q, k, v, la, be, _, S0, rng = _head(2, 150, 8, 6)
    do = rng.standard_normal(v.shape)
    dS = rng.standard_normal(S0.shape)
    got = chunk_backward(q, k, v, la, be, S0, do, dS, C)
    ref = O.backward(_b(q), _b(k), _b(v), _b(la), _b(be), S0[None, None], _b(do), dS[None, None])
    refs = [ref[0][0, :, 0], ref[1][0, :, 0], ref[2][0, :, 0], ref[3][0, :, 0], ref[4][0, :, 0],
            ref[5][0, 0]]
    for name, g, r in zip(("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0"), got, refs):
        assert _rel(g, r) < 1e-12, name


@pytest.mark.parametrize("C", [16, 64])
def test_channel_wise_chunk_form_equals_the_recurrence(C):
    q, k, v, la, b, w, S0, _ = _head(3, 150, 8, 6, channel_wise=True)
    o, S = chunk_forward_cw(q, k, v, la, b, w, S0, C)
    o_ref, S_ref = O.forward_cw(_b(q), _b(k), _b(v), _b(la), _b(b), _b(w), S0[None, None])
    assert _rel(o, o_ref[0, :, 0]) < 1e-13 and _rel(S, S_ref[0, 0]) < 1e-13


@pytest.mark.parametrize("term", ["EtK", "dAA", "h", "ZK"])
def test_the_algebra_test_rejects_a_dropped_term(term):
    """The harness itself: leaving out any one term of the adjoint breaks the match."""
    q, k, v, la, be, _, S0, rng = _head(4, 70, 6, 5)
    do, dS = rng.standard_normal(v.shape), rng.standard_normal(S0.shape)
    ref = O.backward(_b(q), _b(k), _b(v), _b(la), _b(be), S0[None, None], _b(do), dS[None, None])
    refs = [ref[0][0, :, 0], ref[1][0, :, 0], ref[2][0, :, 0], ref[3][0, :, 0], ref[4][0, :, 0],
            ref[5][0, 0]]
    good = chunk_backward(q, k, v, la, be, S0, do, dS, 16)
    bad = chunk_backward(q, k, v, la, be, S0, do, dS, 16, drop=term)
    assert max(_rel(g, r) for g, r in zip(good, refs)) < 1e-12
    assert max(_rel(g, r) for g, r in zip(bad, refs)) > 1e-6
