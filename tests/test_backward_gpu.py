"""Parity of the chunkwise backward (gdn_chunk_bwd) with the oracle's exact
gradient (oracle.backward), element by element over each gradient tensor
(GPU only).

Tolerances: 1e-5 relative L2 for float32 inputs, 2e-2 for bf16 inputs (the
gradients are rounded to bf16 once; the arithmetic is float32).
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_130_b200 import inputs as I
from oracle import oracle as O
from parity import rel_l2

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5
TOL_BF16 = 2e-2
NAMES = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0")


@pytest.fixture(scope="module")
def gdn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gated_delta_rule_130_b200 import binding
    return binding


def _grads_in(w, seed):
    """Forward inputs of workload w plus seeded upstream gradients d_o, dS_T."""
    inp = I.chunk_inputs(w, seed=seed)
    gen = torch.Generator().manual_seed(seed + 99)
    do = torch.randn((w.B, w.T, w.H, w.Dv), generator=gen).to(w.torch_dtype)
    dS = torch.randn((w.B, w.H, w.Dv, w.Dk), generator=gen)
    return inp, do, dS


def _run(gdn, inp, do, dS, chunk):
    d = {n: (t.cuda() if t is not None else None) for n, t in inp.items()}
    out = gdn.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], do.cuda(),
                        dS.cuda() if dS is not None else None, chunk=chunk)
    torch.cuda.synchronize()
    return [x.float().cpu().numpy() if x is not None else None for x in out]


def _check(got, ref, tol, units=None, H=None):
    for name, g, r in zip(NAMES, got, ref):
        if units is not None:
            sel = [divmod(u, H) for u in units]
            if name == "dS0":
                g, r = np.stack([g[b, h] for b, h in sel]), np.stack([r[b, h] for b, h in sel])
            else:
                g, r = np.stack([g[b, :, h] for b, h in sel]), np.stack([r[b, :, h] for b, h in sel])
        e = rel_l2(g, r)
        assert e <= tol, f"{name}: rel-L2 {e:.3e}"


@pytest.mark.parametrize("chunk", [16, 32, 64])
@pytest.mark.parametrize("T", [1, 64, 100])
def test_backward_f32(gdn, chunk, T):
    w = I.workload("tiny_f32", B=2, H=3, T=T, Dk=32, Dv=48, s0_law="normal002", seed=chunk + T)
    inp, do, dS = _grads_in(w, w.seed)
    got = _run(gdn, inp, do, dS, chunk)
    ref = O.backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"], do,
                     dS)
    _check(got, ref, TOL_F32)


def test_backward_f32_d128_without_state_gradients(gdn):
    w = I.workload("tiny_f32", B=1, H=2, T=150, Dk=128, Dv=128, seed=71)
    inp, do, _ = _grads_in(w, w.seed)
    got = _run(gdn, inp, do, None, 64)
    ref = O.backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], None, do, None)
    _check(got, ref, TOL_F32)


def test_backward_bf16_d128(gdn):
    w = I.workload("bf16_T2k", B=2, H=2, T=300, s0_law="normal002", seed=73)
    inp, do, dS = _grads_in(w, w.seed)
    got = _run(gdn, inp, do, dS, 64)
    ref = O.backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"], do,
                     dS)
    _check(got, ref, TOL_BF16)


def test_backward_headline_sampled_heads(gdn):
    w = I.workload(I.HEADLINE)
    inp, do, dS = _grads_in(w, w.seed)
    got = _run(gdn, inp, do, dS, 64)
    units = I.sample_units(w, 3)
    ref = O.backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"], do,
                     dS, units=units)
    _check(got, ref, TOL_BF16, units=units, H=w.H)


def test_backward_chunk_size_invariance(gdn):
    w = I.workload("tiny_f32", B=1, H=2, T=96, Dk=16, Dv=16, s0_law="normal002", seed=5)
    inp, do, dS = _grads_in(w, w.seed)
    a = _run(gdn, inp, do, dS, 16)
    b = _run(gdn, inp, do, dS, 64)
    for x, y in zip(a, b):
        assert rel_l2(x, y) <= 1e-5


def test_backward_no_tokens_passes_the_state_gradient(gdn):
    dS = torch.randn(2, 3, 8, 16, device="cuda")
    z = lambda *s: torch.zeros(*s, device="cuda")
    out = gdn.chunk_bwd(z(2, 0, 3, 16), z(2, 0, 3, 16), z(2, 0, 3, 8), z(2, 0, 3), z(2, 0, 3),
                        None, z(2, 0, 3, 8), dS, chunk=16)
    torch.cuda.synchronize()
    assert torch.equal(out[5], dS)
