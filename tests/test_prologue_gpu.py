"""Parity of the input prologue (per-token L2 normalisation of q and k, gate
logits) on every GPU path against the float64 oracle: the raw inputs go to the
library with the flags set; the oracle applies oracle/prologue.py to the same
raw values and runs the recurrence.

Tolerances as for the plain paths: 1e-5 (float32 CUDA-core path and decode),
2e-2 on o and S_T for bf16 inputs.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_130_b200 import inputs as I
from oracle import oracle as O
from oracle import prologue as PR
from parity import head_slices, rel_l2

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5
TOL_BF16 = 2e-2
FLAG_SETS = [(True, True), (True, False), (False, True)]


@pytest.fixture(scope="module")
def gdn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gated_delta_rule_130_b200 import binding
    return binding


def _oracle(inp, l2, gl, units=None):
    q, k, la, be = PR.apply(inp["q"].double().numpy(), inp["k"].double().numpy(),
                            inp["log_alpha"].double().numpy(), inp["beta"].double().numpy(), l2, gl)
    if not l2:
        # without normalisation the raw keys would blow the state up: use the
        # workload's unit keys for that case
        q, k = inp["_q_unit"], inp["_k_unit"]
    return O.forward(q, k, inp["v"], la, be, inp["S0"], units=units)


def _raw(w, l2):
    inp = I.raw_chunk_inputs(w)
    if not l2:
        unit = I.chunk_inputs(w)
        inp["q"], inp["k"] = unit["q"], unit["k"]
        inp["_q_unit"], inp["_k_unit"] = unit["q"], unit["k"]
    return inp


def _run(gdn, inp, chunk, l2, gl):
    d = {n: (t.cuda() if t is not None else None) for n, t in inp.items() if not n.startswith("_")}
    o, S = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], chunk=chunk,
                         l2norm_qk=l2, gate_logits=gl)
    torch.cuda.synchronize()
    gdn.check_device_status()
    return o, S


@pytest.mark.parametrize("l2,gl", FLAG_SETS)
@pytest.mark.parametrize("T", [64, 200])
def test_prologue_tcgen05_path(gdn, l2, gl, T):
    w = I.workload("bf16_T2k", B=2, H=3, T=T, s0_law="normal002", seed=31 + T)
    assert gdn.chunk_fwd_path(w.B, w.T, w.H, w.Dk, w.Dv, 64, torch.bfloat16) == "tcgen05"
    inp = _raw(w, l2)
    o, S = _run(gdn, inp, 64, l2, gl)
    o_ref, S_ref = _oracle(inp, l2, gl)
    eo, es = rel_l2(o.float().cpu(), o_ref), rel_l2(S.cpu(), S_ref)
    assert eo <= TOL_BF16 and es <= TOL_BF16, f"o {eo:.3e} S {es:.3e}"


@pytest.mark.parametrize("l2,gl", FLAG_SETS)
@pytest.mark.parametrize("chunk", [16, 64])
def test_prologue_cuda_core_path_f32(gdn, l2, gl, chunk):
    w = I.workload("tiny_f32", B=2, H=3, T=100, Dk=32, Dv=48, s0_law="normal002", seed=chunk + 5)
    assert gdn.chunk_fwd_path(w.B, w.T, w.H, w.Dk, w.Dv, chunk, torch.float32) == "simt"
    inp = _raw(w, l2)
    o, S = _run(gdn, inp, chunk, l2, gl)
    o_ref, S_ref = _oracle(inp, l2, gl)
    eo, es = rel_l2(o.cpu(), o_ref), rel_l2(S.cpu(), S_ref)
    assert eo <= TOL_F32 and es <= TOL_F32, f"o {eo:.3e} S {es:.3e}"


def test_prologue_cuda_core_path_bf16(gdn):
    # Dk = 64 takes the CUDA-core path in bf16; normalised q, k are stored as bf16
    w = I.workload("bf16_T2k", B=1, H=2, T=150, Dk=64, Dv=64, s0_law="normal002", seed=41)
    assert gdn.chunk_fwd_path(w.B, w.T, w.H, w.Dk, w.Dv, 64, torch.bfloat16) == "simt"
    inp = _raw(w, True)
    o, S = _run(gdn, inp, 64, True, True)
    o_ref, S_ref = _oracle(inp, True, True)
    assert rel_l2(o.float().cpu(), o_ref) <= TOL_BF16 and rel_l2(S.cpu(), S_ref) <= TOL_BF16


def test_prologue_headline_sampled_heads(gdn):
    w = I.workload(I.HEADLINE)
    inp = _raw(w, True)
    o, S = _run(gdn, inp, 64, True, True)
    units = I.sample_units(w, 4)
    o_ref, S_ref = _oracle(inp, True, True, units=units)
    og, sg = head_slices(o, S, units, w.H)
    orf, srf = head_slices(o_ref, S_ref, units, w.H)
    eo, es = rel_l2(og, orf), rel_l2(sg, srf)
    assert eo <= TOL_BF16 and es <= TOL_BF16, f"o {eo:.3e} S {es:.3e}"


def test_prologue_equals_prepared_inputs(gdn):
    """The fused prologue equals the plain path fed with inputs prepared outside
    (float32 CUDA-core path, where both are exact to float32 rounding)."""
    w = I.workload("tiny_f32", B=1, H=2, T=80, Dk=16, Dv=16, seed=9)
    inp = I.raw_chunk_inputs(w)
    d = {n: (t.cuda() if t is not None else None) for n, t in inp.items()}
    o1, S1 = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None, chunk=16,
                           l2norm_qk=True, gate_logits=True)
    q, k, la, be = PR.apply(inp["q"].numpy(), inp["k"].numpy(), inp["log_alpha"].numpy(),
                            inp["beta"].numpy(), True, True)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).float().cuda()
    o2, S2 = gdn.chunk_fwd(t(q), t(k), d["v"], t(la), t(be), None, chunk=16)
    torch.cuda.synchronize()
    assert rel_l2(o1.cpu(), o2.cpu()) <= 1e-5 and rel_l2(S1.cpu(), S2.cpu()) <= 1e-5


@pytest.mark.parametrize("Dk,Dv,dtype", [(128, 128, "f32"), (128, 128, "bf16"), (48, 20, "f32")])
def test_prologue_decode(gdn, Dk, Dv, dtype):
    w = I.workload("decode_b256", B=3, H=4, Dk=Dk, Dv=Dv, dtype=dtype, seed=Dk + Dv + 3)
    S = I.decode_state(w).cuda()
    S0 = S.cpu().unsqueeze(0).reshape(1, w.B * w.H, w.Dv, w.Dk)
    outs, steps = [], []
    for t in range(12):
        x = I.raw_decode_step_inputs(w, t)
        xd = {n: v.cuda() for n, v in x.items()}
        outs.append(gdn.decode_step(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], S,
                                    l2norm_qk=True, gate_logits=True))
        q, k, la, be = PR.apply(x["q"].double().numpy(), x["k"].double().numpy(),
                                x["log_alpha"].double().numpy(), x["beta"].double().numpy(),
                                True, True)
        steps.append((q, k, x["v"].double().numpy(), la, be))
    torch.cuda.synchronize()
    st = lambda i, shape: np.stack([s[i].reshape(shape) for s in steps])[:, None]
    n = w.B * w.H
    o_ref, S_ref = O.decode(st(0, (n, Dk)), st(1, (n, Dk)), st(2, (n, Dv)), st(3, (n,)),
                            st(4, (n,)), S0)
    o = torch.stack(outs).float().cpu().numpy().reshape(len(steps), n, Dv)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    assert rel_l2(o, o_ref[:, 0]) <= tol
    assert rel_l2(S.cpu().numpy().reshape(n, Dv, Dk), S_ref[0]) <= TOL_F32
