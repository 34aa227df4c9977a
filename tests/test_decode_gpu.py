"""Parity of the CUDA decode step with the oracle's token-by-token recurrence."""
import numpy as np
import pytest
import torch

from gated_delta_rule_130_b200 import inputs as I
from oracle import oracle as O
from parity import rel_l2

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5
TOL_BF16 = 2e-2


@pytest.fixture(scope="module")
def gdn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gated_delta_rule_130_b200 import binding
    return binding


def _steps(gdn, w, n_steps, units=None):
    """Run n_steps decode steps on the GPU and the same steps in the oracle.

    With ``units`` only those heads are kept (GPU outputs gathered per step, the
    oracle run on just those heads); outputs are [steps, n, Dv] / [n, Dv, Dk].
    """
    units = list(range(w.B * w.H)) if units is None else units
    bi = torch.tensor([u // w.H for u in units])
    hi = torch.tensor([u % w.H for u in units])
    S = I.decode_state(w).cuda()
    S0 = S[bi.cuda(), hi.cuda()].cpu().unsqueeze(0)  # [1, n, Dv, Dk]
    os_, sub = [], {n: [] for n in ("q", "k", "v", "log_alpha", "beta")}
    for t in range(n_steps):
        x = I.decode_step_inputs(w, t)
        for n in sub:
            sub[n].append(x[n][bi, hi].unsqueeze(0))
        xd = {n: v.cuda() for n, v in x.items()}
        o = gdn.decode_step(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], S)
        os_.append(o[bi.cuda(), hi.cuda()])
    torch.cuda.synchronize()
    st = lambda n: torch.stack(sub[n])  # [steps, 1, n, ...]
    o_ref, S_ref = O.decode(st("q"), st("k"), st("v"), st("log_alpha"), st("beta"), S0)
    o = torch.stack(os_).float().cpu().numpy()
    return o, S[bi.cuda(), hi.cuda()].cpu().numpy(), o_ref[:, 0], S_ref[0]


@pytest.mark.parametrize("Dk,Dv,dtype", [(16, 16, "f32"), (32, 64, "f32"), (64, 32, "f32"),
                                         (128, 128, "f32"), (256, 512, "f32"), (48, 20, "f32"),
                                         (128, 128, "bf16"), (24, 8, "bf16")])
def test_decode_small(gdn, Dk, Dv, dtype):
    w = I.workload("decode_b256", B=3, H=5, Dk=Dk, Dv=Dv, dtype=dtype, seed=Dk * 3 + Dv)
    o, S, o_ref, S_ref = _steps(gdn, w, 20)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    assert rel_l2(o, o_ref) <= tol and rel_l2(S, S_ref) <= TOL_F32


def test_decode_workload_1000_steps(gdn):
    """batch 256, H 16, d 128: 1000 successive steps from S0 ~ N(0, 0.02), every
    step's output and the final state checked on a seeded sample of heads."""
    w = I.workload("decode_b256")
    units = I.sample_units(w, 16)
    o, S, o_ref, S_ref = _steps(gdn, w, w.steps, units=units)
    eo, es = rel_l2(o, o_ref), rel_l2(S, S_ref)
    print(f"decode 1000 steps: rel-L2 o={eo:.3e} S={es:.3e}")
    assert eo <= TOL_BF16 and es <= TOL_BF16
