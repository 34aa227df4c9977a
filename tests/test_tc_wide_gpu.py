"""The tcgen05 chunkwise forward for wide heads (bf16, Dk = 256, chunk 64) against
the float64 oracle, every output element compared (GPU only): the layer shape
of the pages' 1.3B-parameter models has Dk = 256 and Dv = 512 ("Gated DeltaNet:
Harmonizing Gating and the Delta Rule for Superior Linear RNNs", section
"Hardware-Efficient Training": trained in chunks on tensor cores).  Cases: one
and several value slices, ragged lengths, S0 != 0 and state passing in place,
the degenerate gates, packed sequences and the fused prologue.
Tolerance: relative L2 2e-2 on o and S_T (bf16 inputs, float32 accumulation).
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_130_b200 import inputs as I
from parity import oracle_chunk, oracle_varlen, rel_l2

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2


@pytest.fixture(scope="module")
def gdn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gated_delta_rule_130_b200 import binding
    return binding


def _dev(inp):
    return {n: (t.cuda() if t is not None else None) for n, t in inp.items()}


def _base(T=200, B=1, H=2, Dv=128, s0="normal002", seed=131, gate_law="softplus"):
    w = I.workload("wide_dk256_dv512", B=B, H=H, T=T, Dv=Dv, s0_law=s0, gate_law=gate_law,
                   seed=seed)
    return I.chunk_inputs(w)


def _check(gdn, inp, tol=TOL_BF16, **kw):
    B, T, H, Dk = inp["q"].shape
    Dv = inp["v"].shape[3]
    assert Dk == 256
    assert gdn.chunk_fwd_path(B, T, H, Dk, Dv, 64, torch.bfloat16) == "tcgen05"
    d = _dev(inp)
    o, S = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], chunk=64)
    torch.cuda.synchronize()
    gdn.check_device_status()
    o_ref, S_ref = oracle_chunk(inp)
    og, sg = o.float().cpu().numpy(), S.cpu().numpy()
    assert np.isfinite(og).all() and np.isfinite(sg).all()
    eo, es = rel_l2(og, o_ref), rel_l2(sg, S_ref)
    print(f"rel-L2 o={eo:.2e} S_T={es:.2e} shape={tuple(inp['q'].shape)} Dv={inp['v'].shape[3]}")
    assert eo <= tol and es <= tol, f"rel-L2 o={eo:.3e} S_T={es:.3e} (tol {tol})"
    return eo, es


def test_workspace_size_wide(gdn):
    # one [P; T''] tile (128 x 64) and one W tile (64 x 256), bf16, per chunk and head
    B, T, H = 2, 130, 3
    assert gdn.chunk_fwd_path(B, T, H, 256, 512, 64, torch.bfloat16) == "tcgen05"
    assert gdn.chunk_fwd_workspace_size(B, T, H, 256, 512, 64, torch.bfloat16) == \
        B * H * 3 * (128 * 64 + 64 * 256) * 2


@pytest.mark.parametrize("Dv", [64, 128, 512])
def test_value_slices_wide(gdn, Dv):
    _check(gdn, _base(T=200, Dv=Dv, seed=140 + Dv))


@pytest.mark.parametrize("T", [1, 63, 64, 65, 130])
def test_ragged_lengths_wide(gdn, T):
    _check(gdn, _base(T=T, seed=150 + T))


@pytest.mark.parametrize("gate_law", ["softplus", "slow_softplus", "uniform5"])
def test_gate_laws_wide(gdn, gate_law):
    _check(gdn, _base(T=333, B=2, H=2, Dv=192, gate_law=gate_law, s0="zero", seed=160))


GATES = {
    "alpha_one": lambda b: dict(log_alpha=torch.zeros_like(b["log_alpha"])),
    "beta_zero": lambda b: dict(beta=torch.zeros_like(b["beta"])),
    "alpha_to_zero": lambda b: dict(log_alpha=torch.full_like(b["log_alpha"], -80.0)),
    "beta_one": lambda b: dict(beta=torch.ones_like(b["beta"])),
}


@pytest.mark.parametrize("gate", list(GATES), ids=list(GATES))
def test_degenerate_gates_wide(gdn, gate):
    # slow decay: prod(alpha) over the sequence stays inside float32's range
    base = _base(T=260, gate_law="slow_softplus", seed=170)
    _check(gdn, {**base, **GATES[gate](base)})


def test_state_passing_in_place_wide(gdn):
    inp = _base(T=300, B=2, H=2, seed=180)
    d = _dev(inp)
    sl = lambda x, a, b: x[:, a:b].contiguous()
    state = d["S0"].clone()
    names = ("q", "k", "v", "log_alpha", "beta")
    oa, _ = gdn.chunk_fwd(*(sl(d[n], 0, 100) for n in names), S0=state, S_T=state, chunk=64)
    ob, _ = gdn.chunk_fwd(*(sl(d[n], 100, 300) for n in names), S0=state, S_T=state, chunk=64)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_chunk(inp)
    assert rel_l2(torch.cat([oa, ob], 1).float().cpu().numpy(), o_ref) <= TOL_BF16
    assert rel_l2(state.cpu().numpy(), S_ref) <= TOL_BF16


def test_varlen_wide(gdn):
    lengths = [1, 63, 64, 65, 200, 0, 130]
    inp = I.varlen_inputs(lengths, 2, 256, 128, "bf16", s0_law="normal002", seed=190)
    cu = inp["cu_seqlens"]
    assert gdn.chunk_fwd_path(1, max(lengths), 2, 256, 128, 64, torch.bfloat16) == "tcgen05"
    d = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}
    o, S = gdn.chunk_fwd_varlen(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], cu,
                                S0=d["S0"])
    torch.cuda.synchronize()
    gdn.check_device_status()
    o_ref, S_ref = oracle_varlen(inp)
    assert rel_l2(o.float().cpu().numpy(), o_ref) <= TOL_BF16
    assert rel_l2(S.cpu().numpy(), S_ref) <= TOL_BF16


def test_prologue_wide(gdn):
    """Raw q, k and gate logits, normalised and activated inside the kernels."""
    from oracle import prologue as P
    raw = I.raw_chunk_inputs(I.workload("wide_dk256_dv512", B=1, H=2, T=190, Dv=128,
                                        s0_law="normal002"), seed=200)
    d = _dev(raw)
    o, S = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], chunk=64,
                         l2norm_qk=True, gate_logits=True)
    torch.cuda.synchronize()
    gdn.check_device_status()
    ref_in = dict(raw)
    ref_in["q"] = torch.from_numpy(P.l2_normalise(raw["q"].double().numpy()))
    ref_in["k"] = torch.from_numpy(P.l2_normalise(raw["k"].double().numpy()))
    ref_in["log_alpha"] = torch.from_numpy(P.log_alpha_from_logit(raw["log_alpha"].double().numpy()))
    ref_in["beta"] = torch.from_numpy(P.beta_from_logit(raw["beta"].double().numpy()))
    o_ref, S_ref = oracle_chunk(ref_in)
    assert rel_l2(o.float().cpu().numpy(), o_ref) <= TOL_BF16
    assert rel_l2(S.cpu().numpy(), S_ref) <= TOL_BF16
