"""The tcgen05 chunkwise forward (bf16, Dk = 128, chunk 64) against the float64
oracle on the method's degenerate gates, ragged lengths, several value slices
and state passing -- every output element compared (GPU only).  Each case runs
on both tcgen05 variants: "fused" (the sequential kernel forms Q K^T and the WY
factors; chosen when its grid of Dv / 64 x H x B CTAs fills most of the GPU,
here by taking enough heads) and "precomputed" (the parallel kernel forms them;
few heads).

The gates are the reductions the pages name: alpha = 1 everywhere is DeltaNet
and beta = 0 everywhere is pure gating (Mamba2's scalar decay), both in "Gated
DeltaNet: Harmonizing Gating and the Delta Rule for Superior Linear RNNs",
section "Problem & Motivation"; beta = 1 with unit keys is the exact write-over
S_t k_t = v_t of its section "Critical Insight"; log alpha = -80 erases the
whole memory at every token.  These reach the parts specific to the tensor-core
kernels: decays formed with ex2.approx in log2 units, the two-factor decay of
the gated Q K^T, the state kept in tensor memory pre-scaled by the chunk's last
decay, and the bf16 copy of the state fed to the next chunk's product.
Tolerance: relative L2 2e-2 on o and S_T (bf16 inputs, float32 accumulation).
"""
import math

import numpy as np
import pytest
import torch

from gated_delta_rule_130_b200 import inputs as I
from parity import oracle_chunk, rel_l2

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


VARIANTS = ["fused", "precomputed"]


def _heads(variant, B=1, Dv=128):
    """Heads that make a call take the given variant: the fused one needs at least
    74 sequential CTAs (Dv / 64 x H x B)."""
    return max(2, math.ceil(74 / (Dv // 64 * B))) if variant == "fused" else 2


def _check(gdn, inp, tol=TOL_BF16, variant=None):
    q = inp["q"]
    B, T, H, Dk = q.shape
    Dv = inp["v"].shape[3]
    assert gdn.chunk_fwd_path(B, T, H, Dk, Dv, 64, torch.bfloat16) == "tcgen05"
    if variant is not None:
        assert gdn.chunk_fwd_variant(B, T, H, Dk, Dv, 64, torch.bfloat16) == variant
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


def _base(T=300, B=1, H=2, Dv=128, s0="normal002", seed=31, gate_law="softplus"):
    w = I.workload("bf16_T2k", B=B, H=H, T=T, Dv=Dv, s0_law=s0, gate_law=gate_law, seed=seed)
    return I.chunk_inputs(w)


GATES = {
    "alpha_one": lambda b: dict(log_alpha=torch.zeros_like(b["log_alpha"])),
    "beta_zero": lambda b: dict(beta=torch.zeros_like(b["beta"])),
    "alpha_to_zero": lambda b: dict(log_alpha=torch.full_like(b["log_alpha"], -80.0)),
    "beta_one": lambda b: dict(beta=torch.ones_like(b["beta"])),
    "alpha_one_beta_one": lambda b: dict(log_alpha=torch.zeros_like(b["log_alpha"]),
                                         beta=torch.ones_like(b["beta"])),
}


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("gate", list(GATES), ids=list(GATES))
def test_degenerate_gates_tc(gdn, gate, variant):
    # slow decay (log alpha = -0.1 softplus): with beta = 0 the state decays by
    # prod(alpha) alone, which must stay inside float32's range over the 300
    # tokens (under the faster law it is about e^-210, and 0 is then the float32
    # answer while the float64 reference is ~1e-92: relative error 1 by rounding)
    base = _base(gate_law="slow_softplus", H=_heads(variant))
    _check(gdn, {**base, **GATES[gate](base)}, variant=variant)


@pytest.mark.parametrize("variant", VARIANTS)
def test_beta_zero_is_pure_decay_tc(gdn, variant):
    """beta = 0: S_T = (prod alpha) S0 and o_t = (prod_{i<=t} alpha_i) S0 q_t, in closed form."""
    base = _base(T=200, gate_law="slow_softplus", H=_heads(variant))
    inp = {**base, "beta": torch.zeros_like(base["beta"])}
    d = _dev(inp)
    o, S = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], chunk=64)
    torch.cuda.synchronize()
    g = torch.cumsum(inp["log_alpha"].double(), dim=1)            # [B,T,H]
    S0 = inp["S0"].double()                                        # [B,H,Dv,Dk]
    S_ref = torch.exp(g[:, -1])[..., None, None] * S0
    o_ref = torch.exp(g)[..., None] * torch.einsum("bhvk,bthk->bthv", S0, inp["q"].double())
    assert rel_l2(S.cpu().numpy(), S_ref.numpy()) <= 1e-5      # float32 state, exact decays
    assert rel_l2(o.float().cpu().numpy(), o_ref.numpy()) <= TOL_BF16


@pytest.mark.parametrize("variant", VARIANTS)
def test_write_over_tc(gdn, variant):
    """beta = 1 at the last token: S_T k_T = v_T (unit keys up to their bf16 rounding)."""
    base = _base(T=130, s0="normal002", H=_heads(variant))
    beta = base["beta"].clone()
    beta[:, -1] = 1.0
    d = _dev({**base, "beta": beta})
    _, S = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], chunk=64)
    torch.cuda.synchronize()
    k_last = base["k"][:, -1].double()                             # [B,H,Dk]
    k_last = k_last / k_last.norm(dim=-1, keepdim=True)
    Sk = torch.einsum("bhvk,bhk->bhv", S.cpu().double(), k_last)
    v_last = base["v"][:, -1].double()
    # the key was normalised before its bf16 rounding: |k| = 1 to about 2^-8
    assert rel_l2(Sk.numpy(), v_last.numpy()) <= TOL_BF16


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("T", [1, 63, 64, 65, 129])
def test_ragged_lengths_tc(gdn, T, variant):
    _check(gdn, _base(T=T, seed=40 + T, H=_heads(variant)), variant=variant)


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("Dv", [64, 192, 256])
def test_value_slices_tc(gdn, Dv, variant):
    _check(gdn, _base(T=200, Dv=Dv, seed=50 + Dv, H=_heads(variant, Dv=Dv)), variant=variant)


@pytest.mark.parametrize("variant", VARIANTS)
def test_zero_initial_state_tc(gdn, variant):
    _check(gdn, _base(T=250, B=2, H=_heads(variant, B=2), s0="zero", seed=61), variant=variant)


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("gate_law", ["softplus", "slow_softplus", "uniform5"])
def test_gate_laws_tc(gdn, gate_law, variant):
    _check(gdn, _base(T=333, B=2, H=_heads(variant, B=2), gate_law=gate_law, seed=62),
           variant=variant)


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("T1", [128, 100])
def test_state_passing_in_place_tc(gdn, T1, variant):
    """Two calls, the second continuing from the first's S_T in place (S0 and S_T
    the same buffer), equal one call and the oracle."""
    inp = _base(T=300, B=2, H=_heads(variant, B=2), seed=70 + T1)
    d = _dev(inp)
    o, S = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], chunk=64)
    sl = lambda x, a, b: x[:, a:b].contiguous()
    state = d["S0"].clone()
    names = ("q", "k", "v", "log_alpha", "beta")
    oa, _ = gdn.chunk_fwd(*(sl(d[n], 0, T1) for n in names), S0=state, S_T=state, chunk=64)
    ob, _ = gdn.chunk_fwd(*(sl(d[n], T1, 300) for n in names), S0=state, S_T=state, chunk=64)
    torch.cuda.synchronize()
    o2 = torch.cat([oa, ob], 1)
    o_ref, S_ref = oracle_chunk(inp)
    assert rel_l2(o2.float().cpu().numpy(), o_ref) <= TOL_BF16
    assert rel_l2(state.cpu().numpy(), S_ref) <= TOL_BF16
    # the split and the single call agree far inside the tolerance
    assert rel_l2(o2.float().cpu().numpy(), o.float().cpu().numpy()) <= 1e-2
    assert rel_l2(state.cpu().numpy(), S.cpu().numpy()) <= 1e-2


@pytest.mark.parametrize("variant", VARIANTS)
def test_prologue_write_over_tc(gdn, variant):
    """Raw (unnormalised) q and k with beta = 1 everywhere, normalised in the
    kernels: the oracle gets the normalised inputs."""
    from oracle import prologue as P
    base = _base(T=200, seed=80, H=_heads(variant))
    gen = torch.Generator().manual_seed(81)
    scale = (0.5 + 3 * torch.rand(base["q"].shape[:3], generator=gen))[..., None]
    q_raw = (base["q"].float() * scale).to(torch.bfloat16)
    k_raw = (base["k"].float() / scale).to(torch.bfloat16)
    beta = torch.ones_like(base["beta"])
    d = _dev({**base, "q": q_raw, "k": k_raw, "beta": beta})
    o, S = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], chunk=64,
                         l2norm_qk=True)
    torch.cuda.synchronize()
    qn = torch.from_numpy(P.l2_normalise(q_raw.double().numpy()))
    kn = torch.from_numpy(P.l2_normalise(k_raw.double().numpy()))
    o_ref, S_ref = oracle_chunk({**base, "q": qn, "k": kn, "beta": beta})
    assert rel_l2(o.float().cpu().numpy(), o_ref) <= TOL_BF16
    assert rel_l2(S.cpu().numpy(), S_ref) <= TOL_BF16
