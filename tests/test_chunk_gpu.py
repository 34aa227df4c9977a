"""Parity of the CUDA chunkwise forward with the float64 oracle (GPU only).

Small cases compare every output element; the full-size workloads compare a
seeded sample of whole heads (the oracle runs those heads token by token).
Tolerances (relative L2 over the compared tensor): 1e-5 for the float32 path,
2e-2 on o and S_T for bf16 inputs with float32 accumulation.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_130_b200 import inputs as I
from parity import head_slices, oracle_chunk, rel_l2

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5
TOL_BF16 = 2e-2


@pytest.fixture(scope="module")
def gdn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gated_delta_rule_130_b200 import binding
    return binding


def _run(gdn, inp, chunk):
    dev = {n: (t.cuda() if t is not None else None) for n, t in inp.items()}
    o, S = gdn.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"], dev["S0"],
                         chunk=chunk)
    torch.cuda.synchronize()
    return o, S


def _full_check(gdn, inp, chunk, tol):
    o, S = _run(gdn, inp, chunk)
    o_ref, S_ref = oracle_chunk(inp)
    eo, es = rel_l2(o.float().cpu(), o_ref), rel_l2(S.cpu(), S_ref)
    assert eo <= tol and es <= tol, f"rel-L2 o={eo:.3e} S_T={es:.3e} (tol {tol})"
    return eo, es


def test_tiny_f32_workload(gdn):
    w = I.workload("tiny_f32")
    _full_check(gdn, I.chunk_inputs(w), w.chunk, TOL_F32)


@pytest.mark.parametrize("T", [1, 17, 50, 64, 100])
@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_ragged_f32(gdn, T, chunk):
    w = I.workload("tiny_f32", T=T, B=2, H=3, Dk=32, Dv=48, s0_law="normal002", seed=T * 7 + chunk)
    _full_check(gdn, I.chunk_inputs(w), chunk, TOL_F32)


@pytest.mark.parametrize("Dk,Dv", [(16, 16), (64, 32), (128, 128), (256, 512), (48, 80),
                                   (8, 24), (200, 40)])
def test_shapes_f32(gdn, Dk, Dv):
    w = I.workload("tiny_f32", T=70, B=1, H=2, Dk=Dk, Dv=Dv, s0_law="normal002", seed=Dk + Dv)
    _full_check(gdn, I.chunk_inputs(w), 32, TOL_F32)


@pytest.mark.parametrize("gate_law", ["softplus", "slow_softplus", "uniform5"])
def test_gate_laws_bf16_small(gdn, gate_law):
    w = I.workload("bf16_T2k", B=2, H=2, T=300, gate_law=gate_law, s0_law="normal002", seed=5)
    _full_check(gdn, I.chunk_inputs(w), 64, TOL_BF16)


def test_tc_path_workspace(gdn):
    # fused variant: one bf16 [T'; T''] tile (128 x 64) per chunk of every (batch,
    # head); precomputed variant: one [P; T''] tile (128 x 64) and one W tile (64 x 128)
    B, T = 2, 130
    for H, variant, per_chunk in ((40, "fused", 128 * 64), (3, "precomputed", 2 * 128 * 64)):
        assert gdn.chunk_fwd_path(B, T, H, 128, 128, 64, torch.bfloat16) == "tcgen05"
        assert gdn.chunk_fwd_variant(B, T, H, 128, 128, 64, torch.bfloat16) == variant
        assert gdn.chunk_fwd_workspace_size(B, T, H, 128, 128, 64, torch.bfloat16) == \
            B * H * 3 * per_chunk * 2


def test_tc_path_ignores_workspace_contents(gdn):
    # the workspace is scratch: garbage (NaN) on entry leaves the results unchanged
    w = I.workload("bf16_T2k", B=1, H=2, T=200, s0_law="normal002", seed=11)
    inp = I.chunk_inputs(w)
    dev = {n: (t.cuda() if t is not None else None) for n, t in inp.items()}
    need = gdn.chunk_fwd_workspace_size(w.B, w.T, w.H, w.Dk, w.Dv, 64, torch.bfloat16)
    outs = []
    for fill in (0.0, float("nan")):
        ws = torch.full((need // 4,), fill, dtype=torch.float32, device="cuda")
        outs.append(gdn.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"],
                                  dev["S0"], chunk=64, workspace=ws))
    torch.cuda.synchronize()
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def test_chunk_size_invariance_f32(gdn):
    w = I.workload("tiny_f32", T=96, B=1, H=2, Dk=32, Dv=32, s0_law="normal002", seed=3)
    inp = I.chunk_inputs(w)
    outs = [_run(gdn, inp, c) for c in (16, 32, 64)]
    for o, S in outs[1:]:
        assert rel_l2(o.cpu(), outs[0][0].cpu()) < TOL_F32
        assert rel_l2(S.cpu(), outs[0][1].cpu()) < TOL_F32


def test_state_passing_split(gdn):
    """Two calls (the second starting from the first's S_T, in place) equal one call."""
    w = I.workload("tiny_f32", T=90, B=2, H=2, Dk=32, Dv=32, s0_law="normal002", seed=4)
    inp = {n: (t.cuda() if t is not None else None) for n, t in I.chunk_inputs(w).items()}
    o, S = gdn.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"],
                         chunk=32)
    T1 = 37
    sl = lambda x, a, b: x[:, a:b].contiguous()
    state = inp["S0"].clone()
    oa, _ = gdn.chunk_fwd(*(sl(inp[n], 0, T1) for n in ("q", "k", "v", "log_alpha", "beta")),
                          S0=state, S_T=state, chunk=32)
    ob, _ = gdn.chunk_fwd(*(sl(inp[n], T1, 90) for n in ("q", "k", "v", "log_alpha", "beta")),
                          S0=state, S_T=state, chunk=32)
    torch.cuda.synchronize()
    assert rel_l2(torch.cat([oa, ob], 1).cpu(), o.cpu()) < TOL_F32
    assert rel_l2(state.cpu(), S.cpu()) < TOL_F32


def test_empty_sequence_returns_initial_state(gdn):
    S0 = torch.randn(2, 3, 16, 16, device="cuda")
    z = lambda *s, dt=torch.float32: torch.empty(*s, dtype=dt, device="cuda")
    o, S = gdn.chunk_fwd(z(2, 0, 3, 16), z(2, 0, 3, 16), z(2, 0, 3, 16), z(2, 0, 3), z(2, 0, 3),
                         S0=S0)
    torch.cuda.synchronize()
    assert o.shape == (2, 0, 3, 16)
    assert torch.equal(S, S0)
    o, S = gdn.chunk_fwd(z(2, 0, 3, 16), z(2, 0, 3, 16), z(2, 0, 3, 16), z(2, 0, 3), z(2, 0, 3))
    torch.cuda.synchronize()
    assert torch.count_nonzero(S) == 0


def test_degenerate_gates(gdn):
    """alpha = 1 everywhere and beta = 0 everywhere (the two reductions the pages
    name) and alpha -> 0 (total erasure at every token)."""
    w = I.workload("tiny_f32", T=80, B=1, H=2, Dk=32, Dv=32, s0_law="normal002", seed=9)
    base = I.chunk_inputs(w)
    for mod in (dict(log_alpha=torch.zeros_like(base["log_alpha"])),
                dict(beta=torch.zeros_like(base["beta"])),
                dict(log_alpha=torch.full_like(base["log_alpha"], -80.0)),
                dict(beta=torch.ones_like(base["beta"]))):
        _full_check(gdn, {**base, **mod}, 32, TOL_F32)


def test_rejects_misaligned_and_overlapping(gdn):
    q = torch.randn(1, 16, 2, 16, device="cuda")
    la = torch.zeros(1, 16, 2, device="cuda")
    with pytest.raises(gdn.GdnError):
        gdn.chunk_fwd(q, q, q, la, la, chunk=48)
    buf = torch.randn(1 + 1 * 16 * 2 * 16, device="cuda")
    q_mis = buf[1:].view(1, 16, 2, 16)  # 4-byte offset: not 16-byte aligned
    with pytest.raises(gdn.GdnError):
        gdn.chunk_fwd(q_mis, q, q, la, la)
    with pytest.raises(gdn.GdnError):
        gdn.chunk_fwd(q, q, q, la, la, out=q)


SAMPLED = [("bf16_T2k", 8), ("long_T32k", 4), ("wide_dk256_dv512", 3), ("headline_T4k", 8)]


@pytest.mark.parametrize("name,n_units", SAMPLED, ids=[s[0] for s in SAMPLED])
def test_full_size_workloads_sampled_heads(gdn, name, n_units):
    w = I.workload(name)
    inp = I.chunk_inputs(w)
    o, S = _run(gdn, inp, w.chunk)
    units = I.sample_units(w, n_units)
    o_ref, S_ref = oracle_chunk(inp, units=units)
    og, sg = head_slices(o, S, units, w.H)
    orf, srf = head_slices(o_ref, S_ref, units, w.H)
    eo, es = rel_l2(og, orf), rel_l2(sg, srf)
    print(f"{name}: path={gdn.chunk_fwd_path(w.B, w.T, w.H, w.Dk, w.Dv, w.chunk)} "
          f"rel-L2 o={eo:.3e} S_T={es:.3e} over heads {units}")
    assert np.isfinite(og).all() and np.isfinite(sg).all()
    assert eo <= TOL_BF16 and es <= TOL_BF16, f"rel-L2 o={eo:.3e} S_T={es:.3e}"
