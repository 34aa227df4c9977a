"""The channel-wise-gate forward (Gated DeltaNet-2 reading) on the tensor cores
-- bf16, Dk = 128, chunk 64 -- against the float64 oracle of the token
recurrence (oracle.forward_cw), every output element compared (GPU only).

"Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention" (abstract)
names a decay per key channel, an erase gate on the key side, a write gate on
the value side and a chunkwise WY algorithm with the channel-wise decay
absorbed into asymmetric erase factors; the cases cover the decay laws (strong
per-channel decay included), ragged lengths, several value slices, in-place
state passing, the degenerate gates, and the collapse to the scalar rule.
Tolerance: relative L2 2e-2 on o and S_T (bf16 inputs, float32 accumulation).
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_130_b200 import inputs as I
from oracle import oracle as O
from parity import rel_l2

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2


@pytest.fixture(scope="module")
def gdn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gated_delta_rule_130_b200 import binding
    return binding


def _inputs(T=200, B=1, H=2, Dv=128, law="softplus", s0="normal002", seed=300):
    return I.cw_inputs(I.workload("bf16_T2k", B=B, H=H, T=T, Dv=Dv, gate_law=law, s0_law=s0,
                                  seed=seed))


def _oracle(inp):
    return O.forward_cw(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"],
                        inp["S0"])


def _run(gdn, inp, S0=None, S_T=None):
    d = {n: (t.cuda() if t is not None else None) for n, t in inp.items()}
    B, T, H, Dk = d["q"].shape
    Dv = d["v"].shape[3]
    assert gdn.chunk_fwd_cw_path(B, T, H, Dk, Dv, 64, torch.bfloat16) == "tcgen05"
    o, S = gdn.chunk_fwd_cw(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"],
                            d["S0"] if S0 is None else S0, chunk=64, S_T=S_T)
    torch.cuda.synchronize()
    gdn.check_device_status()
    return o, S


def _check(gdn, inp, tol=TOL_BF16):
    o, S = _run(gdn, inp)
    o_ref, S_ref = _oracle(inp)
    og, sg = o.float().cpu().numpy(), S.cpu().numpy()
    assert np.isfinite(og).all() and np.isfinite(sg).all()
    eo, es = rel_l2(og, o_ref), rel_l2(sg, S_ref)
    print(f"rel-L2 o={eo:.2e} S_T={es:.2e} shape={tuple(inp['q'].shape)} Dv={inp['v'].shape[3]}")
    assert eo <= tol and es <= tol, f"rel-L2 o={eo:.3e} S_T={es:.3e} (tol {tol})"


@pytest.mark.parametrize("law", ["softplus", "slow_softplus", "uniform5"])
def test_cw_tc_decay_laws(gdn, law):
    # uniform5: log alpha ~ U[-5, 0] per channel, so the decays inside a chunk
    # span hundreds of e-folds (the factorisation through reference rows must
    # never overflow)
    _check(gdn, _inputs(T=260, B=2, law=law, seed=301))


@pytest.mark.parametrize("T", [1, 63, 64, 65, 130])
def test_cw_tc_ragged(gdn, T):
    _check(gdn, _inputs(T=T, seed=310 + T))


@pytest.mark.parametrize("Dv", [64, 192])
def test_cw_tc_value_slices(gdn, Dv):
    _check(gdn, _inputs(T=150, Dv=Dv, seed=320 + Dv))


def test_cw_tc_zero_state_and_heads(gdn):
    _check(gdn, _inputs(T=190, B=2, H=3, s0="zero", seed=330))


GATES = {
    "no_decay": lambda x: dict(log_alpha=torch.zeros_like(x["log_alpha"])),
    "erase_zero": lambda x: dict(b=torch.zeros_like(x["b"])),
    "write_zero": lambda x: dict(w=torch.zeros_like(x["w"])),
    "full_decay": lambda x: dict(log_alpha=torch.full_like(x["log_alpha"], -80.0)),
    "erase_write_one": lambda x: dict(b=torch.ones_like(x["b"]), w=torch.ones_like(x["w"])),
}


@pytest.mark.parametrize("gate", list(GATES), ids=list(GATES))
def test_cw_tc_degenerate_gates(gdn, gate):
    inp = _inputs(T=200, law="slow_softplus", seed=340)
    _check(gdn, {**inp, **GATES[gate](inp)})


def test_cw_tc_state_passing_in_place(gdn):
    inp = _inputs(T=300, B=2, seed=350)
    d = {n: (t.cuda() if t is not None else None) for n, t in inp.items()}
    state = d["S0"].clone()
    sl = lambda x, a, b: x[:, a:b].contiguous()
    names = ("q", "k", "v", "log_alpha", "b", "w")
    oa, _ = gdn.chunk_fwd_cw(*(sl(d[n], 0, 100) for n in names), state, chunk=64, S_T=state)
    ob, _ = gdn.chunk_fwd_cw(*(sl(d[n], 100, 300) for n in names), state, chunk=64, S_T=state)
    torch.cuda.synchronize()
    o_ref, S_ref = _oracle(inp)
    assert rel_l2(torch.cat([oa, ob], 1).float().cpu().numpy(), o_ref) <= TOL_BF16
    assert rel_l2(state.cpu().numpy(), S_ref) <= TOL_BF16


def test_cw_tc_scalar_collapse(gdn):
    """Gates that are the same in every channel (log alpha and b = beta per key
    channel, w = beta per value channel) give the scalar rule: compare with the
    scalar oracle."""
    w = I.workload("bf16_T2k", B=1, H=2, T=200, s0_law="normal002", seed=360)
    base = I.chunk_inputs(w)
    la = base["log_alpha"][..., None].expand(-1, -1, -1, w.Dk).contiguous()
    bb = base["beta"][..., None].expand(-1, -1, -1, w.Dk).contiguous()
    wg = base["beta"][..., None].expand(-1, -1, -1, w.Dv).contiguous()
    inp = dict(q=base["q"], k=base["k"], v=base["v"], log_alpha=la, b=bb, w=wg, S0=base["S0"])
    o, S = _run(gdn, inp)
    o_ref, S_ref = O.forward(base["q"], base["k"], base["v"], base["log_alpha"], base["beta"],
                             base["S0"])
    assert rel_l2(o.float().cpu().numpy(), o_ref) <= TOL_BF16
    assert rel_l2(S.cpu().numpy(), S_ref) <= TOL_BF16


def test_cw_tc_workspace_size(gdn):
    # q o 2^Lam, k o 2^(Lam_last - Lam) and w o v per token (bf16), and per chunk
    # and head a [P; T''] tile, a W tile and 2^Lam_last per key channel
    B, T, H, Dv = 2, 130, 3, 192
    tiles = B * 3 * H
    assert gdn.chunk_fwd_cw_workspace_size(B, T, H, 128, Dv, 64, torch.bfloat16) == \
        B * T * H * (256 + Dv) * 2 + tiles * (2 * 64 * 64 + 64 * 128) * 2 + tiles * 128 * 4
    # float32 inputs keep the CUDA-core path
    assert gdn.chunk_fwd_cw_path(B, T, H, 128, Dv, 64, torch.float32) == "simt"
