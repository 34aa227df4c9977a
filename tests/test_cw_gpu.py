"""Parity of the channel-wise-gate forward and decode step (gdn_chunk_fwd_cw,
gdn_decode_step_cw) with the oracle's token recurrence (oracle.forward_cw).

Tolerances: 1e-5 relative L2 for float32 inputs, 2e-2 on o (and S_T) for bf16.
"""
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


def _run(gdn, inp, chunk):
    d = {n: (t.cuda() if t is not None else None) for n, t in inp.items()}
    o, S = gdn.chunk_fwd_cw(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"],
                            chunk=chunk)
    torch.cuda.synchronize()
    return o.float().cpu().numpy(), S.cpu().numpy()


def _oracle(inp, units=None):
    return O.forward_cw(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"],
                        inp["S0"], units=units)


@pytest.mark.parametrize("chunk", [16, 32, 64])
@pytest.mark.parametrize("T", [1, 64, 100])
def test_cw_f32(gdn, chunk, T):
    w = I.workload("tiny_f32", B=2, H=3, T=T, Dk=32, Dv=48, s0_law="normal002", seed=chunk + T)
    inp = I.cw_inputs(w)
    o, S = _run(gdn, inp, chunk)
    o_ref, S_ref = _oracle(inp)
    assert rel_l2(o, o_ref) <= TOL_F32 and rel_l2(S, S_ref) <= TOL_F32


def test_cw_strong_decay_f32(gdn):
    # log alpha ~ U[-5, 0] per channel: the in-chunk decays underflow, which the
    # per-channel exp(Lam_r - Lam_i) <= 1 factors must handle
    w = I.workload("tiny_f32", B=1, H=2, T=130, Dk=16, Dv=16, gate_law="uniform5",
                   s0_law="normal002", seed=9)
    inp = I.cw_inputs(w)
    o, S = _run(gdn, inp, 64)
    o_ref, S_ref = _oracle(inp)
    assert rel_l2(o, o_ref) <= TOL_F32 and rel_l2(S, S_ref) <= TOL_F32


def test_cw_bf16_d128_sampled_heads(gdn):
    w = I.workload("bf16_T2k", B=2, H=4, T=700, s0_law="normal002", seed=13)
    inp = I.cw_inputs(w)
    o, S = _run(gdn, inp, 64)
    units = [0, 5, 7]
    o_ref, S_ref = _oracle(inp, units=units)
    for u in units:
        b, h = divmod(u, w.H)
        assert rel_l2(o[b, :, h], o_ref[b, :, h]) <= TOL_BF16
        assert rel_l2(S[b, h], S_ref[b, h]) <= TOL_BF16


def test_cw_scalar_collapse_equals_the_scalar_path(gdn):
    w = I.workload("tiny_f32", B=1, H=2, T=90, Dk=16, Dv=24, s0_law="normal002", seed=3)
    base = I.chunk_inputs(w)
    d = {n: (t.cuda() if t is not None else None) for n, t in base.items()}
    o1, S1 = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], chunk=32)
    la = d["log_alpha"][..., None].expand(-1, -1, -1, w.Dk).contiguous()
    b = d["beta"][..., None].expand(-1, -1, -1, w.Dk).contiguous()
    wg = d["beta"][..., None].expand(-1, -1, -1, w.Dv).contiguous()
    o2, S2 = gdn.chunk_fwd_cw(d["q"], d["k"], d["v"], la, b, wg, d["S0"], chunk=32)
    torch.cuda.synchronize()
    assert rel_l2(o2.cpu(), o1.cpu()) <= 1e-5 and rel_l2(S2.cpu(), S1.cpu()) <= 1e-5


def test_cw_no_tokens_and_in_place_state(gdn):
    w = I.workload("tiny_f32", B=1, H=2, T=50, Dk=16, Dv=16, s0_law="normal002", seed=4)
    inp = I.cw_inputs(w)
    d = {n: (t.cuda() if t is not None else None) for n, t in inp.items()}
    S = d["S0"].clone()
    gdn.chunk_fwd_cw(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], S, chunk=16, S_T=S)
    torch.cuda.synchronize()
    _, S_ref = _oracle(inp)
    assert rel_l2(S.cpu().numpy(), S_ref) <= TOL_F32
    e = lambda *s: torch.zeros(*s, device="cuda")
    S_T = torch.full_like(d["S0"], float("nan"))
    gdn.chunk_fwd_cw(e(1, 0, 2, 16), e(1, 0, 2, 16), e(1, 0, 2, 16), e(1, 0, 2, 16),
                     e(1, 0, 2, 16), e(1, 0, 2, 16), d["S0"], chunk=16, S_T=S_T)
    torch.cuda.synchronize()
    assert torch.equal(S_T, d["S0"])


@pytest.mark.parametrize("Dk,Dv,dtype", [(128, 128, "f32"), (128, 128, "bf16"), (256, 36, "f32"),
                                         (256, 64, "bf16"), (48, 20, "f32"), (128, 30, "f32")])
def test_cw_decode(gdn, Dk, Dv, dtype):
    w = I.workload("tiny_f32", B=3, H=2, T=12, Dk=Dk, Dv=Dv, dtype=dtype, s0_law="normal002",
                   seed=Dk + Dv)
    inp = I.cw_inputs(w)
    d = {n: (t.cuda() if t is not None else None) for n, t in inp.items()}
    S = d["S0"].clone()
    outs = []
    for t in range(w.T):
        sl = lambda x: x[:, t].contiguous()
        outs.append(gdn.decode_step_cw(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["log_alpha"]),
                                       sl(d["b"]), sl(d["w"]), S))
    torch.cuda.synchronize()
    o_ref, S_ref = _oracle(inp)
    o = torch.stack(outs, dim=1).float().cpu().numpy()
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    assert rel_l2(o, o_ref) <= tol
    assert rel_l2(S.cpu().numpy(), S_ref) <= TOL_F32
