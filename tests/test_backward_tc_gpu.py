"""The tensor-core chunkwise backward (bf16, Dk = 128, chunk 64, Dv 64 or 128)
against the oracle's exact gradient (oracle.backward), every element of all six
gradients compared (GPU only).

The cases reach what is specific to the tensor-core kernels: the state-gradient
chain with dS^T in tensor memory scaled by each chunk's last decay, the bf16
copies of dS' and of the chunk states, the per-chunk products (P^T dO, Z = T^T
dU', the adjoint of the UT transform through Z U'^T, E + E^T), ragged last
chunks (rows past the end loaded as zeros), two value widths, missing S0 /
dS_T, and the degenerate gates the pages name: alpha = 1 (DeltaNet) and
beta = 0 (pure gating), "Gated DeltaNet: Harmonizing Gating and the Delta Rule
for Superior Linear RNNs", section "Problem & Motivation"; beta = 1 with unit
keys (the write-over of its section "Critical Insight"); log alpha = -80 (the
memory erased at every token).
Tolerance: relative L2 2e-2 per gradient (bf16 operands, float32 accumulation,
gradients rounded to bf16 once).
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_130_b200 import inputs as I
from oracle import oracle as O
from parity import rel_l2

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2
NAMES = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0")


@pytest.fixture(scope="module")
def gdn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gated_delta_rule_130_b200 import binding
    return binding


def _case(B=2, H=2, T=300, Dv=128, law="slow_softplus", s0="normal002", seed=900):
    w = I.workload("bf16_T2k", B=B, H=H, T=T, Dv=Dv, gate_law=law, s0_law=s0, seed=seed)
    inp = I.chunk_inputs(w, seed=seed)
    gen = torch.Generator().manual_seed(seed + 99)
    do = torch.randn((B, T, H, Dv), generator=gen).to(torch.bfloat16)
    dS = torch.randn((B, H, Dv, 128), generator=gen)
    return inp, do, dS


def _check(gdn, inp, do, dS, tol=TOL_BF16, with_s0=True):
    B, T, H, Dk = inp["q"].shape
    Dv = inp["v"].shape[3]
    assert gdn.chunk_bwd_path(B, T, H, Dk, Dv, 64, torch.bfloat16) == "tcgen05"
    d = {n: (t.cuda() if t is not None else None) for n, t in inp.items()}
    S0 = d["S0"] if with_s0 else None
    out = gdn.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0, do.cuda(),
                        dS.cuda() if dS is not None else None, chunk=64)
    torch.cuda.synchronize()
    gdn.check_device_status()
    got = [x.float().cpu().numpy() for x in out]
    ref = O.backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                     inp["S0"] if with_s0 else None, do, dS)
    errs = {n: rel_l2(g, np.asarray(r)) for n, g, r in zip(NAMES, got, ref)}
    print("rel-L2", {n: f"{e:.2e}" for n, e in errs.items()}, tuple(inp["q"].shape), Dv)
    for n, g in zip(NAMES, got):
        assert np.isfinite(g).all(), n
    for n, e in errs.items():
        assert e <= tol, f"{n}: rel-L2 {e:.3e} (tol {tol})"


def test_bwd_tc_path_selection(gdn):
    assert gdn.chunk_bwd_path(4, 4096, 16, 128, 128, 64, torch.bfloat16) == "tcgen05"
    assert gdn.chunk_bwd_path(2, 300, 2, 128, 64, 64, torch.bfloat16) == "tcgen05"
    # other value widths, key widths, chunk sizes and float32 keep the CUDA cores
    assert gdn.chunk_bwd_path(2, 300, 2, 128, 192, 64, torch.bfloat16) == "simt"
    assert gdn.chunk_bwd_path(2, 300, 2, 64, 128, 64, torch.bfloat16) == "simt"
    assert gdn.chunk_bwd_path(2, 300, 2, 128, 128, 32, torch.bfloat16) == "simt"
    assert gdn.chunk_bwd_path(2, 300, 2, 128, 128, 64, torch.float32) == "simt"


@pytest.mark.parametrize("T", [1, 63, 64, 65, 300])
def test_bwd_tc_ragged(gdn, T):
    _check(gdn, *_case(T=T, seed=900 + T))


@pytest.mark.parametrize("Dv", [64, 128])
def test_bwd_tc_value_widths(gdn, Dv):
    _check(gdn, *_case(B=1, H=3, T=200, Dv=Dv, seed=950 + Dv))


@pytest.mark.parametrize("law", ["softplus", "uniform5"])
def test_bwd_tc_decay_laws(gdn, law):
    _check(gdn, *_case(T=260, law=law, seed=970))


def test_bwd_tc_without_state_and_state_gradient(gdn):
    inp, do, _ = _case(T=190, s0="zero", seed=980)
    _check(gdn, inp, do, None, with_s0=False)


def _unit_keys(inp):
    k = inp["k"].float()
    return (k / k.norm(dim=-1, keepdim=True)).to(torch.bfloat16)


GATES = {
    "alpha_one": lambda x: dict(log_alpha=torch.zeros_like(x["log_alpha"])),
    "beta_zero": lambda x: dict(beta=torch.zeros_like(x["beta"])),
    "full_decay": lambda x: dict(log_alpha=torch.full_like(x["log_alpha"], -80.0)),
    "beta_one_unit_keys": lambda x: dict(beta=torch.ones_like(x["beta"]), k=_unit_keys(x)),
}


@pytest.mark.parametrize("gate", list(GATES), ids=list(GATES))
def test_bwd_tc_degenerate_gates(gdn, gate):
    inp, do, dS = _case(T=200, seed=990)
    _check(gdn, {**inp, **GATES[gate](inp)}, do, dS)


def test_bwd_tc_workspace_size(gdn):
    # [P; T''], W and T tiles per chunk and head, the chunk states and the state
    # gradients (both bf16), each region rounded up to 256 bytes
    B, T, H, Dv = 2, 130, 3, 128
    NT = 3
    tiles = B * NT * H
    up = lambda n: (n + 255) // 256 * 256
    want = (up(tiles * 2 * 64 * 64 * 2) + up(tiles * 64 * 128 * 2) + up(tiles * 64 * 64 * 2)
            + up(B * H * NT * Dv * 128 * 2) + up(B * H * NT * Dv * 128 * 2))
    assert gdn.chunk_bwd_workspace_size(B, T, H, 128, Dv, 64, torch.bfloat16) == want
