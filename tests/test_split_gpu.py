"""The split tcgen05 variant (GPU only): a fixed-length batch whose sequential grid
covers under a quarter of the GPU has each sequence cut into G segments of whole
chunks.  The chunk recurrence of "Gated Delta Networks: Improving Mamba2 with Delta
Rule" (section "Approach") is affine in the state, so a segment maps its start
state to its end state as S_end = S_start M + N; the segments' maps are formed in
parallel, a scan chains their start states, and the segments then run at once.
Every element of o and S_T is compared with the float64 oracle of the whole
sequence (no segments), at relative L2 2e-2 (bf16 inputs, float32 accumulation).
The gate laws cover slow decay (the maps M far from zero: the scan carries the
state across the segments) and strong decay; S0 = 0, S0 != 0, S_T in place of S0,
both value widths with a split, and the input prologue.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_130_b200 import inputs as I
from oracle import oracle as O
from oracle import prologue as PR
from parity import oracle_chunk, rel_l2

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2


@pytest.fixture(scope="module")
def gdn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gated_delta_rule_130_b200 import binding
    return binding


def test_split_variant_selection(gdn):
    bf = torch.bfloat16
    # one 32K-token sequence of 16 heads: 32 sequential CTAs -> split
    assert gdn.chunk_fwd_variant(1, 32768, 16, 128, 128, 64, bf) == "split"
    assert gdn.chunk_fwd_variant(1, 4096, 2, 128, 128, 64, bf) == "split"
    # T not a multiple of 64 G, segments too short, or a grid that fills the GPU: not split
    assert gdn.chunk_fwd_variant(1, 4000, 2, 128, 128, 64, bf) == "precomputed"
    assert gdn.chunk_fwd_variant(1, 1024, 2, 128, 128, 64, bf) == "precomputed"
    assert gdn.chunk_fwd_variant(4, 4096, 16, 128, 128, 64, bf) == "fused"
    assert gdn.chunk_fwd_variant(1, 32768, 16, 256, 128, 64, bf) == "precomputed"


def _check(gdn, inp, S_in_place=False):
    d = {n: (t.cuda() if t is not None else None) for n, t in inp.items()}
    B, T, H, Dk = d["q"].shape
    Dv = d["v"].shape[3]
    assert gdn.chunk_fwd_variant(B, T, H, Dk, Dv, 64, torch.bfloat16) == "split"
    if S_in_place:
        state = d["S0"].clone()
        o, S = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], state, chunk=64,
                             S_T=state)
    else:
        o, S = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], chunk=64)
    torch.cuda.synchronize()
    gdn.check_device_status()
    o_ref, S_ref = oracle_chunk(inp)
    og, sg = o.float().cpu().numpy(), S.cpu().numpy()
    assert np.isfinite(og).all() and np.isfinite(sg).all()
    eo, es = rel_l2(og, o_ref), rel_l2(sg, S_ref)
    print(f"rel-L2 o={eo:.2e} S_T={es:.2e} shape={tuple(inp['q'].shape)} Dv={Dv}")
    assert eo <= TOL_BF16 and es <= TOL_BF16, f"o {eo:.3e} S_T {es:.3e}"


@pytest.mark.parametrize("law", ["slow_softplus", "softplus", "uniform5"])
def test_split_gate_laws(gdn, law):
    w = I.workload("bf16_T2k", B=1, H=2, T=4096, gate_law=law, s0_law="normal002", seed=1100)
    _check(gdn, I.chunk_inputs(w))


def test_split_two_sequences_zero_state(gdn):
    # B = 2, T = 2048: two segments per sequence
    w = I.workload("bf16_T2k", B=2, H=1, T=2048, s0_law="zero", seed=1110)
    _check(gdn, I.chunk_inputs(w))


def test_split_eight_segments_narrow_values(gdn):
    # Dv = 64: 2 sequential CTAs, eight segments of 16 chunks
    w = I.workload("bf16_T2k", B=1, H=2, T=8192, Dv=64, s0_law="normal002", seed=1120)
    _check(gdn, I.chunk_inputs(w))


def test_split_state_in_place(gdn):
    w = I.workload("bf16_T2k", B=1, H=2, T=4096, s0_law="normal002", seed=1130)
    _check(gdn, I.chunk_inputs(w), S_in_place=True)


def test_split_with_prologue(gdn):
    # raw q, k and gate logits: normalisation and activations in the kernels
    w = I.workload("bf16_T2k", B=1, H=2, T=4096, s0_law="normal002", seed=1140)
    inp = I.raw_chunk_inputs(w)
    d = {n: (t.cuda() if t is not None else None) for n, t in inp.items()}
    assert gdn.chunk_fwd_variant(1, 4096, 2, 128, 128, 64, torch.bfloat16) == "split"
    o, S = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], chunk=64,
                         l2norm_qk=True, gate_logits=True)
    torch.cuda.synchronize()
    gdn.check_device_status()
    q, k, la, be = PR.apply(inp["q"].double().numpy(), inp["k"].double().numpy(),
                            inp["log_alpha"].double().numpy(), inp["beta"].double().numpy(),
                            True, True)
    o_ref, S_ref = O.forward(q, k, inp["v"], la, be, inp["S0"])
    eo, es = rel_l2(o.float().cpu(), o_ref), rel_l2(S.cpu(), S_ref)
    assert eo <= TOL_BF16 and es <= TOL_BF16, f"o {eo:.3e} S_T {es:.3e}"


def test_split_workspace_size(gdn):
    # the precomputed variant's tiles ([P; T''] 16 KiB and W 16 KiB per chunk and
    # head), then per segment N, M, the start state and S_T (float32), 64 zero token
    # rows and one int per segment (an order), each region rounded up to 256 bytes
    B, T, H, Dv, G = 1, 4096, 2, 128, 4
    tiles = B * (T // 64) * H
    nseg = B * G * H
    up = lambda n: (n + 255) // 256 * 256
    want = (up(tiles * 128 * 64 * 2) + up(tiles * 64 * 128 * 2) + up(nseg * Dv * 128 * 4)
            + up(nseg * 128 * 128 * 4) + up(nseg * Dv * 128 * 4) + up(nseg * Dv * 128 * 4)
            + up(64 * H * 128 * 2) + up(B * G * 4))
    assert gdn.chunk_fwd_workspace_size(B, T, H, 128, Dv, 64, torch.bfloat16) == want
