"""Parity of the packed variable-length chunkwise forward (gdn_chunk_fwd_varlen)
with the float64 oracle run sequence by sequence (GPU only).

Tolerances as for the batched paths: 1e-5 on the float32 CUDA-core path,
2e-2 on o and S_T for bf16 inputs.
"""
import pytest
import torch

from gated_delta_rule_130_b200 import inputs as I
from oracle import prologue as PR
from parity import oracle_varlen, rel_l2

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5
TOL_BF16 = 2e-2


@pytest.fixture(scope="module")
def gdn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gated_delta_rule_130_b200 import binding
    return binding


def _run(gdn, inp, chunk=64, **kw):
    d = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}
    o, S = gdn.chunk_fwd_varlen(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                                d["cu_seqlens"], S0=d["S0"], chunk=chunk, **kw)
    torch.cuda.synchronize()
    gdn.check_device_status()
    return o, S


def _check(o, S, inp, tol, heads=None):
    """heads: compare only these heads (the oracle computes only those)."""
    o_ref, S_ref = oracle_varlen(inp, units=heads)
    o, S = o.float().cpu().numpy(), S.cpu().numpy()
    if heads is not None:
        o, S, o_ref, S_ref = o[:, heads], S[:, heads], o_ref[:, heads], S_ref[:, heads]
    eo, es = rel_l2(o, o_ref), rel_l2(S, S_ref)
    assert eo <= tol and es <= tol, f"o {eo:.3e} S {es:.3e}"


@pytest.mark.parametrize("lengths", [[1, 63, 64, 65, 200, 0, 130], [300], [0, 64, 0, 5]])
def test_varlen_tcgen05_path(gdn, lengths):
    inp = I.varlen_inputs(lengths, 3, 128, 128, "bf16", s0_law="normal002", seed=len(lengths))
    assert gdn.chunk_fwd_path(len(lengths), max(lengths), 3, 128, 128, 64, torch.bfloat16) == "tcgen05"
    o, S = _run(gdn, inp)
    _check(o, S, inp, TOL_BF16)


def test_varlen_many_short_sequences(gdn):
    lengths = list(range(1, 41))  # 40 sequences of 1 .. 40 tokens
    inp = I.varlen_inputs(lengths, 2, 128, 128, "bf16", gate_law="softplus", s0_law="normal002",
                          seed=5)
    o, S = _run(gdn, inp)
    _check(o, S, inp, TOL_BF16)


def test_varlen_equal_lengths_match_the_batched_call(gdn):
    """Equal lengths through the varlen entry give the batched call's bits."""
    w = I.workload("bf16_T2k", B=3, H=2, T=150, s0_law="normal002", seed=12)
    b = I.chunk_inputs(w)
    d = {n: (t.cuda() if t is not None else None) for n, t in b.items()}
    o1, S1 = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"])
    pk = lambda t: t.reshape(w.B * w.T, *t.shape[2:])
    o2, S2 = gdn.chunk_fwd_varlen(pk(d["q"]), pk(d["k"]), pk(d["v"]), pk(d["log_alpha"]),
                                  pk(d["beta"]), [0, 150, 300, 450], S0=d["S0"])
    torch.cuda.synchronize()
    assert torch.equal(o1.reshape(-1, w.H, w.Dv), o2) and torch.equal(S1, S2)


def test_varlen_with_prologue(gdn):
    lengths = [70, 0, 129, 3]
    inp = I.varlen_inputs(lengths, 2, 128, 128, "bf16", s0_law="normal002", seed=21)
    # raw keys and queries: scale each row by a power of two (exact in bf16)
    gen = torch.Generator().manual_seed(4)
    for n in ("q", "k"):
        e = torch.randint(-2, 4, inp[n].shape[:2] + (1,), generator=gen).float()
        inp[n] = (inp[n].float() * torch.exp2(e)).to(inp[n].dtype)
    o, S = _run(gdn, inp, l2norm_qk=True, gate_logits=True)
    q, k, la, be = PR.apply(inp["q"].double().numpy(), inp["k"].double().numpy(),
                            inp["log_alpha"].numpy(), inp["beta"].numpy(), True, True)
    ref = dict(inp, q=torch.from_numpy(q), k=torch.from_numpy(k), log_alpha=torch.from_numpy(la),
               beta=torch.from_numpy(be))
    _check(o, S, ref, TOL_BF16)


def test_varlen_all_sequences_empty(gdn):
    inp = I.varlen_inputs([0, 0, 0], 2, 128, 128, "bf16", s0_law="normal002", seed=3)
    d = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}
    S_T = torch.full_like(d["S0"], float("nan"))
    o, S = gdn.chunk_fwd_varlen(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], [0, 0, 0, 0],
                                S0=d["S0"], S_T=S_T)
    torch.cuda.synchronize()
    assert o.numel() == 0 and torch.equal(S, d["S0"])


@pytest.mark.parametrize("chunk", [16, 64])
def test_varlen_cuda_core_path_f32(gdn, chunk):
    lengths = [5, 0, 70, 64, 17]
    inp = I.varlen_inputs(lengths, 2, 32, 48, "f32", gate_law="softplus", s0_law="normal002",
                          seed=chunk)
    assert gdn.chunk_fwd_path(len(lengths), 70, 2, 32, 48, chunk, torch.float32) == "simt"
    o, S = _run(gdn, inp, chunk=chunk)
    _check(o, S, inp, TOL_F32)


def test_varlen_serving_mix_sampled_heads(gdn):
    c = I.VARLEN_SERVING
    lengths = I.varlen_lengths(c["n"], c["total"], c["seed"])
    inp = I.varlen_inputs(lengths, c["H"], c["Dk"], c["Dv"], "bf16", seed=c["seed"])
    o, S = _run(gdn, inp)
    _check(o, S, inp, TOL_BF16, heads=[0, 5, c["H"] - 1])


@pytest.mark.parametrize("H,variant", [(4, "precomputed"), (20, "fused")])
def test_varlen_tcgen05_workspace_size(gdn, H, variant):
    """Per chunk of 64 and head, after the per-sequence chunk offsets: one bf16
    [T'; T''] tile (128 x 64) in the fused variant, one [P; T''] tile and one W
    tile (64 x 128) in the precomputed one (chosen with few sequential CTAs, two
    sequences x H heads x 2 value slices here): the size follows the chunks, not
    the tokens."""
    f = lambda cu, **kw: gdn.chunk_fwd_varlen_workspace_size(cu, H, 128, 128, 64,
                                                             torch.bfloat16, **kw)
    assert gdn.chunk_fwd_variant(2, 66, H, 128, 128, 64, torch.bfloat16) == variant
    tile = H * 128 * 64 * 2 * (2 if variant == "precomputed" else 1)
    assert f([0, 64, 128]) == f([0, 1, 2]) == 256 + 2 * tile
    assert f([0, 1, 66]) == 256 + 3 * tile
    # with L2 normalisation the per-row scales (float32) follow the tiles: 1/|k|
    # in the fused variant, 1/|q| and 1/|k| in the precomputed one
    rows = 64 * 4 * (2 if variant == "precomputed" else 1)
    assert f([0, 1, 66], l2norm_qk=True) == 256 + 3 * tile + 3 * H * rows


def test_varlen_device_offsets_give_the_same_bits(gdn):
    lengths = [100, 3, 64]
    inp = I.varlen_inputs(lengths, 2, 128, 128, "bf16", s0_law="normal002", seed=8,
                          device="cuda")
    cu = inp["cu_seqlens"]
    args = [inp[n] for n in ("q", "k", "v", "log_alpha", "beta")]
    o1, S1 = gdn.chunk_fwd_varlen(*args, cu, S0=inp["S0"])
    o2, S2 = gdn.chunk_fwd_varlen(*args, cu, S0=inp["S0"],
                                  cu_seqlens_device=torch.tensor(cu, dtype=torch.int32,
                                                                 device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_varlen_cuda_core_path_with_prologue_and_state_in_place(gdn):
    lengths = [37, 0, 90, 16]
    inp = I.varlen_inputs(lengths, 2, 32, 24, "f32", s0_law="normal002", seed=31)
    gen = torch.Generator().manual_seed(5)
    for n in ("q", "k"):   # raw rows: scale each by a random factor
        inp[n] = inp[n] * torch.empty(inp[n].shape[:2] + (1,)).uniform_(0.5, 3.0, generator=gen)
    d = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}
    S = d["S0"].clone()
    o, _ = gdn.chunk_fwd_varlen(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                                inp["cu_seqlens"], S0=S, S_T=S, chunk=32, l2norm_qk=True,
                                gate_logits=True)
    torch.cuda.synchronize()
    q, k, la, be = PR.apply(inp["q"].double().numpy(), inp["k"].double().numpy(),
                            inp["log_alpha"].numpy(), inp["beta"].numpy(), True, True)
    ref = dict(inp, q=torch.from_numpy(q), k=torch.from_numpy(k), log_alpha=torch.from_numpy(la),
               beta=torch.from_numpy(be))
    _check(o, S, ref, TOL_F32)
