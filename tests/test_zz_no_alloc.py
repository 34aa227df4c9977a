"""gdn_chunk_fwd_noalloc, the entry point for callers that cannot allocate device
memory (its scratch is a fixed 8 MiB array inside the library), called through
the C ABI and compared with gdn_chunk_fwd on two calls in a row, on the
CUDA-core path and on the tcgen05 path (whose [T'; T''] tiles then live in the
array), and with the float64 oracle on the tcgen05 sizes.

This file is collected last on purpose: a run that stops at the first failure
has already run every other test when it gets here.
"""
import ctypes

import numpy as np
import pytest
import torch

from gated_delta_rule_130_b200 import inputs as I

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5   # the float32 path's parity tolerance
TOL_BF16 = 2e-2  # bf16 inputs, float32 accumulation
SCRATCH = 8 << 20


def _rel(a, b):
    a = a.detach().double().cpu().numpy()
    b = b.detach().double().cpu().numpy()
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


@pytest.fixture(scope="module")
def gdn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gated_delta_rule_130_b200 import binding
    f = binding.LIB.gdn_chunk_fwd_noalloc
    vp, I_ = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [vp] * 8 + [I_] * 7 + [vp]
    f.restype = I_
    return binding


def _noalloc(gdn, d, o, S, w, chunk, dtype=None):
    P = lambda t: t.data_ptr() if t is not None else None
    code = gdn.GDN_F32 if dtype is None else dtype
    return gdn.LIB.gdn_chunk_fwd_noalloc(
        P(d["q"]), P(d["k"]), P(d["v"]), P(d["log_alpha"]), P(d["beta"]), P(d["S0"]), P(o), P(S),
        w.B, w.T, w.H, w.Dk, w.Dv, chunk, code, torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_chunk_fwd_on_two_calls(gdn):
    # float32 sizes take the CUDA-core path, the one that needs scratch
    for seed in (21, 22):
        w = I.workload("tiny_f32", B=2, H=3, T=100, Dk=32, Dv=48, s0_law="normal002", seed=seed)
        assert gdn.chunk_fwd_path(w.B, w.T, w.H, w.Dk, w.Dv, 32, torch.float32) == "simt"
        d = {n: (t.cuda() if t is not None else None) for n, t in I.chunk_inputs(w).items()}
        o_ref, S_ref = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                                     chunk=32)
        o = torch.empty_like(o_ref)
        S = torch.empty_like(S_ref)
        assert _noalloc(gdn, d, o, S, w, 32) == 0
        torch.cuda.synchronize()
        gdn.check_device_status()
        assert _rel(o, o_ref) <= TOL_F32 and _rel(S, S_ref) <= TOL_F32


def test_noalloc_rejects_sizes_beyond_its_scratch(gdn):
    # workspace of 4 x 16 x 64 chunks of 33 KB each is far above 8 MiB: refused on
    # the host, nothing launched, no pointer dereferenced
    w = I.workload("tiny_f32", B=4, H=16, T=4096, Dk=128, Dv=128)
    need = gdn.chunk_fwd_workspace_size(w.B, w.T, w.H, w.Dk, w.Dv, 64, torch.float32)
    assert need > (8 << 20)
    d = dict(q=None, k=None, v=None, log_alpha=None, beta=None, S0=None)
    assert _noalloc(gdn, d, None, None, w, 64) == 2  # GDN_ERR_UNSUPPORTED


@pytest.mark.parametrize("B,H,T,variant,size", [(1, 2, 256, "precomputed", 256 << 10),
                                                 (2, 64, 256, "fused", 8 << 20)],
                         ids=["precomputed-256KiB", "fused-8MiB"])
def test_noalloc_tcgen05_path_matches_oracle(gdn, B, H, T, variant, size):
    # bf16, Dk = 128, chunk 64: the tcgen05 path, its tiles in the fixed array;
    # B2 H64 T256 (fused) needs the whole 8 MiB
    from parity import head_slices, oracle_chunk
    w = I.workload("bf16_T2k", B=B, H=H, T=T, s0_law="normal002")
    assert gdn.chunk_fwd_path(w.B, w.T, w.H, w.Dk, w.Dv, 64, torch.bfloat16) == "tcgen05"
    assert gdn.chunk_fwd_variant(w.B, w.T, w.H, w.Dk, w.Dv, 64, torch.bfloat16) == variant
    need = gdn.chunk_fwd_workspace_size(w.B, w.T, w.H, w.Dk, w.Dv, 64, torch.bfloat16)
    assert need == size <= SCRATCH
    units = I.sample_units(w, min(4, B * H))
    for seed in (31, 32):
        inp = I.chunk_inputs(w, seed=seed)
        d = {n: (t.cuda() if t is not None else None) for n, t in inp.items()}
        o_ref, S_ref = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                                     chunk=64)
        o = torch.empty_like(o_ref)
        S = torch.empty_like(S_ref)
        assert _noalloc(gdn, d, o, S, w, 64, gdn.GDN_BF16) == 0
        torch.cuda.synchronize()
        gdn.check_device_status()
        assert _rel(o.float(), o_ref.float()) <= TOL_BF16 and _rel(S, S_ref) <= TOL_BF16
        oo, so = oracle_chunk(inp, units=units)
        og, sg = head_slices(o, S, units, w.H)
        orf, srf = head_slices(oo, so, units, w.H)
        ratio = lambda a, b: float(np.linalg.norm(a - b) / np.linalg.norm(b))
        assert ratio(og, orf) <= TOL_BF16 and ratio(sg, srf) <= TOL_BF16


def test_noalloc_alternating_paths(gdn):
    # the array keeps the previous call's contents: a tcgen05 call (bf16 tiles)
    # followed by a CUDA-core call (float32 scratch) and back gives the same
    # results as gdn_chunk_fwd with a workspace of its own
    wt = I.workload("bf16_T2k", B=1, H=2, T=300, s0_law="normal002", seed=41)
    ws = I.workload("tiny_f32", B=2, H=3, T=100, Dk=32, Dv=48, s0_law="normal002", seed=42)
    cases = [(wt, 64, gdn.GDN_BF16, TOL_BF16), (ws, 32, gdn.GDN_F32, TOL_F32)] * 2
    for w, chunk, code, tol in cases:
        d = {n: (t.cuda() if t is not None else None) for n, t in I.chunk_inputs(w).items()}
        o_ref, S_ref = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                                     chunk=chunk)
        o = torch.full_like(o_ref, float("nan"))
        S = torch.full_like(S_ref, float("nan"))
        assert _noalloc(gdn, d, o, S, w, chunk, code) == 0
        torch.cuda.synchronize()
        gdn.check_device_status()
        assert _rel(o.float(), o_ref.float()) <= tol and _rel(S, S_ref) <= tol
