"""gdn_chunk_fwd_noalloc, the entry point for callers that cannot allocate device
memory (its CUDA-core scratch is a fixed array inside the library), called
through the C ABI and compared with gdn_chunk_fwd on two calls in a row.

This file is collected last on purpose: a run that stops at the first failure
has already run every other test when it gets here.
"""
import ctypes

import numpy as np
import pytest
import torch

from gated_delta_rule_130_b200 import inputs as I

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5  # the float32 path's parity tolerance


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


def _noalloc(gdn, d, o, S, w, chunk):
    P = lambda t: t.data_ptr() if t is not None else None
    return gdn.LIB.gdn_chunk_fwd_noalloc(
        P(d["q"]), P(d["k"]), P(d["v"]), P(d["log_alpha"]), P(d["beta"]), P(d["S0"]), P(o), P(S),
        w.B, w.T, w.H, w.Dk, w.Dv, chunk, gdn.GDN_F32, torch.cuda.current_stream().cuda_stream)


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
