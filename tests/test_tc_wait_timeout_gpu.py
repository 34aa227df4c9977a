"""Failure detection of the tcgen05 chunkwise forward, made to happen without a
GPU fault: the test hook gdn_debug_withhold_first_arrival makes the fused
variant's sequential kernel's TMA warp withhold the arrival that publishes its first stage, so every
warp's first bounded wait (about two seconds) runs out.  The CTAs record the
error flag, stop, drain their copies and release their tensor memory;
gdn_check_device_status must report it, and the next call (hook off) must run
normally and match the oracle.  Nothing here traps, faults or hangs the GPU.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_130_b200 import inputs as I
from parity import oracle_chunk, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gdn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gated_delta_rule_130_b200 import binding
    return binding


def test_bounded_wait_runs_out_and_context_survives(gdn):
    # the hook is in the fused variant's sequential kernel: 80 CTAs (heads x one
    # value slice) select it
    w = I.workload("bf16_T2k", B=1, H=80, T=128, Dv=64, s0_law="normal002", seed=91)
    assert gdn.chunk_fwd_path(w.B, w.T, w.H, w.Dk, w.Dv, 64, torch.bfloat16) == "tcgen05"
    assert gdn.chunk_fwd_variant(w.B, w.T, w.H, w.Dk, w.Dv, 64, torch.bfloat16) == "fused"
    inp = I.chunk_inputs(w)
    d = {n: (t.cuda() if t is not None else None) for n, t in inp.items()}
    gdn.check_device_status()  # a clean flag to start from
    assert gdn.LIB.gdn_debug_withhold_first_arrival(1) == 0
    try:
        gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], chunk=64)
        with pytest.raises(gdn.GdnError):
            gdn.check_device_status()
    finally:
        assert gdn.LIB.gdn_debug_withhold_first_arrival(0) == 0
    gdn.check_device_status()  # the flag was cleared by the read
    o, S = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], chunk=64)
    gdn.check_device_status()
    o_ref, S_ref = oracle_chunk(inp)
    assert np.isfinite(o.float().cpu().numpy()).all()
    assert rel_l2(o.float().cpu().numpy(), o_ref) <= 2e-2
    assert rel_l2(S.cpu().numpy(), S_ref) <= 2e-2
