"""Helpers for the parity tests: run the oracle on the same (bf16-rounded) inputs
the CUDA path saw, possibly on a sample of heads, and compare by relative L2."""
import numpy as np
import torch

from oracle import oracle as O


def rel_l2(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(x - ref)
    if den == 0.0:
        return float(num)
    return float(num / den)


def oracle_chunk(inp, units=None):
    """Oracle forward on a dict from gated_delta_rule_130_b200.inputs.chunk_inputs."""
    return O.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"],
                     units=units)


def head_slices(o, S, units, H):
    """Gather the sampled heads of o [B,T,H,Dv] and S [B,H,Dv,Dk] (numpy or torch)."""
    if isinstance(o, torch.Tensor):
        o = o.detach().float().cpu().numpy()
    if isinstance(S, torch.Tensor):
        S = S.detach().float().cpu().numpy()
    os_, ss = [], []
    for u in units:
        b, h = divmod(u, H)
        os_.append(o[b, :, h])
        if S is not None:
            ss.append(S[b, h])
    return np.stack(os_), (np.stack(ss) if S is not None else None)


def oracle_varlen(inp, units=None):
    """Oracle forward of packed variable-length sequences (a dict from
    inputs.varlen_inputs): each sequence on its own, outputs packed back.  With
    ``units`` (heads) only those heads are computed (NaN elsewhere)."""
    cu = inp["cu_seqlens"]
    H, Dv, Dk = inp["q"].shape[1], inp["v"].shape[2], inp["q"].shape[2]
    o = np.full((cu[-1], H, Dv), np.nan)
    S = np.full((len(cu) - 1, H, Dv, Dk), np.nan)
    for n in range(len(cu) - 1):
        a, b = cu[n], cu[n + 1]
        sl = lambda t: t[a:b].unsqueeze(0)
        S0 = inp["S0"][n:n + 1] if inp["S0"] is not None else None
        on, Sn = O.forward(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["log_alpha"]),
                           sl(inp["beta"]), S0, units=units)
        o[a:b] = on[0]
        S[n] = Sn[0]
    return o, S
