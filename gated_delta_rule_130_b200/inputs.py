"""Seeded synthetic inputs for the gated delta rule.

This module holds the workload table and the random draws only -- none of the
rule's arithmetic.  Both the CUDA path's tests/benchmark and the CPU oracle are
fed from here, so both see the same bits.

Draw recipe (one ``torch.Generator`` per workload, CPU, float32): q, k, v, the
beta logit, the gate logit, then S0, each ~N(0,1) unless stated.  q and k are
L2-normalised per token and head in float32, then rounded to the workload's
dtype; v is rounded to the dtype; beta = sigmoid(logit); log_alpha is one of
    -softplus(x),  -0.1 * softplus(x)  (slow decay),  Uniform[-5, 0];
S0 is zero or N(0, std 0.02) in float32.  The gates stay float32.

The shapes and laws mirror the layers the pages train (1.3B-parameter Gated
DeltaNet models: "Gated DeltaNet: Harmonizing Gating and the Delta Rule for
Superior Linear RNNs", section "Experiments: Performance at Scale"); no dataset
is involved, the inputs are synthetic stand-ins.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    Dk: int
    Dv: int
    chunk: int
    dtype: str          # "f32" or "bf16": type of q, k, v and o
    gate_law: str       # "softplus", "slow_softplus" or "uniform5"
    s0_law: str         # "zero" or "normal002"
    seed: int
    steps: int = 0      # decode workloads: number of successive single-token steps

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


# The chunkwise-forward shapes, the headline shape and the decode shape.
WORKLOADS = {
    w.name: w for w in [
        Workload("tiny_f32", 1, 2, 64, 16, 16, 16, "f32", "softplus", "zero", 1001),
        Workload("bf16_T2k", 4, 16, 2048, 128, 128, 64, "bf16", "slow_softplus", "zero", 1002),
        Workload("long_T32k", 1, 16, 32768, 128, 128, 64, "bf16", "uniform5", "normal002", 1003),
        Workload("wide_dk256_dv512", 8, 6, 4096, 256, 512, 64, "bf16", "softplus", "zero", 1004),
        Workload("decode_b256", 256, 16, 1, 128, 128, 0, "bf16", "softplus", "normal002", 1005,
                 steps=1000),
        Workload("headline_T4k", 4, 16, 4096, 128, 128, 64, "bf16", "slow_softplus", "zero", 1006),
    ]
}

HEADLINE = "headline_T4k"


def workload(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    return replace(w, **overrides) if overrides else w


def _gates(gen, shape, law):
    beta = torch.sigmoid(torch.randn(shape, generator=gen))
    x = torch.randn(shape, generator=gen)
    if law == "softplus":
        la = -torch.nn.functional.softplus(x)
    elif law == "slow_softplus":
        la = -0.1 * torch.nn.functional.softplus(x)
    elif law == "uniform5":
        la = -5.0 * torch.rand(shape, generator=gen)
    else:
        raise ValueError(law)
    return la.contiguous(), beta.contiguous()


def _unit_rows(x):
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def chunk_inputs(w: Workload, seed: int | None = None, device="cpu"):
    """Inputs of one chunkwise forward call, as CPU (or ``device``) tensors.

    q,k [B,T,H,Dk] dtype; v [B,T,H,Dv] dtype; log_alpha, beta [B,T,H] f32;
    S0 [B,H,Dv,Dk] f32 or None.
    """
    gen = torch.Generator().manual_seed(w.seed if seed is None else seed)
    B, T, H, Dk, Dv = w.B, w.T, w.H, w.Dk, w.Dv
    q = _unit_rows(torch.randn((B, T, H, Dk), generator=gen)).to(w.torch_dtype)
    k = _unit_rows(torch.randn((B, T, H, Dk), generator=gen)).to(w.torch_dtype)
    v = torch.randn((B, T, H, Dv), generator=gen).to(w.torch_dtype)
    la, beta = _gates(gen, (B, T, H), w.gate_law)
    S0 = None
    if w.s0_law == "normal002":
        S0 = 0.02 * torch.randn((B, H, Dv, Dk), generator=gen)
    out = dict(q=q, k=k, v=v, log_alpha=la, beta=beta, S0=S0)
    if device != "cpu":
        out = {n: (t.to(device) if t is not None else None) for n, t in out.items()}
    return out


def cw_inputs(w: Workload, seed: int | None = None, device="cpu"):
    """Inputs with channel-wise gates: as ``chunk_inputs`` (same q, k, v and S0
    draws for the same seed), with log_alpha [B,T,H,Dk] drawn by the workload's
    gate law per key channel, an erase gate b = sigmoid(N) [B,T,H,Dk] and a write
    gate w = sigmoid(N) [B,T,H,Dv], all float32."""
    gen = torch.Generator().manual_seed(w.seed if seed is None else seed)
    B, T, H, Dk, Dv = w.B, w.T, w.H, w.Dk, w.Dv
    q = _unit_rows(torch.randn((B, T, H, Dk), generator=gen)).to(w.torch_dtype)
    k = _unit_rows(torch.randn((B, T, H, Dk), generator=gen)).to(w.torch_dtype)
    v = torch.randn((B, T, H, Dv), generator=gen).to(w.torch_dtype)
    la, b = _gates(gen, (B, T, H, Dk), w.gate_law)
    wg = torch.sigmoid(torch.randn((B, T, H, Dv), generator=gen)).contiguous()
    S0 = None
    if w.s0_law == "normal002":
        S0 = 0.02 * torch.randn((B, H, Dv, Dk), generator=gen)
    out = dict(q=q, k=k, v=v, log_alpha=la, b=b, w=wg, S0=S0)
    if device != "cpu":
        out = {n: (t.to(device) if t is not None else None) for n, t in out.items()}
    return out


def raw_chunk_inputs(w: Workload, seed: int | None = None, device="cpu"):
    """Inputs for the library's optional input prologue (per-token L2 normalisation
    of q and k, gate activations): q, k ~ 2 N(0,1) rounded to the dtype and NOT
    normalised; v as in ``chunk_inputs``; the two gate arrays hold logits ~ N(0,1)
    (decay logit in ``log_alpha``, write logit in ``beta``); S0 per the workload."""
    gen = torch.Generator().manual_seed((w.seed if seed is None else seed) + 500_000)
    B, T, H, Dk, Dv = w.B, w.T, w.H, w.Dk, w.Dv
    q = (2.0 * torch.randn((B, T, H, Dk), generator=gen)).to(w.torch_dtype)
    k = (2.0 * torch.randn((B, T, H, Dk), generator=gen)).to(w.torch_dtype)
    v = torch.randn((B, T, H, Dv), generator=gen).to(w.torch_dtype)
    x = torch.randn((B, T, H), generator=gen)
    y = torch.randn((B, T, H), generator=gen)
    S0 = None
    if w.s0_law == "normal002":
        S0 = 0.02 * torch.randn((B, H, Dv, Dk), generator=gen)
    out = dict(q=q, k=k, v=v, log_alpha=x, beta=y, S0=S0)
    if device != "cpu":
        out = {n: (t.to(device) if t is not None else None) for n, t in out.items()}
    return out


def raw_decode_step_inputs(w: Workload, step: int, device="cpu"):
    """Token ``step`` of a decode run for the input prologue: raw q, k (2 N(0,1)),
    v, and the decay / write logits ~ N(0,1) in ``log_alpha`` / ``beta``."""
    gen = torch.Generator().manual_seed(w.seed * 1_000_003 + step + 7_000_001)
    B, H, Dk, Dv = w.B, w.H, w.Dk, w.Dv
    q = (2.0 * torch.randn((B, H, Dk), generator=gen)).to(w.torch_dtype)
    k = (2.0 * torch.randn((B, H, Dk), generator=gen)).to(w.torch_dtype)
    v = torch.randn((B, H, Dv), generator=gen).to(w.torch_dtype)
    out = dict(q=q, k=k, v=v, log_alpha=torch.randn((B, H), generator=gen),
               beta=torch.randn((B, H), generator=gen))
    if device != "cpu":
        out = {n: t.to(device) for n, t in out.items()}
    return out


def varlen_lengths(n: int, total: int, seed: int, min_len: int = 1):
    """n sequence lengths summing to ``total``: a seeded log-uniform mix (a few long
    prompts, many short ones, ragged ends), each at least ``min_len``."""
    gen = torch.Generator().manual_seed(seed)
    w = torch.exp(torch.rand(n, generator=gen) * 4.0)          # spread of e^4 ~ 55x
    raw = (w / w.sum() * (total - n * min_len)).floor().long() + min_len
    raw[0] += total - int(raw.sum())                            # exact total
    return [int(x) for x in raw]


def varlen_inputs(lengths, H: int, Dk: int, Dv: int, dtype: str = "bf16",
                  gate_law: str = "slow_softplus", s0_law: str = "zero", seed: int = 2001,
                  device="cpu"):
    """Sequences of the given lengths packed along the token dimension: q, k
    [total, H, Dk] (unit rows), v [total, H, Dv], log_alpha, beta [total, H] f32,
    S0 [N, H, Dv, Dk] f32 or None, and cu_seqlens (N + 1 int offsets, a list).
    Same draw recipe as ``chunk_inputs`` with B = 1 and T = total."""
    total = int(sum(lengths))
    w = Workload("varlen", 1, H, total, Dk, Dv, 64, dtype, gate_law, "zero", seed)
    d = chunk_inputs(w)
    out = {n: d[n][0] for n in ("q", "k", "v", "log_alpha", "beta")}
    gen = torch.Generator().manual_seed(seed + 77)
    out["S0"] = (0.02 * torch.randn((len(lengths), H, Dv, Dk), generator=gen)
                 if s0_law == "normal002" else None)
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    if device != "cpu":
        out = {n: (t.to(device) if t is not None else None) for n, t in out.items()}
    out["cu_seqlens"] = cu
    return out


# Serving-shaped prefill batch: 12 sequences of mixed lengths, 16,384 tokens in all
# (the headline's token count), H 16, d 128, bf16.
VARLEN_SERVING = dict(n=12, total=16384, seed=2002, H=16, Dk=128, Dv=128)


def decode_state(w: Workload, device="cpu"):
    """Initial decode state S0 [B,H,Dv,Dk] f32."""
    gen = torch.Generator().manual_seed(w.seed)
    S0 = torch.zeros((w.B, w.H, w.Dv, w.Dk))
    if w.s0_law == "normal002":
        S0 = 0.02 * torch.randn((w.B, w.H, w.Dv, w.Dk), generator=gen)
    return S0.to(device)


def decode_step_inputs(w: Workload, step: int, device="cpu"):
    """Token ``step`` of a decode run: q,k [B,H,Dk], v [B,H,Dv] dtype; gates [B,H] f32."""
    gen = torch.Generator().manual_seed(w.seed * 1_000_003 + step + 1)
    B, H, Dk, Dv = w.B, w.H, w.Dk, w.Dv
    q = _unit_rows(torch.randn((B, H, Dk), generator=gen)).to(w.torch_dtype)
    k = _unit_rows(torch.randn((B, H, Dk), generator=gen)).to(w.torch_dtype)
    v = torch.randn((B, H, Dv), generator=gen).to(w.torch_dtype)
    la, beta = _gates(gen, (B, H), w.gate_law)
    out = dict(q=q, k=k, v=v, log_alpha=la, beta=beta)
    if device != "cpu":
        out = {n: t.to(device) for n, t in out.items()}
    return out


def sample_units(w: Workload, n: int, seed: int = 7):
    """A fixed, seeded sample of (b*H + h) head indices, always including the first
    and the last head."""
    total = w.B * w.H
    if n >= total:
        return list(range(total))
    gen = torch.Generator().manual_seed(seed)
    mid = torch.randperm(total - 2, generator=gen)[: max(n - 2, 0)] + 1
    return sorted({0, total - 1, *[int(x) for x in mid]})
