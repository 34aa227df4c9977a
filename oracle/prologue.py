"""Float64 reference of the optional input prologue of the chunkwise forward and
the decode step: per-token L2 normalisation of q and k, and the gate activations.

TEST INFRASTRUCTURE ONLY (like the rest of this directory): the test suite, the
smoke check and the benchmark's CPU leg call it; the CUDA library never does.

What it follows.  The gated delta rule ("Gated Delta Networks: Improving Mamba2
with Delta Rule", atlas.scime.ai summary, section "Approach") takes keys, queries
and two gates alpha_t, beta_t in (0, 1).  The pages state no parameterisation of
the gates and no normalisation of q and k.  The write-over view ("Gated DeltaNet:
Harmonizing Gating and the Delta Rule ...", wispaper.ai blog, section "Critical
Insight": the state is driven towards S_t k_t = v_t) is exact only for unit-norm
keys, so the plain readings taken here are:
  q_hat = q / sqrt(|q|^2 + EPS),  k_hat = k / sqrt(|k|^2 + EPS)   (EPS = 1e-6)
  log alpha = -softplus(x) = -log(1 + e^x)    (alpha = 1 / (1 + e^x) in (0, 1))
  beta = sigmoid(y) = 1 / (1 + e^-y)          (beta in (0, 1))
with x, y unconstrained real inputs ("gate logits").
"""
from __future__ import annotations

import numpy as np

EPS = 1e-6


def l2_normalise(x) -> np.ndarray:
    """x / sqrt(sum of squares over the last axis + EPS), in float64."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + EPS)


def log_alpha_from_logit(x) -> np.ndarray:
    """-softplus(x) = -log(1 + e^x), written as -(max(x, 0) + log1p(e^-|x|)) so that
    neither branch overflows."""
    x = np.asarray(x, dtype=np.float64)
    return -(np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x))))


def beta_from_logit(y) -> np.ndarray:
    """sigmoid(y) = 1 / (1 + e^-y), evaluated on the side where the exponent is <= 0."""
    y = np.asarray(y, dtype=np.float64)
    e = np.exp(-np.abs(y))
    return np.where(y >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def apply(q, k, log_alpha, beta, l2norm_qk: bool, gate_logits: bool):
    """The prologue as the library applies it: returns (q, k, log_alpha, beta) in
    float64, with q, k normalised over their last axis if ``l2norm_qk`` and the two
    gate arrays read as logits if ``gate_logits``."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    la = np.asarray(log_alpha, dtype=np.float64)
    be = np.asarray(beta, dtype=np.float64)
    if l2norm_qk:
        q, k = l2_normalise(q), l2_normalise(k)
    if gate_logits:
        la, be = log_alpha_from_logit(la), beta_from_logit(be)
    return q, k, la, be
