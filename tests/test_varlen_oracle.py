"""The packed variable-length oracle helper (tests/parity.py: oracle_varlen)
against the batched oracle: equal lengths give the batched result, an empty
sequence hands its initial state through, and splitting a sequence in two with
the state carried across gives the unsplit result."""
import numpy as np
import torch

from gated_delta_rule_130_b200 import inputs as I
from oracle import oracle as O
from parity import oracle_varlen


def _inp(lengths, seed):
    return I.varlen_inputs(lengths, 2, 16, 8, "f32", gate_law="softplus", s0_law="normal002",
                           seed=seed)


def test_equal_lengths_equal_the_batched_oracle():
    inp = _inp([20, 20, 20], 3)
    o, S = oracle_varlen(inp)
    b = lambda t: t.reshape(3, 20, *t.shape[1:])
    ob, Sb = O.forward(b(inp["q"]), b(inp["k"]), b(inp["v"]), b(inp["log_alpha"]),
                       b(inp["beta"]), inp["S0"])
    np.testing.assert_allclose(o, ob.reshape(60, 2, 8), rtol=0, atol=0)
    np.testing.assert_allclose(S, Sb, rtol=0, atol=0)


def test_empty_sequence_keeps_its_initial_state():
    inp = _inp([7, 0, 5], 4)
    o, S = oracle_varlen(inp)
    assert o.shape == (12, 2, 8) and np.all(np.isfinite(o))
    np.testing.assert_array_equal(S[1], inp["S0"][1].double().numpy())


def test_split_sequence_with_carried_state():
    inp = _inp([30], 5)
    o, S = oracle_varlen(inp)
    first = dict(inp, cu_seqlens=[0, 11])
    first = {n: (t[:11] if isinstance(t, torch.Tensor) and n != "S0" else t)
             for n, t in first.items()}
    o1, S1 = oracle_varlen(first)
    second = {n: (t[11:] if isinstance(t, torch.Tensor) and n != "S0" else t)
              for n, t in inp.items()}
    second["cu_seqlens"] = [0, 19]
    second["S0"] = torch.from_numpy(S1)
    o2, S2 = oracle_varlen(second)
    np.testing.assert_allclose(np.concatenate([o1, o2]), o, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(S2, S, rtol=1e-12, atol=1e-14)
