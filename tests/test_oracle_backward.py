"""CPU pins of the oracle's backward (the first step of the gate-aware backward).

The backward of the fp64 recurrence is pinned against the forward oracle itself,
which tests/test_oracle.py pins against the pages: central finite differences of
L = <d_o, o> + <d_final, S_T> with respect to every entry of every input, on tiny
shapes with d_k != d_v (so that a transposed operand cannot pass), an initial
state and a q scale other than 1.  Three planted mistakes in the backward
(mutants 8-10: the sign of the erase term, the decay left out of the state
gradient, the readout term of dk dropped) must each fail that check.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_forward_b200.inputs import make_inputs

VARIANTS = ["deltanet", "gdn", "kda", "gdn2", "kla"]
INPUTS = ["q", "k", "v", "beta", "log_g", "erase_b", "write_w", "initial_state"]
B, T, H, DK, DV = 1, 5, 2, 4, 3
SCALE = 0.7


def _case(variant, seed=1):
    d = make_inputs(variant, B, T, H, DK, DV, dtype=torch.float32, seed=seed)
    d = {k: (None if v is None else v.double().numpy()) for k, v in d.items()}
    rng = np.random.default_rng(seed)
    s0 = rng.standard_normal((B, H, DK, DV))
    d_o = rng.standard_normal((B, T, H, DV))
    d_final = rng.standard_normal((B, H, DK, DV))
    return d, s0, d_o, d_final


def _loss(variant, d, s0, d_o, d_final):
    o, s = oracle.forward(variant, **d, initial_state=s0, scale=SCALE)
    return float((o * d_o).sum() + (0.0 if d_final is None else (s * d_final).sum()))


def _worst_fd_error(variant, d_final_on=True, mutant=0, h=1e-6):
    """Largest |fd - analytic| / (1 + |analytic|) over every input entry."""
    d, s0, d_o, d_final = _case(variant)
    if not d_final_on:
        d_final = None
    g = oracle.backward(variant, d_o=d_o, d_final=d_final, initial_state=s0, scale=SCALE, mutant=mutant, **d)
    worst = 0.0
    for name in INPUTS:
        base = s0 if name == "initial_state" else d.get(name)
        if g[name] is None or base is None:
            continue
        assert g[name].shape == base.shape, name
        for idx in np.ndindex(base.shape):
            xp, xm = base.copy(), base.copy()
            xp[idx] += h
            xm[idx] -= h
            if name == "initial_state":
                fd = (_loss(variant, d, xp, d_o, d_final) - _loss(variant, d, xm, d_o, d_final)) / (2 * h)
            else:
                fd = (_loss(variant, {**d, name: xp}, s0, d_o, d_final) -
                      _loss(variant, {**d, name: xm}, s0, d_o, d_final)) / (2 * h)
            worst = max(worst, abs(fd - g[name][idx]) / (1.0 + abs(g[name][idx])))
    return worst


@pytest.mark.parametrize("variant", VARIANTS)
def test_backward_matches_finite_differences(variant):
    assert _worst_fd_error(variant) < 1e-7


@pytest.mark.parametrize("variant", ["gdn", "gdn2"])
def test_backward_without_final_state_gradient(variant):
    assert _worst_fd_error(variant, d_final_on=False) < 1e-7


@pytest.mark.parametrize("mutant", [8, 9, 10])
def test_backward_mutants_are_caught(mutant):
    worst = max(_worst_fd_error(v, mutant=mutant) for v in VARIANTS)
    assert worst > 1e-3, f"mutant {mutant} passed the finite-difference pin"


def test_backward_is_linear_in_the_output_gradients():
    d, s0, d_o, d_final = _case("kda", seed=3)
    g1 = oracle.backward("kda", d_o=d_o, d_final=d_final, initial_state=s0, **d)
    g2 = oracle.backward("kda", d_o=2.5 * d_o, d_final=2.5 * d_final, initial_state=s0, **d)
    for name in INPUTS:
        if g1[name] is not None:
            np.testing.assert_allclose(g2[name], 2.5 * g1[name], rtol=1e-12, atol=1e-12)


def test_backward_sequences_are_independent():
    """Two sequences in one call give the gradients of two separate calls."""
    d = make_inputs("gdn", 2, 6, 3, DK, DV, dtype=torch.float32, seed=4)
    d = {k: (None if v is None else v.double().numpy()) for k, v in d.items()}
    rng = np.random.default_rng(4)
    d_o = rng.standard_normal((2, 6, 3, DV))
    g = oracle.backward("gdn", d_o=d_o, **d)
    for b in range(2):
        db = {k: (None if v is None else v[b:b + 1]) for k, v in d.items()}
        gb = oracle.backward("gdn", d_o=d_o[b:b + 1], **db)
        for name in ("q", "k", "v", "beta", "log_g", "initial_state"):
            np.testing.assert_array_equal(gb[name], g[name][b:b + 1])
