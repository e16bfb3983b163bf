"""Pins for the oracle's MLP block y = L2(GELU(L1(x))) and its GELU.

* GELU against torch's exact (erf) GELU in float64, against the standard-normal
  table values in tests/golden/gelu_values.txt, and against the identities
  GELU(v) - GELU(-v) = v and GELU(0) = 0;
* the block against a plain torch float64 MLP (Linear -> GELU -> Linear) when
  G = 1, where EQ-Linear is an ordinary linear layer;
* the block against two calls of the pinned forward oracle with torch's GELU in
  between, and its equivariance under cyclic shifts of the group axis (a pointwise
  nonlinearity commutes with the shift).
"""
from __future__ import annotations

import os

import numpy as np
import pytest
import torch

import oracle
from conftest import parse_facts

RNG = np.random.default_rng(77)


def test_gelu_matches_torch_exact_gelu():
    v = np.concatenate([np.linspace(-8, 8, 4001), RNG.standard_normal(1000) * 3])
    ref = torch.nn.functional.gelu(torch.tensor(v), approximate="none").numpy()
    assert np.abs(oracle.gelu(v) - ref).max() <= 1e-15 * max(1.0, np.abs(ref).max())


def test_gelu_table_values_and_identities(golden_dir):
    facts = parse_facts(os.path.join(golden_dir, "gelu_values.txt"))
    got = oracle.gelu(np.array([1.0, 2.0, -1.0, 0.0]))
    assert got[0] == pytest.approx(facts["gelu_at_1"][0], abs=1e-15)
    assert got[1] == pytest.approx(facts["gelu_at_2"][0], abs=1e-15)
    assert got[2] == pytest.approx(facts["gelu_at_minus_1"][0], abs=1e-15)
    assert got[3] == 0.0
    v = RNG.standard_normal(500) * 4
    assert np.abs(oracle.gelu(v) - oracle.gelu(-v) - v).max() <= 1e-14


def _rand_block(N, Cin, H, Cout, G):
    return (RNG.standard_normal((N, Cin, G)), RNG.standard_normal((H, Cin, G)) / np.sqrt(Cin * G),
            RNG.standard_normal(H) * 0.3, RNG.standard_normal((Cout, H, G)) / np.sqrt(H * G),
            RNG.standard_normal(Cout) * 0.3)


def test_mlp_g1_is_a_plain_mlp():
    x, w1, b1, w2, b2 = _rand_block(9, 6, 12, 5, 1)
    t = torch.tensor
    h = torch.nn.functional.linear(t(x[:, :, 0]), t(w1[:, :, 0]), t(b1))
    ref = torch.nn.functional.linear(torch.nn.functional.gelu(h), t(w2[:, :, 0]), t(b2)).numpy()
    got = oracle.mlp_forward(x, w1, b1, w2, b2)[:, :, 0]
    assert np.abs(got - ref).max() <= 1e-12 * np.abs(ref).max()


@pytest.mark.parametrize("G", [2, 4, 8])
def test_mlp_is_two_forwards_around_gelu(G):
    x, w1, b1, w2, b2 = _rand_block(7, 5, 9, 4, G)
    h = oracle.forward(x, w1, b1)
    a = torch.nn.functional.gelu(torch.tensor(h), approximate="none").numpy()
    ref = oracle.forward(a, w2, b2)
    got = oracle.mlp_forward(x, w1, b1, w2, b2)
    assert np.abs(got - ref).max() <= 1e-13 * np.abs(ref).max()


@pytest.mark.parametrize("G", [4, 8])
def test_mlp_block_is_equivariant(G):
    x, w1, b1, w2, b2 = _rand_block(6, 4, 8, 3, G)
    y = oracle.mlp_forward(x, w1, b1, w2, b2)
    for s in range(G):
        ys = oracle.mlp_forward(np.roll(x, s, axis=-1), w1, b1, w2, b2)
        assert np.abs(ys - np.roll(y, s, axis=-1)).max() <= 1e-12 * np.abs(y).max()


def test_mlp_rejects_bad_shapes():
    x, w1, b1, w2, b2 = _rand_block(3, 4, 8, 3, 4)
    with pytest.raises(ValueError):
        oracle.mlp_forward(x, w1, b1, w2[:, :4], b2)


def test_pins_reject_plausible_gelu_mistakes():
    """The tanh approximation, a missing 1/2 or a swapped sign each miss the torch pin."""
    v = np.linspace(-6, 6, 1201)
    ref = torch.nn.functional.gelu(torch.tensor(v), approximate="none").numpy()
    tanh_form = 0.5 * v * (1 + np.tanh(np.sqrt(2 / np.pi) * (v + 0.044715 * v ** 3)))
    from scipy.special import erf
    no_half = v * (1 + erf(v / np.sqrt(2)))
    sign_swapped = 0.5 * v * (1 - erf(v / np.sqrt(2)))
    for bad in (tanh_form, no_half, sign_swapped):
        assert np.abs(bad - ref).max() > 1e-6
