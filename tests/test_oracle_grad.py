"""Pins of the oracle's gradients (oracle/prism_grad.py).

The torch restatement of the forward must equal the numpy sequence oracle, and
its autograd gradients must equal central finite differences of that forward
(computed here with no derivative at all), for both residual chains, with S0, a
final-state cotangent and right padding.  Plus two closed forms.
"""
import numpy as np
import pytest
import torch

from oracle import prism_seq
from oracle.prism_grad import INPUTS, prism_seq_grad, prism_seq_torch
from tests.test_oracle_pins import rand_inputs


def _t(d):
    return {n: (None if d[n] is None else torch.tensor(np.asarray(d[n], dtype=np.float64)))
            for n in ("q", "k", "v", "gamma", "beta", "u", "alpha", "gain", "conv_w", "S0")}


@pytest.mark.parametrize("chain", ["linear", "gelu"])
def test_torch_forward_equals_numpy_oracle(chain):
    rng = np.random.default_rng(60)
    d = rand_inputs(rng, B=2, T=19, H=2, dk=5, dv=4, L=4, W=3, s0=True, lengths=np.array([19, 11]))
    o_ref, S_ref = prism_seq(**d, chain=chain)
    o, S = prism_seq_torch(**_t(d), lengths=d["lengths"], chain=chain)
    np.testing.assert_allclose(o.numpy(), o_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S.numpy(), S_ref, rtol=1e-12, atol=1e-12)


def _loss(d, dO, dSf, lengths, chain):
    o, S = prism_seq(**{**d, "lengths": lengths}, chain=chain)
    return float((o * dO).sum() + (S * dSf).sum())


@pytest.mark.parametrize("chain", ["linear", "gelu"])
@pytest.mark.parametrize("lengths", [None, np.array([6, 4])])
def test_gradients_equal_central_differences(chain, lengths):
    rng = np.random.default_rng(61)
    d = rand_inputs(rng, B=2, T=6, H=1, dk=3, dv=2, L=3, W=2, s0=True)
    d.pop("lengths")
    if chain == "gelu":  # the predictor may take any real value
        d["gain"] = rng.standard_normal(d["gain"].shape)
    dO = rng.standard_normal((2, 6, 1, 2))
    dSf = rng.standard_normal((2, 1, 2, 3))
    g = prism_seq_grad(**d, dO=dO, dS_final=dSf, lengths=lengths, chain=chain)
    eps = 1e-6
    for name in INPUTS:
        x = d[name]
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            fd = (_loss({**d, name: xp}, dO, dSf, lengths, chain) - _loss({**d, name: xm}, dO, dSf, lengths, chain)) / (2 * eps)
            assert abs(g[name][idx] - fd) <= 1e-6 * max(1.0, abs(fd)), (name, idx, g[name][idx], fd)


def test_frozen_state_gradient_closed_form():
    """gamma = 1, beta = 0, alpha = 0: S_t = S0 for all t, so
    dL/dS0 = dS_final + sum_t dO_t q_t^T and every write input has zero gradient."""
    rng = np.random.default_rng(62)
    d = rand_inputs(rng, B=1, T=7, H=2, dk=4, dv=3, L=3, W=2, s0=True)
    d.pop("lengths")
    d["gamma"][:] = 1.0
    d["beta"][:] = 0.0
    d["alpha"][:] = 0.0
    dO = rng.standard_normal((1, 7, 2, 3))
    dSf = rng.standard_normal((1, 2, 3, 4))
    g = prism_seq_grad(**d, dO=dO, dS_final=dSf)
    expect = dSf + np.einsum("bthc,bthj->bhcj", dO, d["q"])
    np.testing.assert_allclose(g["S0"], expect, rtol=1e-12, atol=1e-12)
    for n in ("v", "u", "gain", "conv_w"):
        np.testing.assert_allclose(g[n], 0.0, atol=1e-14)


def test_padded_steps_have_no_gradient():
    rng = np.random.default_rng(63)
    d = rand_inputs(rng, B=2, T=9, H=1, dk=3, dv=3, L=2, W=3, s0=True)
    d.pop("lengths")
    lens = np.array([9, 5])
    dO = rng.standard_normal((2, 9, 1, 3))
    g = prism_seq_grad(**d, dO=dO, lengths=lens)
    for n in ("q", "k", "v", "gamma", "beta", "u", "alpha", "gain"):
        np.testing.assert_array_equal(g[n][1, 5:], 0.0)
