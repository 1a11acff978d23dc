"""Pins of the oracle's one-token decode step (the O(1)-state form of the scan).

The decode step carries the ShortConv history explicitly instead of reading
it from the sequence.  It is pinned to the hand-worked two-token example
(tests/golden), to the delta rule's exact recall, and to the pinned sequence
form: decoding a sequence token by token, or decoding the continuation of a
prefix, must give what the sequence form gives.
"""
import json
import os

import numpy as np
import pytest

from oracle import prism_decode_step, prism_seq
from tests.test_oracle_pins import GOLDEN, rand_inputs

TOK = ("q", "k", "v", "gamma", "beta", "u", "alpha", "gain")


def _token(d, t):
    return {n: (None if d[n] is None else d[n][:, t]) for n in TOK}


def _decode_range(d, t_from, t_to, S, hist, chain="linear"):
    outs = []
    for t in range(t_from, t_to):
        o, S, hist = prism_decode_step(**_token(d, t), conv_w=d["conv_w"], conv_state=hist, S=S, chain=chain)
        outs.append(o)
    return np.stack(outs, axis=1), S, hist


def test_decode_reproduces_hand_worked_example():
    with open(os.path.join(GOLDEN, "two_token_hand_example.json")) as f:
        g = json.load(f)
    i = g["inputs"]
    shp = lambda x, *s: np.asarray(x, dtype=np.float64).reshape(*s)
    d = dict(q=shp(i["q"], 1, 2, 1, 2), k=shp(i["k"], 1, 2, 1, 2), v=shp(i["v"], 1, 2, 1, 2),
             gamma=shp(i["gamma"], 1, 2, 1), beta=shp(i["beta"], 1, 2, 1), u=shp(i["u"], 1, 2, 1, 1, 2),
             alpha=shp(i["alpha"], 1, 2, 1, 1), gain=shp(i["gain"], 1, 2, 1, 1, 2),
             conv_w=shp(i["conv_w"], 1, 2, 2))
    o, S, hist = _decode_range(d, 0, 2, np.zeros((1, 1, 2, 2)), np.zeros((1, 1, 1, 2)))
    np.testing.assert_allclose(o.reshape(2, 2), g["expected"]["o"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(S.reshape(2, 2), g["expected"]["S_final"], rtol=0, atol=1e-15)
    np.testing.assert_array_equal(hist.reshape(1, 2), [[6.0, 8.0]])  # v_1 is the history of step 2


def test_decode_exact_recall_of_the_delta_rule():
    """L = 1, beta = 1, unit k: the step stores v under k exactly, so reading
    with q = k returns v (the delta rule's defining property) whatever S held."""
    rng = np.random.default_rng(40)
    B, H, dk, dv = 2, 3, 6, 5
    k = rng.standard_normal((B, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, H, dv))
    S = rng.standard_normal((B, H, dv, dk))
    o, S_new, _ = prism_decode_step(q=k, k=k, v=v, gamma=np.full((B, H), 0.7), beta=np.ones((B, H)), u=None,
                                    alpha=None, gain=None, conv_w=rng.standard_normal((H, dv, 4)),
                                    conv_state=rng.standard_normal((B, H, 3, dv)), S=S)
    np.testing.assert_allclose(o, v, atol=1e-13)


@pytest.mark.parametrize("chain", ["linear", "gelu"])
@pytest.mark.parametrize("W", [1, 2, 4])
def test_decode_loop_equals_sequence_form(chain, W):
    rng = np.random.default_rng(41 + W)
    d = rand_inputs(rng, B=2, T=23, H=2, dk=7, dv=5, L=4, W=W, s0=True)
    o_ref, S_ref = prism_seq(**d, chain=chain)
    B, T, H, dv = d["v"].shape
    o, S, _ = _decode_range(d, 0, T, d["S0"], np.zeros((B, H, W - 1, dv)), chain)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S, S_ref, rtol=1e-12, atol=1e-12)


def test_decode_continues_a_prefix():
    """Prefill [0, T1) with the sequence form, then decode [T1, T) from its final
    state and the last W-1 values of v: the same outputs as one sequence run."""
    rng = np.random.default_rng(45)
    W = 4
    d = rand_inputs(rng, B=2, T=30, H=2, dk=6, dv=6, L=3, W=W, s0=True)
    o_ref, S_ref = prism_seq(**d)
    T1 = 19
    pre = {n: (x[:, :T1] if n in TOK else x) for n, x in d.items()}
    o1, S1 = prism_seq(**pre)
    hist = np.transpose(d["v"][:, T1 - (W - 1):T1], (0, 2, 1, 3))  # [B,H,W-1,dv], oldest first
    o2, S2, _ = _decode_range(d, T1, 30, S1, hist)
    np.testing.assert_allclose(o1, o_ref[:, :T1], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(o2, o_ref[:, T1:], rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(S2, S_ref, rtol=1e-11, atol=1e-11)
