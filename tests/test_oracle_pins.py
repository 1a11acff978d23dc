"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test states which passage of the PRISM pages, which textbook identity or
which library routine fixes the expected value.  A plausible slip in the
oracle (a wrong tap direction, a transposed state, a pre- instead of a
post-update readout, gamma applied to the write, a dropped residual term, a
sign error in the delta rule) fails at least one of them.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.signal

from oracle import (
    affine_maps,
    gdn_seq,
    max_abs_rel_err,
    prism_chunked,
    prism_seq,
    residual_chain,
    residual_write,
    shortconv_anchor,
)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_inputs(rng, B=2, T=37, H=2, dk=8, dv=6, L=3, W=4, s0=False, lengths=None):
    """Generic fp64 inputs (no bf16 rounding needed for oracle-only pins)."""
    m = L - 1
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q = rng.standard_normal((B, T, H, dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    d = dict(
        q=q,
        k=k,
        v=rng.standard_normal((B, T, H, dv)),
        gamma=1.0 / (1.0 + np.exp(-rng.normal(3.0, 0.5, (B, T, H)))),
        beta=1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H)))),
        u=rng.standard_normal((B, T, H, m, dk)) / np.sqrt(dk),
        alpha=1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H, m)))),
        gain=1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H, m, dv)))),
        conv_w=rng.standard_normal((H, dv, W)) / np.sqrt(W),
        S0=(0.3 * rng.standard_normal((B, H, dv, dk))) if s0 else None,
        lengths=lengths,
    )
    return d


# ---------------------------------------------------------------- hand example
def test_hand_worked_two_token_example():
    with open(os.path.join(GOLDEN, "two_token_hand_example.json")) as f:
        g = json.load(f)
    i = g["inputs"]
    T, dk, dv = 2, 2, 2
    shp = lambda x, *s: np.asarray(x, dtype=np.float64).reshape(*s)
    o, S = prism_seq(
        q=shp(i["q"], 1, T, 1, dk), k=shp(i["k"], 1, T, 1, dk), v=shp(i["v"], 1, T, 1, dv),
        gamma=shp(i["gamma"], 1, T, 1), beta=shp(i["beta"], 1, T, 1),
        u=shp(i["u"], 1, T, 1, 1, dk), alpha=shp(i["alpha"], 1, T, 1, 1),
        gain=shp(i["gain"], 1, T, 1, 1, dv), conv_w=shp(i["conv_w"], 1, dv, 2),
    )
    np.testing.assert_allclose(o.reshape(T, dv), g["expected"]["o"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(S.reshape(dv, dk), g["expected"]["S_final"], rtol=0, atol=1e-15)


# ---------------------------------------------------------------- anchor
def test_anchor_matches_library_fir_filter():
    """The ShortConv anchor is a causal FIR filter along t with zero initial
    history; scipy.signal.lfilter(b=w, a=[1]) computes exactly that."""
    rng = np.random.default_rng(1)
    v = rng.standard_normal((2, 19, 3, 5))
    w = rng.standard_normal((3, 5, 4))
    a = shortconv_anchor(v, w)
    for b in range(2):
        for h in range(3):
            for c in range(5):
                ref = scipy.signal.lfilter(w[h, c], [1.0], v[b, :, h, c])
                np.testing.assert_allclose(a[b, :, h, c], ref, rtol=1e-13, atol=1e-13)


def test_anchor_window_longer_than_sequence():
    rng = np.random.default_rng(2)
    v = rng.standard_normal((1, 2, 1, 3))
    w = rng.standard_normal((1, 3, 4))
    a = shortconv_anchor(v, w)
    ref = np.stack([w[0, :, 0] * v[0, 0, 0], w[0, :, 0] * v[0, 1, 0] + w[0, :, 1] * v[0, 0, 0]])
    np.testing.assert_allclose(a[0, :, 0], ref, atol=1e-15)


# ---------------------------------------------------------------- residual chain
def test_residual_chain_closed_form_and_monotone():
    """[blog] 消除 Step 间串行: the linearised chain has a closed form, a cumulative
    product; [blog] 关键洞察: the residual decreases step by step (g in (0,1))."""
    rng = np.random.default_rng(3)
    d = rand_inputs(rng, L=5)
    r = residual_chain(d["v"], d["conv_w"], d["gain"])
    r0 = d["v"] - shortconv_anchor(d["v"], d["conv_w"])
    closed = np.cumprod(1.0 - d["gain"], axis=3) * r0[:, :, :, None, :]
    np.testing.assert_allclose(r, closed, rtol=1e-13, atol=1e-14)
    prev = np.abs(r0)
    for l in range(r.shape[3]):
        assert np.all(np.abs(r[:, :, :, l]) <= prev + 1e-15)
        prev = np.abs(r[:, :, :, l])


def test_rank_of_residual_and_total_write():
    """[summary] sec. 3 / [poster]: the injection has rank L per token; the
    residual part alone has rank L-1 on generic inputs."""
    rng = np.random.default_rng(4)
    for L in (2, 4, 8):
        d = rand_inputs(rng, B=1, T=6, H=1, dk=12, dv=12, L=L)
        dS = residual_write(d["v"], d["u"], d["alpha"], d["gain"], d["conv_w"])
        _, Bt = affine_maps(d["k"], d["v"], d["gamma"], d["beta"], d["u"], d["alpha"], d["gain"], d["conv_w"])
        for t in range(6):
            s = np.linalg.svd(dS[0, t, 0], compute_uv=False)
            assert int((s > 1e-10 * s[0]).sum()) == L - 1
            s = np.linalg.svd(Bt[0, t, 0], compute_uv=False)
            assert int((s > 1e-10 * s[0]).sum()) == L


def test_affine_transition_eigenstructure_and_gdn_product():
    """The transition half of affine_maps, A_t = gamma_t (I - beta_t k_t k_t^T)
    ([summary] sec. 2.1: the forgetting path is the rank-1 gated-delta transition),
    pinned without the oracle's own scan.  Textbook facts of a rank-1 update of the
    identity with a unit vector k: A_t is symmetric, k_t is an eigenvector with
    eigenvalue gamma_t (1 - beta_t), every vector orthogonal to k_t has eigenvalue
    gamma_t; padded steps give the identity.  And with the writes off (v = 0), the
    ordered product S0 A_1 A_2 ... A_T is the final state of the separately written
    gated-delta recurrence gdn_seq started from S0.  Dropping gamma or beta, or a
    transposed or reversed product, fails one of these."""
    rng = np.random.default_rng(11)
    B, T, H, dk, dv = 2, 9, 2, 6, 5
    d = rand_inputs(rng, B=B, T=T, H=H, dk=dk, dv=dv, L=3)
    d["gamma"] = rng.uniform(0.3, 0.9, (B, T, H))   # both well away from 1 and 0
    d["beta"] = rng.uniform(0.2, 0.8, (B, T, H))
    lengths = np.array([T, T - 3])
    A, _ = affine_maps(d["k"], d["v"], d["gamma"], d["beta"], d["u"], d["alpha"], d["gain"], d["conv_w"],
                       lengths=lengths)
    for b in range(B):
        for t in range(T):
            for h in range(H):
                a = A[b, t, h]
                if t >= lengths[b]:
                    np.testing.assert_array_equal(a, np.eye(dk))
                    continue
                k, g, be = d["k"][b, t, h], d["gamma"][b, t, h], d["beta"][b, t, h]
                np.testing.assert_allclose(a, a.T, rtol=0, atol=1e-15)
                np.testing.assert_allclose(a @ k, g * (1 - be) * k, rtol=0, atol=1e-14)
                x = rng.standard_normal(dk)
                x -= (x @ k) * k  # orthogonal to the unit key
                np.testing.assert_allclose(a @ x, g * x, rtol=0, atol=1e-14)
    S0 = rng.standard_normal((B, H, dv, dk))
    _, S_ref = gdn_seq(d["q"], d["k"], np.zeros((B, T, H, dv)), d["gamma"], d["beta"], S0=S0, lengths=lengths)
    for b in range(B):
        for h in range(H):
            S = S0[b, h]
            for t in range(T):
                S = S @ A[b, t, h]
            np.testing.assert_allclose(S, S_ref[b, h], rtol=0, atol=1e-13)


def test_gain_extremes():
    """g = 0: every step keeps r_0, so dS_res = r_0 (sum_l alpha_l u_l)^T (rank 1).
    g = 1: the first step removes the whole residual, dS_res = 0 and PRISM = GDN."""
    rng = np.random.default_rng(5)
    d = rand_inputs(rng, L=4)
    d0 = dict(d, gain=np.zeros_like(d["gain"]))
    dS = residual_write(d0["v"], d0["u"], d0["alpha"], d0["gain"], d0["conv_w"])
    r0 = d["v"] - shortconv_anchor(d["v"], d["conv_w"])
    ref = np.einsum("bthc,bthj->bthcj", r0, np.einsum("bthl,bthlj->bthj", d["alpha"], d["u"]))
    np.testing.assert_allclose(dS, ref, rtol=1e-13, atol=1e-13)
    d1 = dict(d, gain=np.ones_like(d["gain"]))
    o, S = prism_seq(**d1)
    og, Sg = gdn_seq(d["q"], d["k"], d["v"], d["gamma"], d["beta"])
    assert max_abs_rel_err(o, og) < 1e-12
    np.testing.assert_allclose(S, Sg, rtol=1e-11, atol=1e-12)


def test_identity_anchor_gives_gdn_for_any_L():
    """Anchor tap w[.,.,0] = 1, others 0: the anchor equals v, r_0 = 0, every
    residual write vanishes and the layer is exactly GDN."""
    rng = np.random.default_rng(6)
    d = rand_inputs(rng, L=5)
    w = np.zeros_like(d["conv_w"])
    w[..., 0] = 1.0
    o, S = prism_seq(**dict(d, conv_w=w))
    og, Sg = gdn_seq(d["q"], d["k"], d["v"], d["gamma"], d["beta"])
    assert max_abs_rel_err(o, og) < 1e-12
    np.testing.assert_allclose(S, Sg, rtol=1e-11, atol=1e-12)


def test_zero_anchor_writes_v():
    rng = np.random.default_rng(7)
    d = rand_inputs(rng, L=2)
    r = residual_chain(d["v"], np.zeros_like(d["conv_w"]), d["gain"])
    np.testing.assert_allclose(r[:, :, :, 0], (1 - d["gain"][:, :, :, 0]) * d["v"], rtol=1e-14)


def test_strictly_past_anchor_taps():
    """A strictly-past anchor (tap 0 = 0, tap 1 = 1) gives r_0,t = v_t - v_{t-1}
    (numpy's first difference, with v_{-1} = 0)."""
    rng = np.random.default_rng(8)
    d = rand_inputs(rng, L=2)
    w = np.zeros_like(d["conv_w"])
    w[..., 1] = 1.0
    g0 = np.zeros_like(d["gain"])
    r = residual_chain(d["v"], w, g0)[:, :, :, 0]
    ref = np.diff(d["v"], axis=1, prepend=0.0)
    np.testing.assert_allclose(r, ref, rtol=1e-14, atol=1e-14)


# ---------------------------------------------------------------- GDN part
@pytest.mark.parametrize("s0,lens", [(False, None), (True, [30, 11])])
def test_L1_equals_separate_gdn(s0, lens):
    """[blog] 架构形式: with L = 1 PRISM is exactly GDN."""
    rng = np.random.default_rng(9)
    d = rand_inputs(rng, L=1, s0=s0, lengths=None if lens is None else np.array(lens))
    o, S = prism_seq(**dict(d, u=None, alpha=None, gain=None))
    og, Sg = gdn_seq(d["q"], d["k"], d["v"], d["gamma"], d["beta"], S0=d["S0"], lengths=d["lengths"])
    assert max_abs_rel_err(o, og) < 1e-12
    np.testing.assert_allclose(S, Sg, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("L", [1, 3])
def test_delta_rule_exact_recall(L):
    """With beta = 1, alpha = 0 and unit keys the delta rule stores v_t exactly
    under k_t: the post-update state satisfies S_t k_t = v_t, whatever gamma and
    the history.  Reading with q_t = k_t then returns v_t (this also pins the
    readout to the post-update state and the orientation S in R^{d_v x d_k})."""
    rng = np.random.default_rng(10)
    d = rand_inputs(rng, L=L, s0=True, dv=5, dk=7)
    d["beta"] = np.ones_like(d["beta"])
    d["q"] = d["k"].copy()
    if L > 1:
        d["alpha"] = np.zeros_like(d["alpha"])
    else:
        d.update(u=None, alpha=None, gain=None)
    o, _ = prism_seq(**d)
    np.testing.assert_allclose(o, d["v"], rtol=1e-12, atol=1e-12)


def test_zero_and_frozen_state():
    """gamma = 1, beta = 0, alpha = 0: nothing is written or forgotten, so S stays
    at S0 (zero state -> zero output; S0 != 0 -> o_t = S0 q_t)."""
    rng = np.random.default_rng(11)
    d = rand_inputs(rng, L=3, s0=True)
    d.update(gamma=np.ones_like(d["gamma"]), beta=np.zeros_like(d["beta"]), alpha=np.zeros_like(d["alpha"]))
    o, S = prism_seq(**dict(d, S0=None))
    assert np.all(o == 0) and np.all(S == 0)
    o, S = prism_seq(**d)
    np.testing.assert_array_equal(S, d["S0"])
    np.testing.assert_allclose(o, np.einsum("bhcj,bthj->bthc", d["S0"], d["q"]), rtol=1e-14, atol=1e-14)


def test_pure_decay_closed_form():
    """beta = 0, alpha = 0: S_t = (prod_{j<=t} gamma_j) S0."""
    rng = np.random.default_rng(12)
    d = rand_inputs(rng, L=2, s0=True)
    d.update(beta=np.zeros_like(d["beta"]), alpha=np.zeros_like(d["alpha"]))
    _, S = prism_seq(**d)
    decay = np.prod(d["gamma"], axis=1)  # [B,H]
    np.testing.assert_allclose(S, decay[..., None, None] * d["S0"], rtol=1e-12)


# ---------------------------------------------------------------- affine form, exact
def _frac_inputs(rng, T, dk, dv, L, W):
    """Dyadic rationals (exact in fp64) and their Fraction copies."""
    def dy(shape, lo, hi, den=16):
        return rng.integers(lo, hi, size=shape) / den
    m = L - 1
    d = dict(
        q=dy((1, T, 1, dk), -16, 17), k=dy((1, T, 1, dk), -16, 17), v=dy((1, T, 1, dv), -32, 33),
        gamma=dy((1, T, 1), 10, 16), beta=dy((1, T, 1), 1, 16),
        u=dy((1, T, 1, m, dk), -8, 9), alpha=dy((1, T, 1, m), 1, 16),
        gain=dy((1, T, 1, m, dv), 1, 16), conv_w=dy((1, dv, W), -8, 9),
        S0=dy((1, 1, dv, dk), -8, 9),
    )
    return d


def _F(x):
    return np.vectorize(lambda z: Fraction(z))(np.asarray(x, dtype=np.float64)).astype(object)


def test_affine_scan_exact_rational():
    """[summary] sec. 2.1: S_t = S_{t-1} A_t + B_t with A_t = gamma(I - beta k k^T)
    and B_t the injection.  [blog] 背景: because A_t, B_t depend on inputs only,
    the maps compose associatively (parallel prefix scan).  Here the maps are
    built and composed in exact rational arithmetic, by recursive doubling
    (a tree order unlike the oracle's token loop), and o_t = S_t q_t is compared
    with the fp64 oracle."""
    rng = np.random.default_rng(13)
    T, dk, dv, L, W = 7, 3, 2, 3, 3
    d = _frac_inputs(rng, T, dk, dv, L, W)
    F = {n: _F(x) for n, x in d.items()}
    m = L - 1
    # anchor + residuals in Fractions (closed form of the chain)
    A, Bm = [], []
    for t in range(T):
        a = [sum(F["conv_w"][0, c, i] * (F["v"][0, t - i, 0, c] if t - i >= 0 else 0) for i in range(W)) for c in range(dv)]
        r = [F["v"][0, t, 0, c] - a[c] for c in range(dv)]
        k = F["k"][0, t, 0]
        g, b = F["gamma"][0, t, 0], F["beta"][0, t, 0]
        At = np.array([[g * ((1 if i == j else 0) - b * k[i] * k[j]) for j in range(dk)] for i in range(dk)], dtype=object)
        Bt = np.array([[b * F["v"][0, t, 0, c] * k[j] for j in range(dk)] for c in range(dv)], dtype=object)
        for l in range(m):
            r = [(1 - F["gain"][0, t, 0, l, c]) * r[c] for c in range(dv)]
            for c in range(dv):
                for j in range(dk):
                    Bt[c, j] += F["alpha"][0, t, 0, l] * r[c] * F["u"][0, t, 0, l, j]
        A.append(At)
        Bm.append(Bt)
    # recursive-doubling inclusive scan of the maps x -> x A + B
    pre = [(A[t], Bm[t]) for t in range(T)]
    step = 1
    while step < T:
        nxt = list(pre)
        for t in range(step, T):
            (A1, B1), (A2, B2) = pre[t - step], pre[t]
            nxt[t] = (A1.dot(A2), B1.dot(A2) + B2)
        pre = nxt
        step *= 2
    S0 = F["S0"][0, 0]
    o_exact = np.array([[float(x) for x in (S0.dot(pre[t][0]) + pre[t][1]).dot(F["q"][0, t, 0])] for t in range(T)])
    S_exact = np.array([[float(x) for x in row] for row in (S0.dot(pre[-1][0]) + pre[-1][1])])
    o, S = prism_seq(**d)
    np.testing.assert_allclose(o[0, :, 0], o_exact, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S[0, 0], S_exact, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- chunk form
@pytest.mark.parametrize("chunk", [1, 4, 16, 64])
def test_chunked_equals_sequential(chunk):
    """The chunkwise decomposition reaches the token recurrence exactly (up to
    rounding), for chunks that do and do not divide T, with S0 and ragged lengths."""
    rng = np.random.default_rng(14)
    d = rand_inputs(rng, B=2, T=83, H=2, dk=8, dv=6, L=4, s0=True, lengths=np.array([83, 50]))
    o, S = prism_seq(**d)
    oc, Sc = prism_chunked(**d, chunk=chunk)
    assert max_abs_rel_err(oc, o) < 1e-10
    assert max_abs_rel_err(Sc, S, slice_axes=(0, 1)) < 1e-10


def test_chunked_L1_is_gdn_chunk_form():
    rng = np.random.default_rng(15)
    d = rand_inputs(rng, B=1, T=40, H=3, L=1)
    oc, Sc = prism_chunked(**dict(d, u=None, alpha=None, gain=None), chunk=16)
    og, Sg = gdn_seq(d["q"], d["k"], d["v"], d["gamma"], d["beta"])
    assert max_abs_rel_err(oc, og) < 1e-10


# ---------------------------------------------------------------- structure
def test_linearity_in_v_and_S0():
    """o and S_final are jointly linear in (v, S0) with the other inputs fixed:
    the anchor, the chain and the write are linear in v, the update is linear in S."""
    rng = np.random.default_rng(16)
    d1 = rand_inputs(rng, T=21, s0=True)
    d2 = dict(d1, v=rng.standard_normal(d1["v"].shape), S0=rng.standard_normal(d1["S0"].shape))
    o1, S1 = prism_seq(**d1)
    o2, S2 = prism_seq(**d2)
    o3, S3 = prism_seq(**dict(d1, v=d1["v"] - 2.5 * d2["v"], S0=d1["S0"] - 2.5 * d2["S0"]))
    np.testing.assert_allclose(o3, o1 - 2.5 * o2, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(S3, S1 - 2.5 * S2, rtol=1e-11, atol=1e-11)


def test_split_invariance():
    """Running [0, T) equals running [0, T1) and then [T1, T) from the handed-over
    state.  The second run is given the last W-1 tokens of the first part as a
    convolution history whose own writes are switched off (gamma=1, beta=alpha=0)."""
    rng = np.random.default_rng(17)
    W = 4
    d = rand_inputs(rng, B=2, T=40, W=W, L=3, s0=True)
    o, S = prism_seq(**d)
    T1 = 17
    first = {n: (x[:, :T1] if n in ("q", "k", "v", "gamma", "beta", "u", "alpha", "gain") else x) for n, x in d.items()}
    o1, S1 = prism_seq(**first)
    h = T1 - (W - 1)
    second = {n: (x[:, h:].copy() if n in ("q", "k", "v", "gamma", "beta", "u", "alpha", "gain") else x) for n, x in d.items()}
    second["gamma"][:, : W - 1] = 1.0
    second["beta"][:, : W - 1] = 0.0
    second["alpha"][:, : W - 1] = 0.0
    second["S0"] = S1
    o2, S2 = prism_seq(**second)
    np.testing.assert_allclose(o1, o[:, :T1], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(o2[:, W - 1:], o[:, T1:], rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(S2, S, rtol=1e-11, atol=1e-11)


def test_masking_equals_truncation():
    """Right-padded rows: the valid outputs equal a run on the truncated row, the
    padded outputs are zero and the final state is the state after the last
    valid token."""
    rng = np.random.default_rng(18)
    lens = np.array([25, 9, 31])
    d = rand_inputs(rng, B=3, T=31, L=3, s0=True, lengths=lens)
    o, S = prism_seq(**d)
    for b, n in enumerate(lens):
        db = {x: (y[b:b + 1, :n] if x in ("q", "k", "v", "gamma", "beta", "u", "alpha", "gain") else y) for x, y in d.items()}
        db["S0"] = d["S0"][b:b + 1]
        db["lengths"] = None
        ob, Sb = prism_seq(**db)
        np.testing.assert_allclose(o[b:b + 1, :n], ob, rtol=1e-13, atol=1e-13)
        assert np.all(o[b, n:] == 0)
        np.testing.assert_allclose(S[b:b + 1], Sb, rtol=1e-13, atol=1e-13)


def test_max_abs_rel_err_metric():
    ref = np.zeros((2, 3, 2, 4))
    ref[0, :, 0] = 2.0
    ref[1, :, 1] = 10.0
    x = ref.copy()
    x[1, 0, 1, 0] += 0.5
    assert max_abs_rel_err(x, ref) == pytest.approx(0.05)
    x[0, 1, 1, 2] = 1e-3   # an all-zero slice uses the 1e-6 floor
    assert max_abs_rel_err(x, ref) == pytest.approx(1e3)


# ---------------------------------------------------------------- exact GELU chain (NEXT variant)
def test_gelu_matches_library():
    """The oracle's GELU is the exact erf form: torch's gelu(approximate='none') and the
    standard library's math.erf give the same numbers."""
    import math

    import torch

    x = np.linspace(-6, 6, 97)
    ours = __import__("oracle").gelu(x)
    ref = torch.nn.functional.gelu(torch.tensor(x, dtype=torch.float64), approximate="none").numpy()
    np.testing.assert_allclose(ours, ref, rtol=1e-14, atol=1e-15)
    for xi, oi in zip(x[::8], ours[::8]):
        assert abs(oi - 0.5 * xi * (1.0 + math.erf(xi / math.sqrt(2.0)))) < 1e-14


def test_gelu_chain_special_cases():
    """p = 0: GELU(0) = 0, nothing is removed, every r_l equals r_0.  A single step
    against a hand-evaluated GELU (math.erf), and the linear chain is unchanged."""
    import math

    rng = np.random.default_rng(20)
    d = rand_inputs(rng, L=4)
    r = residual_chain(d["v"], d["conv_w"], np.zeros_like(d["gain"]), chain="gelu")
    r0 = d["v"] - shortconv_anchor(d["v"], d["conv_w"])
    for l in range(3):
        np.testing.assert_array_equal(r[:, :, :, l], r0)
    v = np.array([[[[0.7, -1.3]]]])              # B=T=H=1, d_v=2
    w = np.zeros((1, 2, 1))                      # no anchor: r_0 = v
    p = np.array([[[[[2.0, 0.5]]]]])             # one step
    r1 = residual_chain(v, w, p, chain="gelu")[0, 0, 0, 0]
    for c in range(2):
        x = p[0, 0, 0, 0, c] * v[0, 0, 0, c]
        ref = v[0, 0, 0, c] - 0.5 * x * (1.0 + math.erf(x / math.sqrt(2.0)))
        assert abs(r1[c] - ref) < 1e-15
    np.testing.assert_array_equal(residual_chain(d["v"], d["conv_w"], d["gain"]),
                                  residual_chain(d["v"], d["conv_w"], d["gain"], chain="linear"))


@pytest.mark.parametrize("chunk", [4, 64])
def test_gelu_chain_chunked_equals_sequential(chunk):
    rng = np.random.default_rng(21)
    d = rand_inputs(rng, B=2, T=70, H=2, dk=8, dv=6, L=4, s0=True, lengths=np.array([70, 33]))
    o, S = prism_seq(**d, chain="gelu")
    oc, Sc = prism_chunked(**d, chunk=chunk, chain="gelu")
    assert max_abs_rel_err(oc, o) < 1e-10
    assert max_abs_rel_err(Sc, S, slice_axes=(0, 1)) < 1e-10


def test_gelu_chain_rank():
    rng = np.random.default_rng(22)
    d = rand_inputs(rng, B=1, T=5, H=1, dk=12, dv=12, L=5)
    dS = residual_write(d["v"], d["u"], d["alpha"], d["gain"], d["conv_w"], chain="gelu")
    for t in range(5):
        s = np.linalg.svd(dS[0, t, 0], compute_uv=False)
        assert int((s > 1e-10 * s[0]).sum()) == 4
