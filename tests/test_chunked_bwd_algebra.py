"""The chunked backward's algebra, restated in fp64 numpy, against the oracle's autograd
gradients (CPU, no GPU).

The chunked backward of the library (records of a forward pass at 64-token chunk
boundaries, a reverse adjoint pass, then per-chunk products) rests on three facts
that autograd through the token loop does not state by itself:

* inside a chunk, S_t and the adjoint G_t = dL/dS_t are sums over the chunk's
  writes with decays D_{ti} = e^{c_t - c_i} from the boundary values S_n and H_n;
* the gradient products per token (S_t^T dO_t, gamma_t S_{t-1}^T G_t k_t,
  G_t^T x_{t,a}) are then masked, decayed chunk products;
* gamma_t dgamma_t = <H_n, S_{n+1}> + sum_{j >= t in the chunk} (q_j . dq_j - w_j)
  with w_j = <G_j, W_j>, which replaces the per-token Frobenius product
  <G_t, S_{t-1}>.

This module restates those formulas (with a small chunk, so that several chunks, a
ragged last chunk and the ShortConv halo across a chunk boundary all occur) and
checks every gradient against ``oracle.prism_grad.prism_seq_grad`` to 1e-10.  The
recurrence is the one of the ICML 2026 PRISM write-up (核心迭代形式 / 架构形式) and
the PRISM explainer (2.1-2.2).
"""
import math

import numpy as np
import pytest
from scipy.special import erf

from oracle.prism_grad import prism_seq_grad


def _gelu(x):
    return 0.5 * x * (1 + erf(x / math.sqrt(2)))


def _gelu_grad(x):
    return 0.5 * (1 + erf(x / math.sqrt(2))) + x * np.exp(-0.5 * x * x) / math.sqrt(2 * math.pi)


def chunked_grads(q, k, v, gamma, beta, u, alpha, gain, conv_w, dO, S0, lengths, dSf, chain, C):
    B, T, H, dk = k.shape
    dv, W, m = v.shape[-1], conv_w.shape[-1], u.shape[3]
    NC = (T + C - 1) // C
    g = {n: np.zeros(x.shape) for n, x in dict(q=q, k=k, v=v, gamma=gamma, beta=beta, u=u, alpha=alpha, gain=gain,
                                               conv_w=conv_w).items()}
    g["S0"] = np.zeros((B, H, dv, dk))
    for b in range(B):
        ln = T if lengths is None else int(lengths[b])
        ncb = (ln + C - 1) // C
        for h in range(H):
            w = conv_w[h]

            def resid(t):  # r_0 .. r_m of token t
                rs = [v[b, t, h] - sum(w[:, i] * v[b, t - i, h] for i in range(W) if t - i >= 0)]
                for l in range(m):
                    r = rs[-1]
                    rs.append((1 - gain[b, t, h, l]) * r if chain == "linear" else r - _gelu(gain[b, t, h, l] * r))
                return rs

            # forward records: S at chunk boundaries, psi_t = v_t - gamma_t S_{t-1} k_t
            S = S0[b, h].copy()
            st = np.zeros((NC + 1, dv, dk))
            st[0] = S
            psi = np.zeros((T, dv))
            for t in range(ln):
                sk = S @ k[b, t, h]
                psi[t] = v[b, t, h] - gamma[b, t, h] * sk
                S = gamma[b, t, h] * (S - beta[b, t, h] * np.outer(sk, k[b, t, h])) + \
                    beta[b, t, h] * np.outer(v[b, t, h], k[b, t, h])
                rs = resid(t)
                for l in range(m):
                    S = S + alpha[b, t, h, l] * np.outer(rs[l + 1], u[b, t, h, l])
                if (t + 1) % C == 0 or t + 1 == ln:
                    st[(t + C) // C] = S
            # adjoint records: G_t k_t, G_t u_l, H_n, <H_n, S_{n+1}>, dS0
            G = dSf[b, h].copy()
            Hn, hs = np.zeros((NC, dv, dk)), np.zeros(NC)
            gk, gu = np.zeros((T, dv)), np.zeros((T, m, dv))
            if ncb:
                Hn[ncb - 1], hs[ncb - 1] = G, np.sum(G * st[ncb])
            for t in range(ln - 1, -1, -1):
                G = G + np.outer(dO[b, t, h], q[b, t, h])
                gk[t] = G @ k[b, t, h]
                for l in range(m):
                    gu[t, l] = G @ u[b, t, h, l]
                G = gamma[b, t, h] * (G - beta[b, t, h] * np.outer(gk[t], k[b, t, h]))
                if t % C == 0 and t > 0:
                    Hn[t // C - 1], hs[t // C - 1] = G, np.sum(G * st[t // C])
            g["S0"][b, h] = G
            # per chunk: masked, decayed chunk products
            for n in range(ncb):
                t0 = n * C
                nt = min(C, ln - t0)
                ii = np.arange(t0, t0 + nt)
                c = np.cumsum(np.log(gamma[b, ii, h]))
                be = beta[b, ii, h]
                Q, K, DO, GK = q[b, ii, h], k[b, ii, h], dO[b, ii, h], gk[ii]
                R = [resid(t) for t in ii]
                X = [be[:, None] * psi[ii]] + [alpha[b, ii, h, l][:, None] * np.array([r[l + 1] for r in R])
                                               for l in range(m)]
                Y = [K] + [u[b, ii, h, l] for l in range(m)]
                Dm = np.tril(np.exp(c[:, None] - c[None, :]))
                Dms = Dm - np.diag(np.diag(Dm))
                dq = np.exp(c)[:, None] * (DO @ st[n])
                F = np.exp(c)[:, None] * (GK @ st[n])
                Gx = []
                for a in range(m + 1):
                    Ma, Na = Dm * (DO @ X[a].T), Dms * (GK @ X[a].T)
                    dq += Ma @ Y[a]
                    F += Na @ Y[a]
                    Gx.append(np.exp(c[-1] - c)[:, None] * (X[a] @ Hn[n]) + Ma.T @ Q - (be[:, None] * Na).T @ K)
                wt = be * np.sum(v[b, ii, h] * GK, 1) + sum(np.sum(X[l + 1] * gu[ii, l], 1) for l in range(m))
                gdg = hs[n] + np.cumsum((np.sum(Q * dq, 1) - wt)[::-1])[::-1]
                g["q"][b, ii, h] = dq
                g["k"][b, ii, h] = Gx[0] - be[:, None] * F
                g["beta"][b, ii, h] = np.sum(GK * psi[ii], 1)
                g["gamma"][b, ii, h] = gdg / gamma[b, ii, h]
                for l in range(m):
                    g["u"][b, ii, h, l] = Gx[l + 1]
                    g["alpha"][b, ii, h, l] = np.sum(np.array([r[l + 1] for r in R]) * gu[ii, l], 1)
            # the residual chain backwards, then the ShortConv transpose (crosses chunks)
            dr0 = np.zeros((T, dv))
            for t in range(ln):
                rs, dr = resid(t), np.zeros(dv)
                for l in range(m, 0, -1):
                    dr = dr + alpha[b, t, h, l - 1] * gu[t, l - 1]
                    gl, rp = gain[b, t, h, l - 1], rs[l - 1]
                    slope = np.ones(dv) if chain == "linear" else _gelu_grad(gl * rp)
                    g["gain"][b, t, h, l - 1] = -rp * slope * dr
                    dr = dr * (1 - gl * slope)
                dr0[t] = dr
            for t in range(ln):
                g["v"][b, t, h] = beta[b, t, h] * gk[t] + dr0[t] - sum(w[:, i] * dr0[t + i] for i in range(W)
                                                                       if t + i < ln)
                for i in range(W):
                    if t - i >= 0:
                        g["conv_w"][h][:, i] -= dr0[t] * v[b, t - i, h]
    return g


@pytest.mark.parametrize("chain,L,W,C,T,lengths", [
    ("linear", 3, 3, 8, 21, [21, 12]),
    ("gelu", 3, 4, 8, 21, [21, 8]),
    ("linear", 1, 2, 4, 13, None),
    ("linear", 4, 5, 4, 30, [30, 1]),
    ("gelu", 2, 1, 8, 16, [16, 0]),
])
def test_chunked_formulas_match_autograd(chain, L, W, C, T, lengths):
    rng = np.random.default_rng(L * 100 + W * 10 + C)
    B, H, dk, dv, m = 2, 2, 6, 5, L - 1
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    x = dict(q=0.5 * rng.standard_normal((B, T, H, dk)), k=k, v=rng.standard_normal((B, T, H, dv)),
             gamma=rng.uniform(0.5, 1.0, (B, T, H)), beta=rng.uniform(0.1, 1.0, (B, T, H)),
             u=0.3 * rng.standard_normal((B, T, H, m, dk)), alpha=rng.uniform(0.0, 0.5, (B, T, H, m)),
             gain=0.5 * rng.standard_normal((B, T, H, m, dv)), conv_w=0.3 * rng.standard_normal((H, dv, W)))
    dO = rng.standard_normal((B, T, H, dv))
    S0 = 0.3 * rng.standard_normal((B, H, dv, dk))
    dSf = rng.standard_normal((B, H, dv, dk))
    lens = None if lengths is None else np.array(lengths)
    ref = prism_seq_grad(**{n: (None if (m == 0 and n in ("u", "alpha", "gain")) else a) for n, a in x.items()},
                         dO=dO, S0=S0, lengths=lens, dS_final=dSf, chain=chain)
    got = chunked_grads(**x, dO=dO, S0=S0, lengths=lens, dSf=dSf, chain=chain, C=C)
    for n, r in ref.items():
        err = np.abs(got[n] - r).max() / max(np.abs(r).max(), 1e-12)
        assert err < 1e-10, (n, err)


def chunk_boundary_passes(q, k, v, gamma, beta, u, alpha, gain, conv_w, dO, S0, dSf, chain, C):
    """The two boundary passes in chunk (GEMM) form, one sequence (B = H = 1, full
    length): the forward carry S_n -> S_{n+1} through T = (I + A)^{-1}, and the
    adjoint carry H_n -> H_{n-1} through T^T, with the per-token records psi and gk
    they produce.  Returns (states [NC+1], psi [T], Hn [NC], gk [T])."""
    T_, dk = k.shape[1], k.shape[-1]
    dv, W, m = v.shape[-1], conv_w.shape[-1], u.shape[3]
    NC = (T_ + C - 1) // C
    w = conv_w[0]

    def resid(t):
        rs = [v[0, t, 0] - sum(w[:, i] * v[0, t - i, 0] for i in range(W) if t - i >= 0)]
        for l in range(m):
            r = rs[-1]
            rs.append((1 - gain[0, t, 0, l]) * r if chain == "linear" else r - _gelu(gain[0, t, 0, l] * r))
        return rs

    chunks = []
    for n in range(NC):
        ii = np.arange(n * C, min(T_, n * C + C))
        c = np.cumsum(np.log(gamma[0, ii, 0]))
        Dm = np.tril(np.exp(c[:, None] - c[None, :]))
        Dms = Dm - np.diag(np.diag(Dm))
        K, Q, V, be = k[0, ii, 0], q[0, ii, 0], v[0, ii, 0], beta[0, ii, 0]
        R = [resid(t) for t in ii]
        Rt = [alpha[0, ii, 0, l][:, None] * np.array([r[l + 1] for r in R]) for l in range(m)]
        U = [u[0, ii, 0, l] for l in range(m)]
        A = be[:, None] * Dms * (K @ K.T)
        Tinv = np.linalg.inv(np.eye(len(ii)) + A)
        chunks.append((ii, c, Dm, Dms, K, Q, V, be, Rt, U, Tinv))
    # forward carry: X = diag(beta)(V - P'), Delta = T X, psi = V - P' - Kp_0 Delta
    S = S0[0, 0].copy()
    states, psi = [S.copy()], np.zeros((T_, dv))
    for ii, c, Dm, Dms, K, Q, V, be, Rt, U, Tinv in chunks:
        Pp = np.exp(c)[:, None] * (K @ S.T) + sum((Dms * (K @ U[l].T)) @ Rt[l] for l in range(m))
        Delta = Tinv @ (be[:, None] * (V - Pp))
        psi[ii] = V - Pp - (Dms * (K @ K.T)) @ Delta
        dec = np.exp(c[-1] - c)[:, None]
        S = np.exp(c[-1]) * S + (dec * Delta).T @ K + sum((dec * Rt[l]).T @ U[l] for l in range(m))
        states.append(S.copy())
    # adjoint carry: Y = diag(e^{c_C - c}) K H^T + (D o Q K^T)^T dO, gk = T^T Y
    H = dSf[0, 0].copy()
    Hn, gk = [None] * NC, np.zeros((T_, dv))
    for n in range(NC - 1, -1, -1):
        ii, c, Dm, Dms, K, Q, V, be, Rt, U, Tinv = chunks[n]
        Hn[n] = H.copy()
        DO = dO[0, ii, 0]
        Y = np.exp(c[-1] - c)[:, None] * (K @ H.T) + (Dm * (Q @ K.T)).T @ DO
        G = Tinv.T @ Y
        gk[ii] = G
        E = be[:, None] * G
        H = np.exp(c[-1]) * H + DO.T @ (np.exp(c)[:, None] * Q) - E.T @ (np.exp(c)[:, None] * K)
    return states, psi, Hn, gk, H


@pytest.mark.parametrize("chain,L,C,T", [("linear", 3, 8, 29), ("gelu", 4, 4, 16), ("linear", 1, 8, 8)])
def test_chunk_form_boundary_passes_equal_token_records(chain, L, C, T):
    """The boundary passes in chunk form (serial over chunks, GEMM-shaped) reproduce
    the token-by-token records: the states at every chunk boundary, psi, the adjoint
    H_n at every chunk end, gk, and dS0."""
    rng = np.random.default_rng(7 + L + C)
    dk, dv, W, m = 6, 5, 3, L - 1
    k = rng.standard_normal((1, T, 1, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    x = dict(q=0.5 * rng.standard_normal((1, T, 1, dk)), k=k, v=rng.standard_normal((1, T, 1, dv)),
             gamma=rng.uniform(0.5, 1.0, (1, T, 1)), beta=rng.uniform(0.1, 1.0, (1, T, 1)),
             u=0.3 * rng.standard_normal((1, T, 1, m, dk)), alpha=rng.uniform(0.0, 0.5, (1, T, 1, m)),
             gain=0.5 * rng.standard_normal((1, T, 1, m, dv)), conv_w=0.3 * rng.standard_normal((1, dv, W)))
    dO = rng.standard_normal((1, T, 1, dv))
    S0 = 0.3 * rng.standard_normal((1, 1, dv, dk))
    dSf = rng.standard_normal((1, 1, dv, dk))
    states, psi, Hn, gk, dS0 = chunk_boundary_passes(**x, dO=dO, S0=S0, dSf=dSf, chain=chain, C=C)
    # the token-by-token records, written out directly
    NC = (T + C - 1) // C
    S, ref_states, ref_psi = S0[0, 0].copy(), [S0[0, 0].copy()], np.zeros((T, dv))
    w = x["conv_w"][0]
    for t in range(T):
        rs = [x["v"][0, t, 0] - sum(w[:, i] * x["v"][0, t - i, 0] for i in range(W) if t - i >= 0)]
        for l in range(m):
            r = rs[-1]
            g = x["gain"][0, t, 0, l]
            rs.append((1 - g) * r if chain == "linear" else r - _gelu(g * r))
        kt, gm, bt = x["k"][0, t, 0], x["gamma"][0, t, 0], x["beta"][0, t, 0]
        sk = S @ kt
        ref_psi[t] = x["v"][0, t, 0] - gm * sk
        S = gm * (S - bt * np.outer(sk, kt)) + bt * np.outer(x["v"][0, t, 0], kt)
        for l in range(m):
            S = S + x["alpha"][0, t, 0, l] * np.outer(rs[l + 1], x["u"][0, t, 0, l])
        if (t + 1) % C == 0 or t + 1 == T:
            ref_states.append(S.copy())
    G, ref_Hn, ref_gk = dSf[0, 0].copy(), [None] * NC, np.zeros((T, dv))
    ref_Hn[NC - 1] = G.copy()
    for t in range(T - 1, -1, -1):
        G = G + np.outer(dO[0, t, 0], x["q"][0, t, 0])
        kt = x["k"][0, t, 0]
        ref_gk[t] = G @ kt
        G = x["gamma"][0, t, 0] * (G - x["beta"][0, t, 0] * np.outer(ref_gk[t], kt))
        if t % C == 0 and t > 0:
            ref_Hn[t // C - 1] = G.copy()
    for a, b in zip(states, ref_states):
        assert np.abs(a - b).max() < 1e-10
    assert np.abs(psi - ref_psi).max() < 1e-10
    for a, b in zip(Hn, ref_Hn):
        assert np.abs(a - b).max() < 1e-10
    assert np.abs(gk - ref_gk).max() < 1e-10
    assert np.abs(dS0 - G).max() < 1e-10
