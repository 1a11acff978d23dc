"""Gradients of the PRISM scan for the CPU oracle (PyTorch, fp64, CPU).

TEST INFRASTRUCTURE, like prism_oracle.py: only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py`` may import it; the library never does.

The forward is the token loop of ``prism_seq`` restated with torch operations
(ICML 2026 PRISM write-up, 核心迭代形式 / 架构形式; PRISM explainer 2.1-2.2):

    a_t = sum_i w[:, i] v_{t-i};  r_0 = v_t - a_t;  r_l = chain step(r_{l-1}, g_l)
    S_t = gamma_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T + sum_l alpha_l r_l u_l^T
    o_t = S_t q_t          (padded steps t >= lengths[b]: S unchanged, o_t = 0)

and the gradients of L = <o, dO> + <S_final, dS_final> with respect to every
input are taken by reverse-mode automatic differentiation of that loop (the
definition of the gradient; no hand-derived formula is involved).  Pinned in
tests/test_oracle_grad.py against the numpy ``prism_seq`` (forward) and central
finite differences (gradients).
"""
from __future__ import annotations

import math

import numpy as np
import torch

INPUTS = ("q", "k", "v", "gamma", "beta", "u", "alpha", "gain", "conv_w", "S0")


def _gelu(x):
    return 0.5 * x * (1.0 + torch.erf(x / math.sqrt(2.0)))


def prism_seq_torch(q, k, v, gamma, beta, u, alpha, gain, conv_w, S0=None, lengths=None, chain="linear"):
    """The token loop on torch fp64 tensors (differentiable).  Shapes as prism_seq;
    u/alpha/gain may be None when L = 1.  Returns (o [B,T,H,d_v], S_final)."""
    if chain not in ("linear", "gelu"):
        raise ValueError(f"unknown chain {chain!r}")
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    W = conv_w.shape[-1]
    m = 0 if u is None else u.shape[3]
    S = torch.zeros(B, H, dv, dk, dtype=torch.float64) if S0 is None else S0
    lens = [T] * B if lengths is None else [int(x) for x in lengths]
    outs = []
    for t in range(T):
        a = torch.zeros(B, H, dv, dtype=torch.float64)
        for i in range(W):
            if t - i >= 0:
                a = a + conv_w[None, :, :, i] * v[:, t - i]
        r = v[:, t] - a
        write = beta[:, t][..., None, None] * v[:, t][..., :, None] * k[:, t][..., None, :]
        for l in range(m):
            g = gain[:, t, :, l]
            r = (1.0 - g) * r if chain == "linear" else r - _gelu(g * r)
            write = write + alpha[:, t, :, l][..., None, None] * r[..., :, None] * u[:, t, :, l][..., None, :]
        kt = k[:, t]
        Sk = torch.einsum("bhcj,bhj->bhc", S, kt)
        S_new = gamma[:, t][..., None, None] * (S - beta[:, t][..., None, None] * Sk[..., :, None] * kt[..., None, :]) + write
        valid = torch.tensor([t < n for n in lens], dtype=torch.bool)[:, None, None, None]
        S = torch.where(valid, S_new, S)
        o_t = torch.einsum("bhcj,bhj->bhc", S, q[:, t])
        outs.append(torch.where(valid[..., 0], o_t, torch.zeros_like(o_t)))
    return torch.stack(outs, dim=1), S


def prism_seq_grad(q, k, v, gamma, beta, u, alpha, gain, conv_w, dO, S0=None, lengths=None, dS_final=None,
                   chain="linear"):
    """Gradients of L = <o, dO> + <S_final, dS_final> (numpy in, numpy fp64 out).

    Returns a dict with keys of ``INPUTS`` (``u``, ``alpha``, ``gain`` absent when
    L = 1; ``S0`` the gradient with respect to the initial state, present always).
    """
    def t64(x):
        return None if x is None else torch.tensor(np.asarray(x, dtype=np.float64), requires_grad=True)

    B, T, H, dk = np.asarray(k).shape
    dv = np.asarray(v).shape[-1]
    args = {n: t64(x) for n, x in dict(q=q, k=k, v=v, gamma=gamma, beta=beta, u=u, alpha=alpha, gain=gain,
                                       conv_w=conv_w).items()}
    if args["u"] is not None and args["u"].shape[3] == 0:
        args["u"] = args["alpha"] = args["gain"] = None
    S0t = t64(S0 if S0 is not None else np.zeros((B, H, dv, dk)))
    o, S = prism_seq_torch(**args, S0=S0t, lengths=lengths, chain=chain)
    loss = (o * torch.tensor(np.asarray(dO, dtype=np.float64))).sum()
    if dS_final is not None:
        loss = loss + (S * torch.tensor(np.asarray(dS_final, dtype=np.float64))).sum()
    named = [(n, x) for n, x in args.items() if x is not None] + [("S0", S0t)]
    grads = torch.autograd.grad(loss, [x for _, x in named], allow_unused=True)
    out = {}
    for (n, x), g in zip(named, grads):
        out[n] = np.zeros(tuple(x.shape)) if g is None else g.detach().numpy()
    return out
