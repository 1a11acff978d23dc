"""CPU oracle for the PRISM sequence-mixer scan (NumPy, fp64).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import or run this module.  The library
(``linear_attention_sequence_shortconv_b200``) never calls it, shares no code
with it, and fails loudly when its CUDA extension is missing.

Sources (web pages on PRISM, cited by title and section):

* [blog]    "ICML 2026 | 当线性注意力学会"写入前思考"：并行化的多步记忆写入"
            (Tencent Ads / Peking University write-up of PRISM).
* [summary] "PRISM: Parallel Residual Iterative Sequence Model", technical summary
            of arXiv 2602.10796 (sections 2.1 and 2.2).
* [poster]  "PRISM: Parallel Residual Iterative Sequence Model", ICML 2026 poster
            abstract.

What is computed (the reading of the pages used throughout this repository):
for every batch row b and head h, with state S in R^{d_v x d_k} (S0 or zeros),

    a_t     = sum_{i=0}^{W-1} w[h,:,i] * v_{t-i}          (ShortConv anchor, v_{<0}=0)
    r_{t,0} = v_t - a_t                                    (anchor residual)
    r_{t,l} = (1 - g_{t,l}) * r_{t,l-1},  l = 1..L-1        (linearised residual chain)
    S_t     = gamma_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
              + sum_{l=1}^{L-1} alpha_{t,l} r_{t,l} u_{t,l}^T
    o_t     = S_t q_t                                      (post-update readout)

for t < lengths[b]; padded steps leave S unchanged and write o_t = 0.  L = 1 is
the gated delta rule.  Readings taken where the pages are silent or garbled:
the anchor is a depthwise causal convolution over v whose taps include the
current token; the gain g is a per-channel value in (0, 1) supplied by the
caller (the GELU of [summary] sec. 2.2 is absorbed into it, as [blog] "消除 Step
间串行" states); the written vector is r (not the decrement); gamma decays the
old state only; there is no 1/sqrt(d) scale on q.

Parity pins (all in tests/test_oracle_*.py): L=1 against the separately written
gated-delta recurrence ``gdn_seq``; exact recall of the delta rule; the
chunkwise form ``prism_chunked`` against the token loop; the rank of the
residual write; the zero-state and frozen-state special cases; the anchor
against a library FIR filter; an exact rational evaluation of the affine form
S_t = S_{t-1} A_t + B_t; linearity; split invariance; masking against
truncation; and a hand-worked two-token example under tests/golden/.  The
one-token decode step ``prism_decode_step`` is pinned to the same hand-worked
example, to exact recall, and to the sequence form (token-by-token decoding
and the continuation of a prefix).
"""
from __future__ import annotations

from typing import Optional

import numpy as np

__all__ = [
    "shortconv_anchor",
    "residual_chain",
    "gelu",
    "residual_write",
    "affine_maps",
    "prism_seq",
    "gdn_seq",
    "prism_chunked",
    "prism_decode_step",
    "max_abs_rel_err",
]


def _f64(x):
    return None if x is None else np.asarray(x, dtype=np.float64)


def _valid_mask(B: int, T: int, lengths) -> np.ndarray:
    """valid[b, t] is True for the real (unpadded) steps of row b."""
    if lengths is None:
        return np.ones((B, T), dtype=bool)
    lengths = np.asarray(lengths).reshape(B)
    return np.arange(T)[None, :] < lengths[:, None]


def shortconv_anchor(v, conv_w) -> np.ndarray:
    """ShortConv local anchor a_t ([blog] "消除 Token 间串行": a short convolution of
    the input stands in for the global state; [summary] sec. 2.2 stage 1: the
    anchor approximates S_{t-1} k_t from local history; [blog] "混合架构是必然":
    the window covers the last 3-4 tokens).

    Depthwise and causal: a[b,t,h,c] = sum_i conv_w[h,c,i] * v[b,t-i,h,c], with
    v before the start of each sequence taken as zero.

    v: [B,T,H,d_v]; conv_w: [H,d_v,W].  Returns a: [B,T,H,d_v].
    """
    v = _f64(v)
    conv_w = _f64(conv_w)
    T = v.shape[1]
    W = conv_w.shape[-1]
    a = np.zeros_like(v)
    for i in range(min(W, T)):
        a[:, i:] += conv_w[None, None, :, :, i] * v[:, : T - i]
    return a


def gelu(x):
    """GELU(x) = x * Phi(x) = 0.5 x (1 + erf(x / sqrt(2))), the exact (erf) form."""
    from scipy.special import erf

    x = _f64(x)
    return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))


def residual_chain(v, conv_w, gain, chain: str = "linear") -> np.ndarray:
    """Residuals r_{t,1..L-1} of the residual chain.

    [summary] sec. 2.2: the residual is reduced greedily step by step starting
    from the anchor residual, r^{(l+1)} = r^{(l)} - delta^{(l)} with
    delta^{(l)} = GELU(p^{(l)} * r^{(l)}).

    chain = "linear" (the path the library runs by default): [blog] "消除 Step
    间串行": with the nonlinearity absorbed into the preconditioner the chain is
    an element-wise linear recurrence, r_l = (1 - g_l) * r_{l-1}, g the
    per-channel gain.  chain = "gelu": the exact step above with p = gain,
    r_l = r_{l-1} - GELU(g_l * r_{l-1}).  Both start at r_0 = v - a and are taken
    one step at a time (the linear closed form is a test).

    gain: [B,T,H,m,d_v] with m = L-1.  Returns r: [B,T,H,m,d_v].
    """
    if chain not in ("linear", "gelu"):
        raise ValueError(f"unknown chain {chain!r}")
    v = _f64(v)
    gain = _f64(gain)
    m = gain.shape[3]
    r = v - shortconv_anchor(v, conv_w)
    out = np.empty(gain.shape, dtype=np.float64)
    for l in range(m):
        g = gain[:, :, :, l, :]
        r = (1.0 - g) * r if chain == "linear" else r - gelu(g * r)
        out[:, :, :, l, :] = r
    return out


def residual_write(v, u, alpha, gain, conv_w, chain: str = "linear") -> np.ndarray:
    """Per-token residual write dS_res,t = sum_l alpha_{t,l} r_{t,l} u_{t,l}^T
    ([blog] "核心迭代形式" and "架构形式": the write is the GDN write plus a
    low-rank correction).  Returns [B,T,H,d_v,d_k]."""
    r = residual_chain(v, conv_w, gain, chain)
    u = _f64(u)
    alpha = _f64(alpha)
    return np.einsum("bthl,bthlc,bthlj->bthcj", alpha, r, u)


def affine_maps(k, v, gamma, beta, u, alpha, gain, conv_w, lengths=None, chain: str = "linear"):
    """The pair (A_t, B_t) of the state update S_t = S_{t-1} A_t + B_t
    ([summary] sec. 2.1: forgetting A_t is the rank-1 gated-delta transition,
    all expressiveness sits in the injection B_t; [blog] "背景": this linear form
    with input-only A_t, B_t is what makes a parallel scan possible).

    A_t = gamma_t (I - beta_t k_t k_t^T)           [B,T,H,d_k,d_k]
    B_t = beta_t v_t k_t^T + dS_res,t              [B,T,H,d_v,d_k]
    Padded steps get A_t = I and B_t = 0.
    """
    k = _f64(k)
    v = _f64(v)
    gamma = _f64(gamma)
    beta = _f64(beta)
    B, T, H, dk = k.shape
    eye = np.eye(dk)
    A = gamma[..., None, None] * (eye - beta[..., None, None] * k[..., :, None] * k[..., None, :])
    Bt = beta[..., None, None] * v[..., :, None] * k[..., None, :]
    if u is not None and np.asarray(u).shape[3] > 0:
        Bt = Bt + residual_write(v, u, alpha, gain, conv_w, chain)
    valid = _valid_mask(B, T, lengths)[:, :, None, None, None]
    A = np.where(valid, A, eye)
    Bt = np.where(valid, Bt, 0.0)
    return A, Bt


def prism_seq(q, k, v, gamma, beta, u, alpha, gain, conv_w, S0=None, lengths=None, chain: str = "linear"):
    """Token-by-token PRISM scan (the definition in the module docstring).

    Shapes (token-major): q, k [B,T,H,d_k]; v [B,T,H,d_v]; gamma, beta [B,T,H];
    u [B,T,H,m,d_k]; alpha [B,T,H,m]; gain [B,T,H,m,d_v]; conv_w [H,d_v,W];
    S0 [B,H,d_v,d_k] or None; lengths [B] or None.  m = L-1 may be 0 (then u,
    alpha and gain may be None).

    Returns (o [B,T,H,d_v], S_final [B,H,d_v,d_k]), fp64.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    gamma, beta = _f64(gamma), _f64(beta)
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    m = 0 if u is None else np.asarray(u).shape[3]
    if m > 0:
        u, alpha = _f64(u), _f64(alpha)
        r = residual_chain(v, conv_w, gain, chain)
    S = np.zeros((B, H, dv, dk)) if S0 is None else _f64(S0).copy()
    o = np.zeros((B, T, H, dv))
    valid = _valid_mask(B, T, lengths)
    for t in range(T):
        kt, qt, vt = k[:, t], q[:, t], v[:, t]
        bt = beta[:, t][..., None, None]
        gt = gamma[:, t][..., None, None]
        write = bt * vt[..., :, None] * kt[..., None, :]
        for l in range(m):
            write = write + alpha[:, t, :, l][..., None, None] * r[:, t, :, l][..., :, None] * u[:, t, :, l][..., None, :]
        Sk = np.einsum("bhcj,bhj->bhc", S, kt)
        S_new = gt * (S - bt * Sk[..., :, None] * kt[..., None, :]) + write
        ok = valid[:, t][:, None, None, None]
        S = np.where(ok, S_new, S)
        o[:, t] = np.where(valid[:, t][:, None, None], np.einsum("bhcj,bhj->bhc", S, qt), 0.0)
    return o, S


def prism_decode_step(q, k, v, gamma, beta, u, alpha, gain, conv_w, conv_state, S, chain: str = "linear"):
    """One recurrent step of the scan (the O(1)-state inference form of the same
    recurrence: [blog] "背景" / "Rank-1 写入瓶颈", a linear-attention model keeps a
    fixed-size state and updates it once per token).

    The ShortConv history that the sequence form reads from v_{t-1..t-W+1} is
    carried explicitly: conv_state [B,H,W-1,d_v] holds v_{t-W+1}, ..., v_{t-1}
    (oldest first; zeros before the start of a sequence).

    q, k [B,H,d_k]; v [B,H,d_v]; gamma, beta [B,H]; u [B,H,m,d_k] (or None when
    m = 0); alpha [B,H,m]; gain [B,H,m,d_v]; conv_w [H,d_v,W]; S [B,H,d_v,d_k].
    Returns (o [B,H,d_v], S_new, conv_state_new), fp64.
    """
    if chain not in ("linear", "gelu"):
        raise ValueError(f"unknown chain {chain!r}")
    q, k, v = _f64(q), _f64(k), _f64(v)
    gamma, beta, S = _f64(gamma), _f64(beta), _f64(S)
    w = _f64(conv_w)
    W = w.shape[2]
    hist = _f64(conv_state) if W > 1 else np.zeros(v.shape[:2] + (0, v.shape[2]))
    a = w[None, :, :, 0] * v
    for i in range(1, W):
        a = a + w[None, :, :, i] * hist[:, :, W - 1 - i]
    r = v - a
    bt = beta[..., None, None]
    write = bt * v[..., :, None] * k[..., None, :]
    m = 0 if u is None else np.asarray(u).shape[2]
    if m > 0:
        u, alpha, gain = _f64(u), _f64(alpha), _f64(gain)
        for l in range(m):
            g = gain[:, :, l]
            r = (1.0 - g) * r if chain == "linear" else r - gelu(g * r)
            write = write + alpha[:, :, l][..., None, None] * r[..., :, None] * u[:, :, l][..., None, :]
    Sk = np.einsum("bhcj,bhj->bhc", S, k)
    S_new = gamma[..., None, None] * (S - bt * Sk[..., :, None] * k[..., None, :]) + write
    o = np.einsum("bhcj,bhj->bhc", S_new, q)
    hist_new = np.concatenate([hist[:, :, 1:], v[:, :, None]], axis=2) if W > 1 else hist
    return o, S_new, hist_new


def gdn_seq(q, k, v, gamma, beta, S0=None, lengths=None):
    """Plain gated delta rule, written separately from ``prism_seq`` in its
    error-correcting form: decay, predict, correct, read.

        S <- gamma_t S;  e = v_t - S k_t;  S <- S + beta_t e k_t^T;  o_t = S q_t

    ([blog] "架构形式": PRISM with L = 1 is exactly GDN; [summary] sec. 2.1: the
    forgetting path is kept identical to Gated DeltaNet.)
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    gamma, beta = _f64(gamma), _f64(beta)
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    valid = _valid_mask(B, T, lengths)
    S = np.zeros((B, H, dv, dk)) if S0 is None else _f64(S0).copy()
    o = np.zeros((B, T, H, dv))
    for b in range(B):
        for h in range(H):
            s = S[b, h]
            for t in range(T):
                if not valid[b, t]:
                    continue
                s = gamma[b, t, h] * s
                e = v[b, t, h] - s @ k[b, t, h]
                s = s + beta[b, t, h] * np.outer(e, k[b, t, h])
                o[b, t, h] = s @ q[b, t, h]
            S[b, h] = s
    return o, S


def prism_chunked(q, k, v, gamma, beta, u, alpha, gain, conv_w, chunk, S0=None, lengths=None, chain: str = "linear"):
    """Chunkwise-parallel form of the same scan, fp64 (the decomposition the
    tensor-core path uses; the chunkwise scan is how the method keeps GDN-class
    throughput, [blog] "消除 Token 间串行").

    Within a chunk, with S_n the state before its first token,
    b_t = prod_{j<=t} gamma_j (in-chunk), D[t,i] = b_t / b_i, rho_{i,l} = alpha r:
      A[t,i]        = beta_t D[t,i] k_t.k_i                  (i < t)
      Bku[t,(i,l)]  = beta_t D[t,i] k_t.u_{i,l}              (i < t)
      T             = (I + A)^{-1}
      Delta         = T (diag(beta) V - Bku P - diag(beta b) K S_n^T)
      O             = diag(b) Q S_n^T + (M<= . D . Q K^T) Delta + (M<= . D . Q U^T) P
      S_{n+1}       = b_C S_n + Delta^T diag(b_C/b) K + P^T diag(b_C/b) U
    where Delta stacks delta_t = beta_t (v_t - gamma_t S_{t-1} k_t) and P stacks
    rho.  Padded steps are exact no-ops (gamma=1, beta=alpha=0) and read o=0.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    gamma, beta = _f64(gamma).copy(), _f64(beta).copy()
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    m = 0 if u is None else np.asarray(u).shape[3]
    valid = _valid_mask(B, T, lengths)
    gamma = np.where(valid[:, :, None], gamma, 1.0)
    beta = np.where(valid[:, :, None], beta, 0.0)
    if m > 0:
        u = _f64(u)
        alpha = np.where(valid[:, :, None, None], _f64(alpha), 0.0)
        rho = alpha[..., None] * residual_chain(v, conv_w, gain, chain)  # [B,T,H,m,dv]
    S = np.zeros((B, H, dv, dk)) if S0 is None else _f64(S0).copy()
    o = np.zeros((B, T, H, dv))
    # move heads next to batch: [B,H,T,...]
    qh, kh, vh = (x.transpose(0, 2, 1, 3) for x in (q, k, v))
    gh, bh = gamma.transpose(0, 2, 1), beta.transpose(0, 2, 1)
    if m > 0:
        uh = u.transpose(0, 2, 1, 3, 4)       # [B,H,T,m,dk]
        ph = rho.transpose(0, 2, 1, 3, 4)     # [B,H,T,m,dv]
    for s in range(0, T, chunk):
        e = min(s + chunk, T)
        n = e - s
        Qc, Kc, Vc = qh[:, :, s:e], kh[:, :, s:e], vh[:, :, s:e]
        bc = np.cumprod(gh[:, :, s:e], axis=-1)                         # b_t
        beta_c = bh[:, :, s:e]
        D = bc[..., :, None] / bc[..., None, :]                         # [B,H,n,n]
        strict = np.tril(np.ones((n, n)), -1)
        incl = np.tril(np.ones((n, n)))
        A = beta_c[..., :, None] * D * np.einsum("bhtj,bhij->bhti", Kc, Kc) * strict
        Tm = np.linalg.inv(np.eye(n) + A)
        rhs = beta_c[..., None] * Vc - (beta_c * bc)[..., None] * np.einsum("bhtj,bhcj->bhtc", Kc, S)
        if m > 0:
            Uc = uh[:, :, s:e].reshape(B, H, n * m, dk)                # rows (i, l)
            Pc = ph[:, :, s:e].reshape(B, H, n * m, dv)
            Dm = np.repeat(D, m, axis=-1)                               # D[t,(i,l)] = D[t,i]
            Sm = np.repeat(strict, m, axis=-1)
            Im = np.repeat(incl, m, axis=-1)
            Bku = beta_c[..., :, None] * Dm * np.einsum("bhtj,bhrj->bhtr", Kc, Uc) * Sm
            rhs = rhs - np.einsum("bhtr,bhrc->bhtc", Bku, Pc)
        Delta = np.einsum("bhti,bhic->bhtc", Tm, rhs)
        Oc = bc[..., None] * np.einsum("bhtj,bhcj->bhtc", Qc, S)
        Oc = Oc + np.einsum("bhti,bhic->bhtc", D * incl * np.einsum("bhtj,bhij->bhti", Qc, Kc), Delta)
        if m > 0:
            QU = Dm * Im * np.einsum("bhtj,bhrj->bhtr", Qc, Uc)
            Oc = Oc + np.einsum("bhtr,bhrc->bhtc", QU, Pc)
        decay = bc[..., -1:] / bc                                       # b_C / b_i
        S_next = bc[..., -1][..., None, None] * S
        S_next = S_next + np.einsum("bhic,bhij->bhcj", decay[..., None] * Delta, Kc)
        if m > 0:
            S_next = S_next + np.einsum("bhrc,bhrj->bhcj", np.repeat(decay, m, axis=-1)[..., None] * Pc, Uc)
        S = S_next
        o[:, s:e] = Oc.transpose(0, 2, 1, 3)
    o = np.where(valid[:, :, None, None], o, 0.0)
    return o, S


def max_abs_rel_err(x, ref, slice_axes=None) -> float:
    """Max-abs-relative error: max|x - ref| / max(max|ref|, 1e-6) taken per
    (batch, head) slice and maximised over slices.  ``slice_axes`` names the
    axes that index slices (default: (0, 2) for [B,T,H,...] outputs)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if slice_axes is None:
        slice_axes = (0, 2) if x.ndim >= 3 else ()
    other = tuple(a for a in range(x.ndim) if a not in slice_axes)
    num = np.abs(x - ref).max(axis=other) if other else np.abs(x - ref)
    den = np.maximum(np.abs(ref).max(axis=other) if other else np.abs(ref), 1e-6)
    return float((num / den).max()) if np.size(num) else 0.0
