"""Seeded synthetic inputs for the PRISM sequence-mixer scan.

This module only draws random numbers and rounds them to the run dtype. It holds
none of the method's arithmetic, and both the CUDA path (through the tests and
the bench) and the CPU oracle consume what it returns.

Recipe (one CPU ``torch.Generator`` seeded per workload, fixed draw order
q, k, v, gamma, beta, u, alpha, gain, conv_w, lengths; everything is drawn in
fp32 and then rounded to the run dtype before anything consumes it):

* q, k ~ N(0, 1), then L2-normalised over d_k (the caller of a gated-delta layer
  normalises q and k; the mixer itself applies no 1/sqrt(d) scale);
* v ~ N(0, 1);
* gamma = sigmoid(N(3, 0.5))   (decay gate, mostly near 0.95);
* beta  = sigmoid(N(0, 1))     (delta-rule step size);
* u_l ~ N(0, 1/d_k)            (residual-write directions, l = 1 .. L-1);
* alpha = sigmoid(N(0, 1))     (residual step sizes);
* gain  = sigmoid(N(0, 1))     (per-channel preconditioner gains in (0, 1));
* conv_w ~ N(0, 1/W)           (ShortConv taps, kept in fp32);
* lengths ~ U{lo .. T}         (only for right-padded variable-length batches).

gamma, beta and alpha are returned as fp32 tensors that hold values already
rounded to the run dtype.  The shapes follow the token-major layout of the
C ABI: q, k [B,T,H,d_k]; v [B,T,H,d_v]; gamma, beta [B,T,H]; u [B,T,H,L-1,d_k];
alpha [B,T,H,L-1]; gain [B,T,H,L-1,d_v]; conv_w [H,d_v,W]; S0 [B,H,d_v,d_k].
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One named problem shape of the PRISM mixer scan."""

    name: str
    B: int
    T: int
    H: int
    d_k: int
    d_v: int
    L: int
    chunk: int
    W: int = 4
    dtype: str = "bf16"            # "bf16" or "fp32": dtype of q, k, v, u, gain and o
    lengths_lo: Optional[int] = None  # right-padded batch: lengths ~ U{lengths_lo .. T}
    with_s0: bool = False
    seed: int = 0

    @property
    def m(self) -> int:
        return self.L - 1

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five problem shapes of the method's evaluation: a tiny fp32 parity case, the
# L=1 gated-DeltaNet special case, a recommendation-shaped batch of right-padded
# user sequences, one layer of a 130M-parameter language model (hidden 768 as
# 6 heads of 128), and one long-context sequence.
WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", B=1, T=64, H=1, d_k=16, d_v=16, L=2, chunk=16, dtype="fp32"),
    "gdn_l1": Workload("gdn_l1", B=4, T=1024, H=4, d_k=64, d_v=64, L=1, chunk=64),
    "recsys": Workload("recsys", B=128, T=1024, H=2, d_k=64, d_v=64, L=4, chunk=64, lengths_lo=200),
    "lm_130m": Workload("lm_130m", B=16, T=2048, H=6, d_k=128, d_v=128, L=4, chunk=64),
    "long_ctx": Workload("long_ctx", B=1, T=65536, H=8, d_k=128, d_v=128, L=8, chunk=64),
}


def _round(x: torch.Tensor, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return x.to(torch.bfloat16)
    if dtype == "fp32":
        return x.to(torch.float32)
    raise ValueError(f"unknown dtype {dtype!r}")


def _round_f32(x: torch.Tensor, dtype: str) -> torch.Tensor:
    """Round to the run dtype but keep the fp32 container (gates, step sizes)."""
    return _round(x, dtype).to(torch.float32)


def make_inputs(w: Workload, device: str = "cpu") -> dict:
    """Draw the inputs of workload ``w``; returns a dict of torch tensors on ``device``."""
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    B, T, H, dk, dv, m, W = w.B, w.T, w.H, w.d_k, w.d_v, w.m, w.W
    f32 = torch.float32

    def randn(*shape, mean=0.0, std=1.0):
        x = torch.randn(*shape, generator=g, dtype=f32)
        if std != 1.0:
            x.mul_(std)
        if mean != 0.0:
            x.add_(mean)
        return x

    q = randn(B, T, H, dk)
    q = q / q.norm(dim=-1, keepdim=True)
    k = randn(B, T, H, dk)
    k = k / k.norm(dim=-1, keepdim=True)
    v = randn(B, T, H, dv)
    gamma = torch.sigmoid(randn(B, T, H, mean=3.0, std=0.5))
    beta = torch.sigmoid(randn(B, T, H))
    u = randn(B, T, H, m, dk, std=dk ** -0.5)
    alpha = torch.sigmoid(randn(B, T, H, m))
    gain = torch.sigmoid(randn(B, T, H, m, dv))
    conv_w = randn(H, dv, W, std=W ** -0.5)
    if w.lengths_lo is not None:
        lengths = torch.randint(w.lengths_lo, T + 1, (B,), generator=g, dtype=torch.int32)
    else:
        lengths = None
    S0 = randn(B, H, dv, dk, std=0.1) if w.with_s0 else None

    out = {
        "q": _round(q, w.dtype), "k": _round(k, w.dtype), "v": _round(v, w.dtype),
        "gamma": _round_f32(gamma, w.dtype), "beta": _round_f32(beta, w.dtype),
        "u": _round(u, w.dtype), "alpha": _round_f32(alpha, w.dtype),
        "gain": _round(gain, w.dtype), "conv_w": conv_w.contiguous(),
        "S0": S0, "lengths": lengths,
    }
    if device != "cpu":
        out = {n: (t.to(device) if isinstance(t, torch.Tensor) else t) for n, t in out.items()}
    return out


def to_float64_numpy(inputs: dict) -> dict:
    """Exact fp64 numpy copies of the inputs (what the CPU oracle consumes)."""
    res = {}
    for n, t in inputs.items():
        if t is None:
            res[n] = None
        elif n == "lengths":
            res[n] = t.detach().cpu().numpy().astype("int64")
        else:
            res[n] = t.detach().cpu().to(torch.float64).numpy()
    return res
