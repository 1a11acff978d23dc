"""Shared test plumbing: run the CUDA path and the oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

from linear_attention_sequence_shortconv_b200 import synth

TOL = {"bf16": 2e-2, "fp32": 1e-4}   # max-abs-relative error bars of the method's evaluation


def gpu_run(inp: dict, w: synth.Workload, device="cuda:0", want_state=True, chunk=None, chain="linear"):
    import linear_attention_sequence_shortconv_b200 as prism

    d = {n: (t.to(device) if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}
    o, S = prism.scan_fwd(d["q"], d["k"], d["v"], d["gamma"], d["beta"], d["u"], d["alpha"], d["gain"],
                          d["conv_w"], L=w.L, chunk=chunk or w.chunk, S0=d["S0"], lengths=d["lengths"],
                          want_state=want_state, chain=chain)
    torch.cuda.synchronize()
    return o.float().cpu().numpy(), (S.cpu().numpy() if S is not None else None)


def oracle_run(inp: dict, w: synth.Workload, bh=None, chain="linear"):
    """fp64 oracle; ``bh`` = list of (b, h) pairs to evaluate (sampling), else all."""
    from oracle import prism_seq

    x = synth.to_float64_numpy(inp)
    if w.L == 1:
        x["u"] = x["alpha"] = x["gain"] = None
    if bh is None:
        return prism_seq(**x, chain=chain)
    outs, states = [], []
    for b, h in bh:
        sl = {}
        for n, a in x.items():
            if a is None:
                sl[n] = None
            elif n == "conv_w":
                sl[n] = a[h:h + 1]
            elif n == "S0":
                sl[n] = a[b:b + 1, h:h + 1]
            elif n == "lengths":
                sl[n] = a[b:b + 1]
            else:
                sl[n] = a[b:b + 1, :, h:h + 1]
        o, S = prism_seq(**sl, chain=chain)
        outs.append(o[0, :, 0])
        states.append(S[0, 0])
    return outs, states


def rel_err(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(x - ref).max() / max(np.abs(ref).max(), 1e-6))
