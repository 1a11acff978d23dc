"""The ShortConv history argument of prism_scan_fwd_ex: a sequence scanned in two
calls, the second from the first's final state and with the first's last W - 1 rows of
v as conv_state, against the oracle's scan of the whole sequence (ICML 2026 PRISM
write-up, 消除 Token 间串行: the anchor reads the last few tokens; 核心迭代形式 for the
state carry), at the forward bars (2e-2 bf16 per (batch, head) slice, 1e-4 fp32)."""
import numpy as np
import pytest
import torch

import linear_attention_sequence_shortconv_b200 as prism
from linear_attention_sequence_shortconv_b200 import synth
from oracle import max_abs_rel_err, prism_seq

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "gamma", "beta", "u", "alpha", "gain")


def _two_calls(w, T1, chain="linear"):
    inp = synth.make_inputs(w)
    d = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}
    W = w.W
    part = lambda s, e: {n: (d[n][:, s:e].contiguous() if d[n] is not None else None) for n in NAMES}
    a, b = part(0, T1), part(T1, w.T)
    o1, S1 = prism.scan_fwd(*(a[n] for n in NAMES), d["conv_w"], L=w.L, chunk=w.chunk, S0=d["S0"], chain=chain)
    hist = d["v"][:, T1 - (W - 1):T1].permute(0, 2, 1, 3).contiguous()  # [B, H, W-1, d_v]
    o2, S2 = prism.scan_fwd(*(b[n] for n in NAMES), d["conv_w"], L=w.L, chunk=w.chunk, S0=S1, chain=chain,
                            conv_state=hist)
    torch.cuda.synchronize()
    assert prism.stream_status() == 0
    o_ref, S_ref = prism_seq(**synth.to_float64_numpy(inp), chain=chain)
    o = torch.cat([o1, o2], 1).float().cpu().numpy()
    return o, S2.cpu().numpy(), o_ref, S_ref


def test_split_bf16_tensor_core_path():
    """d = 128, L = 4, W = 4 (tensor-core scan), split at a token that is not a chunk
    boundary."""
    w = synth.WORKLOADS["lm_130m"].replace(B=2, T=700, H=2, with_s0=True, seed=51)
    o, S, o_ref, S_ref = _two_calls(w, 333)
    assert max_abs_rel_err(o, o_ref) <= 2e-2
    assert max_abs_rel_err(S, S_ref, slice_axes=(0, 1)) <= 2e-2


def test_split_bf16_wide_window():
    """d = 64, W = 8 (the wide-window residual-write variant), L = 2, split inside a chunk."""
    w = synth.Workload("cs_w8", B=2, T=300, H=2, d_k=64, d_v=64, L=2, chunk=64, W=8, with_s0=True, seed=52)
    o, S, o_ref, S_ref = _two_calls(w, 129)
    assert max_abs_rel_err(o, o_ref) <= 2e-2
    assert max_abs_rel_err(S, S_ref, slice_axes=(0, 1)) <= 2e-2


@pytest.mark.parametrize("d", [64, 128])
def test_split_fp32_gelu(d):
    """fp32, exact GELU chain: the fp32 chunk-form kernel (d = 64) and the token-by-token
    kernel (d = 128)."""
    w = synth.Workload("cs_fp32", B=3, T=150, H=2, d_k=d, d_v=d, L=3, chunk=64, W=4, dtype="fp32",
                       with_s0=True, seed=53)
    o, S, o_ref, S_ref = _two_calls(w, 61, chain="gelu")
    assert max_abs_rel_err(o, o_ref) <= 1e-4
    assert max_abs_rel_err(S, S_ref, slice_axes=(0, 1)) <= 1e-4


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_zero_history_equals_no_history(dtype):
    """conv_state of zeros gives bit for bit what no conv_state gives."""
    w = synth.Workload("cs_zero", B=2, T=200, H=2, d_k=64, d_v=64, L=3, chunk=64, W=4, dtype=dtype, seed=54)
    d = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in synth.make_inputs(w).items()}
    args = [d[n] for n in NAMES] + [d["conv_w"]]
    o0, S0 = prism.scan_fwd(*args, L=w.L, chunk=w.chunk)
    z = torch.zeros((w.B, w.H, w.W - 1, w.d_v), dtype=d["v"].dtype, device="cuda")
    o1, S1 = prism.scan_fwd(*args, L=w.L, chunk=w.chunk, conv_state=z)
    torch.cuda.synchronize()
    assert torch.equal(o0, o1) and torch.equal(S0, S1)
