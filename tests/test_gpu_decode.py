"""The one-token decode step on the GPU (through the C ABI) against the oracle's
decode step, and the split-invariance of the scan: prefill with prism_scan_fwd,
then decode the rest of the sequence token by token, and compare with one
prism_scan_fwd over the whole sequence.
"""
import numpy as np
import pytest
import torch

from linear_attention_sequence_shortconv_b200 import synth
from oracle import max_abs_rel_err, prism_decode_step, prism_seq
from tests.helpers import TOL, gpu_run

pytestmark = pytest.mark.gpu

TOK = ("q", "k", "v", "gamma", "beta", "u", "alpha", "gain")


def _token(inp, t, device=None):
    out = {}
    for n in TOK:
        x = inp[n]
        out[n] = None if x is None else x[:, t].contiguous()
        if device is not None and out[n] is not None:
            out[n] = out[n].to(device)
    return out


def _gpu_decode(tok, conv_w, hist, S, L, chain="linear"):
    import linear_attention_sequence_shortconv_b200 as prism

    return prism.decode_step(tok["q"], tok["k"], tok["v"], tok["gamma"], tok["beta"], tok["u"], tok["alpha"],
                             tok["gain"], conv_w, hist, S, L=L, chain=chain)


def _f64(x):
    return None if x is None else x.double().cpu().numpy()


CASES = [
    synth.Workload("lm", B=3, T=2, H=4, d_k=128, d_v=128, L=4, chunk=64, W=4),
    synth.Workload("fp32", B=2, T=2, H=3, d_k=32, d_v=32, L=16, chunk=16, W=8, dtype="fp32"),
    synth.Workload("mixed", B=2, T=2, H=2, d_k=64, d_v=16, L=1, chunk=16, W=1, dtype="fp32"),
    synth.Workload("d16", B=5, T=2, H=1, d_k=16, d_v=128, L=3, chunk=16, W=2),
]


@pytest.mark.parametrize("chain", ["linear", "gelu"])
@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_decode_step_matches_oracle(w, chain):
    inp = synth.make_inputs(w)
    g = torch.Generator().manual_seed(w.seed + 7)
    dt = inp["v"].dtype
    S = 0.3 * torch.randn((w.B, w.H, w.d_v, w.d_k), generator=g)
    hist = torch.randn((w.B, w.H, w.W - 1, w.d_v), generator=g).to(dt) if w.W > 1 else None
    tok = _token(inp, 1)
    o_ref, S_ref, h_ref = prism_decode_step(**{n: _f64(x) for n, x in tok.items()}, conv_w=_f64(inp["conv_w"]),
                                            conv_state=_f64(hist), S=_f64(S), chain=chain)
    dev = "cuda:0"
    S_d = S.to(dev)
    hist_d = hist.to(dev) if hist is not None else None
    o = _gpu_decode(_token(inp, 1, dev), inp["conv_w"].to(dev), hist_d, S_d, w.L, chain)
    torch.cuda.synchronize()
    tol = TOL[w.dtype]
    assert max_abs_rel_err(o.float().cpu().numpy()[:, None], o_ref[:, None]) <= tol
    assert max_abs_rel_err(S_d.cpu().numpy(), S_ref, slice_axes=(0, 1)) <= tol
    if hist is not None:  # the history is a shift of exact values
        assert np.array_equal(hist_d.double().cpu().numpy(), h_ref)


@pytest.mark.parametrize("name,T1", [("lm_130m", 130), ("recsys", 64), ("fp32", 37)])
def test_prefill_then_decode_equals_one_scan(name, T1):
    """Split invariance on the GPU: prism_scan_fwd over [0, T1), then decode steps
    over [T1, T) from its S_final and the last W-1 values of v, against one
    prism_scan_fwd over [0, T) and against the oracle."""
    w = {
        "lm_130m": synth.WORKLOADS["lm_130m"].replace(B=2, T=160, H=2, with_s0=True),
        "recsys": synth.WORKLOADS["recsys"].replace(B=3, T=80, lengths_lo=None),
        "fp32": synth.Workload("fp32", B=2, T=50, H=2, d_k=32, d_v=32, L=5, chunk=16, W=3, dtype="fp32"),
    }[name]
    inp = synth.make_inputs(w)
    dev = "cuda:0"
    o_full, S_full = gpu_run(inp, w)
    pre = {n: (x[:, :T1].contiguous() if n in TOK else x) for n, x in inp.items()}
    o_pre, S = gpu_run(pre, w.replace(T=T1))
    S = torch.from_numpy(S).to(dev)
    hist = inp["v"][:, T1 - (w.W - 1):T1].permute(0, 2, 1, 3).contiguous().to(dev)
    conv_w = inp["conv_w"].to(dev)
    outs = []
    for t in range(T1, w.T):
        outs.append(_gpu_decode(_token(inp, t, dev), conv_w, hist, S, w.L).float().cpu().numpy())
    torch.cuda.synchronize()
    o_dec = np.stack(outs, axis=1)
    o_cat = np.concatenate([o_pre, o_dec], axis=1)
    S_dec = S.cpu().numpy()
    x = synth.to_float64_numpy(inp)
    o_ref, S_ref = prism_seq(**x)
    tol = TOL[w.dtype]
    assert max_abs_rel_err(o_cat, o_ref) <= tol
    assert max_abs_rel_err(S_dec, S_ref, slice_axes=(0, 1)) <= tol
    assert max_abs_rel_err(o_cat, o_full) <= tol
    assert max_abs_rel_err(S_dec, S_full, slice_axes=(0, 1)) <= tol


def test_decode_from_zero_state_reproduces_the_scan():
    """Decoding every token from S = 0 and a zero history is the scan itself."""
    w = synth.Workload("dec", B=2, T=24, H=3, d_k=64, d_v=64, L=4, chunk=16, W=4, dtype="fp32")
    inp = synth.make_inputs(w)
    dev = "cuda:0"
    o_scan, S_scan = gpu_run(inp, w)
    S = torch.zeros((w.B, w.H, w.d_v, w.d_k), device=dev)
    hist = torch.zeros((w.B, w.H, w.W - 1, w.d_v), device=dev)
    conv_w = inp["conv_w"].to(dev)
    o = np.stack([_gpu_decode(_token(inp, t, dev), conv_w, hist, S, w.L).cpu().numpy() for t in range(w.T)], axis=1)
    assert max_abs_rel_err(o, o_scan) <= TOL["fp32"]
    assert max_abs_rel_err(S.cpu().numpy(), S_scan, slice_axes=(0, 1)) <= TOL["fp32"]
