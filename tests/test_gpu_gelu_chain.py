"""The exact GELU residual chain, r <- r - GELU(p * r) (gist.science PRISM
explainer, 2.2 Input-Anchored Loop Unrolling), on every CUDA path against the
fp64 oracle run with chain="gelu".

The predictor p may take any real value, so besides the synthetic gain in
(0, 1) one case draws it from N(0, 1.5^2): negative and >1 gains, where GELU's
curvature matters most.
"""
import numpy as np
import pytest
import torch

from linear_attention_sequence_shortconv_b200 import synth
from oracle import max_abs_rel_err, residual_chain
from tests.helpers import TOL, gpu_run, oracle_run

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS

CASES = {
    # tcgen05 chunk kernel (bf16, d = 128, L = 4, W = 4), ragged tail and S0
    "lm_130m": W["lm_130m"].replace(B=2, T=200, H=3, with_s0=True),
    # tcgen05 chunk kernel at d = 64 with right-padded rows
    "recsys": W["recsys"].replace(B=5, T=260, lengths_lo=30),
    # token-by-token kernel: fp32 at d = 128
    "lm_fp32": W["lm_130m"].replace(B=1, T=130, H=2, dtype="fp32"),
    # fp32 chunk-form kernel: d = 64, several chunks and ragged rows
    "recsys_fp32": W["recsys"].replace(B=3, T=200, lengths_lo=30, dtype="fp32"),
    # tcgen05 chunk kernel with seven residual directions (three U slots)
    "long_ctx": W["long_ctx"].replace(T=150, H=2),
    # three U slots in the two-halves scan (11 chunks), W = 8, ragged rows
    "many_dirs_ragged": synth.Workload("mdr", B=4, T=700, H=2, d_k=64, d_v=64, L=6, chunk=64, W=8,
                                       lengths_lo=100, with_s0=True),
    "d32_L16_W8": synth.Workload("d32", B=2, T=97, H=3, d_k=32, d_v=32, L=16, chunk=32, W=8),
}


def _wide_gain(inp, w):
    g = torch.Generator().manual_seed(w.seed + 101)
    p = 1.5 * torch.randn(inp["gain"].shape, generator=g)
    inp = dict(inp)
    inp["gain"] = p.to(inp["gain"].dtype)
    return inp


@pytest.mark.parametrize("name", list(CASES))
def test_gelu_chain_parity(name):
    w = CASES[name]
    inp = synth.make_inputs(w)
    o, S = gpu_run(inp, w, chain="gelu")
    o_ref, S_ref = oracle_run(inp, w, chain="gelu")
    tol = TOL[w.dtype]
    assert max_abs_rel_err(o, o_ref) <= tol, name
    assert max_abs_rel_err(S, S_ref, slice_axes=(0, 1)) <= tol, name
    if w.lengths_lo is not None:
        for b, n in enumerate(inp["lengths"].numpy()):
            assert np.all(o[b, n:] == 0)


@pytest.mark.parametrize("name", ["lm_130m", "lm_fp32", "recsys_fp32"])
def test_gelu_chain_parity_wide_predictor(name):
    w = CASES[name]
    inp = _wide_gain(synth.make_inputs(w), w)
    o, S = gpu_run(inp, w, chain="gelu")
    o_ref, S_ref = oracle_run(inp, w, chain="gelu")
    tol = TOL[w.dtype]
    assert max_abs_rel_err(o, o_ref) <= tol
    assert max_abs_rel_err(S, S_ref, slice_axes=(0, 1)) <= tol


def test_gelu_chain_differs_from_linear_chain():
    """The flag reaches the kernel: same inputs, the two chains give different outputs."""
    w = CASES["lm_130m"]
    inp = synth.make_inputs(w)
    o_lin, _ = gpu_run(inp, w, chain="linear")
    o_gelu, _ = gpu_run(inp, w, chain="gelu")
    o_ref_lin, _ = oracle_run(inp, w, chain="linear")
    o_ref_gelu, _ = oracle_run(inp, w, chain="gelu")
    gap = max_abs_rel_err(o_ref_lin, o_ref_gelu)
    assert gap > 10 * TOL["bf16"]
    assert max_abs_rel_err(o_lin, o_gelu) > 0.5 * gap


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_gelu_prologue_kernel(dtype):
    import linear_attention_sequence_shortconv_b200 as prism

    w = synth.Workload("pro", B=3, T=70, H=2, d_k=64, d_v=64, L=5, chunk=64, lengths_lo=10, dtype=dtype)
    inp = _wide_gain(synth.make_inputs(w), w)
    d = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}
    rho = prism.prologue_fwd(d["v"], d["alpha"], d["gain"], d["conv_w"], L=w.L, lengths=d["lengths"],
                             chain="gelu")
    torch.cuda.synchronize()
    x = synth.to_float64_numpy(inp)
    ref = x["alpha"][..., None] * residual_chain(x["v"], x["conv_w"], x["gain"], chain="gelu")
    valid = np.arange(w.T)[None, :] < x["lengths"][:, None]
    ref = np.where(valid[:, :, None, None, None], ref, 0.0)
    got = rho.cpu().numpy()
    assert np.abs(got - ref).max() <= 1e-5 * max(np.abs(ref).max(), 1.0)
