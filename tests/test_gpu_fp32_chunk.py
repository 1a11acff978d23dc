"""The fp32 build of the chunk form (fp32 I/O, d_k = d_v in {16, 32, 64}): the same
decomposition the tensor-core scan runs, every product in fp32 FMAs, against the fp64
oracle at the fp32 bar (1e-4 max-abs-relative per (batch, head) slice).

The chunkwise scan is the ICML 2026 PRISM write-up's 消除 Token 间串行; the algebra
(A, T = (I + A)^{-1}, U', W', Delta, the masked output products and the state carry)
follows from the technical summary 2.1 (the update is affine in S with input-only
coefficients).  The cases cover the tiny fp32 configuration, every chunk length, several
chunks with a ragged tail, right-padded and empty rows, an initial state, the ShortConv
history input, W = 1 and W = 8, L = 1 (plain gated delta) and L = 16, both residual
chains, and strongly decaying gates.
"""
import numpy as np
import pytest
import torch

import linear_attention_sequence_shortconv_b200 as prism
from linear_attention_sequence_shortconv_b200 import synth
from oracle import max_abs_rel_err, prism_seq
from tests.helpers import gpu_run, oracle_run

pytestmark = pytest.mark.gpu

TOL = 1e-4

CASES = {
    "tiny": synth.WORKLOADS["tiny_fp32"],
    "d16_c16_s0": synth.Workload("a", B=2, T=75, H=2, d_k=16, d_v=16, L=3, chunk=16, W=4, dtype="fp32",
                                 with_s0=True, seed=61),
    "d32_c32_L16_W8": synth.Workload("b", B=2, T=97, H=3, d_k=32, d_v=32, L=16, chunk=32, W=8, dtype="fp32",
                                     seed=62),
    "d64_c64_ragged": synth.Workload("c", B=4, T=200, H=2, d_k=64, d_v=64, L=4, chunk=64, W=4, dtype="fp32",
                                     lengths_lo=1, with_s0=True, seed=63),
    "d64_c16_L1": synth.Workload("d", B=2, T=90, H=2, d_k=64, d_v=64, L=1, chunk=16, W=4, dtype="fp32", seed=64),
    "d32_c64_W1": synth.Workload("e", B=3, T=130, H=1, d_k=32, d_v=32, L=3, chunk=64, W=1, dtype="fp32",
                                 lengths_lo=0, seed=65),
}


@pytest.mark.parametrize("chain", ["linear", "gelu"])
@pytest.mark.parametrize("name", list(CASES))
def test_fp32_chunk_form_parity(name, chain):
    w = CASES[name]
    assert prism.lib().prism_scan_fwd_uses_tensor_cores(w.d_k, w.d_v, w.L, w.W, w.chunk, 1) == 0
    inp = synth.make_inputs(w)
    if w.lengths_lo is not None:
        inp["lengths"][0] = 0  # an empty row beside ragged ones
    o, S = gpu_run(inp, w, chain=chain)
    o_ref, S_ref = oracle_run(inp, w, chain=chain)
    assert prism.stream_status() == 0
    e_o = max_abs_rel_err(o, o_ref)
    e_s = max_abs_rel_err(S, S_ref, slice_axes=(0, 1))
    assert e_o <= TOL and e_s <= TOL, (name, chain, e_o, e_s)
    if w.lengths_lo is not None:  # outputs past a row's length are zero
        ln = inp["lengths"].numpy()
        for b in range(w.B):
            assert not np.any(o[b, ln[b]:])


def test_fp32_chunk_lengths_agree():
    """The result does not depend on the chunk length beyond rounding."""
    w = synth.Workload("f", B=2, T=150, H=2, d_k=32, d_v=32, L=4, chunk=16, W=4, dtype="fp32", with_s0=True,
                       seed=66)
    inp = synth.make_inputs(w)
    outs = [gpu_run(inp, w, chunk=c) for c in (16, 32, 64)]
    for o, S in outs[1:]:
        assert max_abs_rel_err(o, outs[0][0]) <= TOL
        assert max_abs_rel_err(S, outs[0][1], slice_axes=(0, 1)) <= TOL


def test_fp32_chunk_strongly_decaying_gates():
    """Gates near zero: every decay factor is e^{c_t - c_i} with i <= t, so nothing
    overflows and the chunk form stays at the fp32 bar."""
    w = synth.Workload("g", B=2, T=140, H=2, d_k=64, d_v=64, L=3, chunk=64, W=4, dtype="fp32", seed=67)
    inp = synth.make_inputs(w)
    gen = torch.Generator().manual_seed(5)
    inp["gamma"] = (0.02 + 0.1 * torch.rand(inp["gamma"].shape, generator=gen)).float()
    o, S = gpu_run(inp, w)
    o_ref, S_ref = oracle_run(inp, w)
    assert max_abs_rel_err(o, o_ref) <= TOL
    assert max_abs_rel_err(S, S_ref, slice_axes=(0, 1)) <= TOL


def test_fp32_chunk_bitwise_deterministic():
    w = CASES["d64_c64_ragged"]
    inp = synth.make_inputs(w)
    a = gpu_run(inp, w)
    b = gpu_run(inp, w)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_fp32_chunk_conv_state_split():
    """Two calls with the ShortConv history and the state handed over equal one call."""
    w = synth.Workload("h", B=2, T=160, H=2, d_k=64, d_v=64, L=3, chunk=64, W=4, dtype="fp32", with_s0=True,
                       seed=68)
    inp = synth.make_inputs(w)
    d = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}
    cut = 71
    args = lambda sl: [d[n][:, sl].contiguous() for n in ("q", "k", "v", "gamma", "beta", "u", "alpha", "gain")]
    o1, S1 = prism.scan_fwd(*args(slice(0, cut)), d["conv_w"], L=w.L, chunk=w.chunk, S0=d["S0"], chain="gelu")
    hist = d["v"][:, cut - (w.W - 1):cut].permute(0, 2, 1, 3).contiguous()
    o2, S2 = prism.scan_fwd(*args(slice(cut, w.T)), d["conv_w"], L=w.L, chunk=w.chunk, S0=S1, chain="gelu",
                            conv_state=hist)
    torch.cuda.synchronize()
    o = torch.cat([o1, o2], dim=1).cpu().numpy()
    x = synth.to_float64_numpy(inp)
    o_ref, S_ref = prism_seq(**x, chain="gelu")
    assert max_abs_rel_err(o, o_ref) <= TOL
    assert max_abs_rel_err(S2.cpu().numpy(), S_ref, slice_axes=(0, 1)) <= TOL


@pytest.mark.parametrize("T,chunk", [(1, 16), (15, 16), (16, 16), (17, 16), (33, 16), (1, 64), (63, 64), (65, 64)])
def test_fp32_chunk_boundary_lengths(T, chunk):
    """Sequences of one token, one short of a chunk, exactly one chunk, one past it, and two
    chunks plus one, with an initial state and the ShortConv window reaching before token 0."""
    w = synth.Workload("j", B=2, T=T, H=2, d_k=16, d_v=16, L=3, chunk=chunk, W=4, dtype="fp32", with_s0=True,
                       seed=90 + T)
    inp = synth.make_inputs(w)
    o, S = gpu_run(inp, w)
    o_ref, S_ref = oracle_run(inp, w)
    assert max_abs_rel_err(o, o_ref) <= TOL
    assert max_abs_rel_err(S, S_ref, slice_axes=(0, 1)) <= TOL
