"""Gradients of the scan on the GPU (prism_scan_bwd, through the C ABI) against the
oracle's autograd gradients (oracle/prism_grad.py) on the same, already rounded
inputs.  fp32 arithmetic on both the fp32 and the bf16 inputs, so one bar: 2e-4
max-abs-relative per gradient tensor.
"""
import numpy as np
import pytest
import torch

from linear_attention_sequence_shortconv_b200 import synth
from oracle.prism_grad import prism_seq_grad

pytestmark = pytest.mark.gpu

TOL = 2e-4

CASES = {
    "fp32_d32_L3": (synth.Workload("a", B=2, T=37, H=2, d_k=32, d_v=32, L=3, chunk=16, W=4, dtype="fp32",
                                   lengths_lo=20, with_s0=True), "linear"),
    "fp32_d16_L4_gelu": (synth.Workload("b", B=1, T=25, H=2, d_k=16, d_v=16, L=4, chunk=16, W=2, dtype="fp32",
                                        with_s0=True), "gelu"),
    "bf16_d128_L4": (synth.Workload("c", B=1, T=70, H=2, d_k=128, d_v=128, L=4, chunk=64, W=4, with_s0=True),
                     "linear"),
    "fp32_d64_L1": (synth.Workload("d", B=2, T=40, H=1, d_k=64, d_v=64, L=1, chunk=16, W=4, dtype="fp32"), "linear"),
    "fp32_dk64_dv32_W1": (synth.Workload("e", B=1, T=30, H=3, d_k=64, d_v=32, L=2, chunk=16, W=1, dtype="fp32"),
                          "linear"),
}


# d_k = d_v in {64, 128} and L <= 4 take the chunked backward (64-token chunks):
# several chunks, a ragged last chunk, lengths ending mid-chunk, on a chunk edge, and
# sequences shorter than the ShortConv window behind a chunk start.
CHUNKED = {
    "chunked_bf16_d128_L4": (synth.Workload("f", B=2, T=200, H=2, d_k=128, d_v=128, L=4, chunk=64, W=4,
                                            lengths_lo=60, with_s0=True, seed=21), "linear"),
    "chunked_fp32_d64_L3_gelu": (synth.Workload("g", B=3, T=150, H=2, d_k=64, d_v=64, L=3, chunk=64, W=8,
                                                dtype="fp32", lengths_lo=1, with_s0=True, seed=22), "gelu"),
    "chunked_bf16_d64_L1": (synth.Workload("h", B=2, T=129, H=3, d_k=64, d_v=64, L=1, chunk=64, W=3,
                                           seed=23), "linear"),
    "chunked_fp32_d128_L2_W1": (synth.Workload("i", B=1, T=256, H=1, d_k=128, d_v=128, L=2, chunk=64, W=1,
                                               dtype="fp32", seed=24), "linear"),
    "chunked_bf16_d128_L3_gelu_edges": (synth.Workload("j", B=4, T=192, H=1, d_k=128, d_v=128, L=3, chunk=64,
                                                       W=4, lengths_lo=64, with_s0=True, seed=25), "gelu"),
}


def _run(w, chain, seed=5, lengths=None):
    import linear_attention_sequence_shortconv_b200 as prism

    inp = synth.make_inputs(w)
    if chain == "gelu":
        gg = torch.Generator().manual_seed(w.seed + 101)
        inp["gain"] = (1.5 * torch.randn(inp["gain"].shape, generator=gg)).to(inp["gain"].dtype)
    gen = torch.Generator().manual_seed(seed)
    dO = torch.randn((w.B, w.T, w.H, w.d_v), generator=gen).to(inp["v"].dtype)
    dSf = torch.randn((w.B, w.H, w.d_v, w.d_k), generator=gen)
    if lengths is not None:
        inp["lengths"] = torch.tensor(lengths, dtype=torch.int32)
    d = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}
    g = prism.scan_bwd(d["q"], d["k"], d["v"], d["gamma"], d["beta"], d["u"], d["alpha"], d["gain"], d["conv_w"],
                       dO.cuda(), L=w.L, S0=d["S0"], lengths=d["lengths"], dS_final=dSf.cuda(), chain=chain)
    torch.cuda.synchronize()
    return inp, dO, dSf, {n: t.cpu().numpy().astype(np.float64) for n, t in g.items()}


def _rel(x, ref):
    return float(np.abs(x - ref).max() / max(np.abs(ref).max(), 1e-6))


@pytest.mark.parametrize("name", list(CASES))
def test_backward_matches_oracle(name):
    w, chain = CASES[name]
    inp, dO, dSf, got = _run(w, chain)
    x = synth.to_float64_numpy(inp)
    if w.L == 1:
        x["u"] = x["alpha"] = x["gain"] = None
    ref = prism_seq_grad(**x, dO=dO.double().numpy(), dS_final=dSf.double().numpy(), chain=chain)
    for n, r in ref.items():
        assert n in got, n
        assert got[n].shape == r.shape, (n, got[n].shape, r.shape)
        assert _rel(got[n], r) <= TOL, (name, n, _rel(got[n], r))


def test_backward_is_deterministic():
    w, chain = CASES["bf16_d128_L4"]
    _, _, _, g1 = _run(w, chain)
    _, _, _, g2 = _run(w, chain)
    for n in g1:
        assert np.array_equal(g1[n], g2[n]), n


def test_backward_long_chain_full_width():
    """L = 16 (fifteen residual directions) at d = 128: the largest per-token reduction."""
    w = synth.Workload("long_chain", B=1, T=12, H=1, d_k=128, d_v=128, L=16, chunk=64, W=4, with_s0=True)
    inp, dO, dSf, got = _run(w, "linear")
    x = synth.to_float64_numpy(inp)
    ref = prism_seq_grad(**x, dO=dO.double().numpy(), dS_final=dSf.double().numpy())
    for n, r in ref.items():
        assert _rel(got[n], r) <= TOL, (n, _rel(got[n], r))


CHUNKED.update({
    # an empty row, one token, a chunk and one more, and shorter than one chunk
    "chunked_fp32_d64_L4_empty_rows": (synth.Workload("l", B=4, T=65, H=2, d_k=64, d_v=64, L=4, chunk=64, W=8,
                                                      dtype="fp32", with_s0=True, seed=28), "linear"),
    "chunked_bf16_d128_L2_T1": (synth.Workload("m", B=2, T=1, H=2, d_k=128, d_v=128, L=2, chunk=64, W=4,
                                               with_s0=True, seed=29), "gelu"),
    "chunked_bf16_d64_L3_T40": (synth.Workload("n", B=1, T=40, H=3, d_k=64, d_v=64, L=3, chunk=64, W=2,
                                               seed=30), "linear"),
})

# lengths on a chunk edge (64, 128), one token into a chunk (65), one short of it (127);
# an empty row (0), a single token (1)
EDGE_LENGTHS = {"chunked_bf16_d128_L3_gelu_edges": [64, 65, 127, 128],
                "chunked_fp32_d64_L4_empty_rows": [0, 1, 64, 65]}


@pytest.mark.parametrize("name", list(CHUNKED))
def test_chunked_backward_matches_oracle(name):
    w, chain = CHUNKED[name]
    inp, dO, dSf, got = _run(w, chain, lengths=EDGE_LENGTHS.get(name))
    x = synth.to_float64_numpy(inp)
    if w.L == 1:
        x["u"] = x["alpha"] = x["gain"] = None
    ref = prism_seq_grad(**x, dO=dO.double().numpy(), dS_final=dSf.double().numpy(), chain=chain)
    for n, r in ref.items():
        assert got[n].shape == r.shape, (n, got[n].shape, r.shape)
        assert _rel(got[n], r) <= TOL, (name, n, _rel(got[n], r))


def test_chunked_backward_strong_decay():
    """gamma around 0.3: dgamma comes out of gamma_t dgamma_t divided by gamma_t."""
    w = synth.Workload("k", B=1, T=130, H=2, d_k=64, d_v=64, L=3, chunk=64, W=4, dtype="fp32", with_s0=True,
                       seed=26)
    import linear_attention_sequence_shortconv_b200 as prism

    inp = synth.make_inputs(w)
    gg = torch.Generator().manual_seed(27)
    inp["gamma"] = torch.sigmoid(torch.randn(inp["gamma"].shape, generator=gg) - 1.0)
    gen = torch.Generator().manual_seed(5)
    dO = torch.randn((w.B, w.T, w.H, w.d_v), generator=gen)
    d = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}
    g = prism.scan_bwd(d["q"], d["k"], d["v"], d["gamma"], d["beta"], d["u"], d["alpha"], d["gain"], d["conv_w"],
                       dO.cuda(), L=w.L, S0=d["S0"], lengths=d["lengths"])
    torch.cuda.synchronize()
    x = synth.to_float64_numpy(inp)
    ref = prism_seq_grad(**x, dO=dO.double().numpy())
    for n, r in ref.items():
        assert _rel(g[n].cpu().numpy().astype(np.float64), r) <= TOL, (n,)


def test_full_size_lm_layer_sampled_chains():
    """The backward at the benchmarked size and launch configuration (130M-LM layer,
    B=16 T=2048 H=6 d=128 L=4, bf16), checked on two sampled (b, h) chains: each
    chain's gradients depend on that chain's inputs only, so the oracle (about 15 s a
    chain) runs on the chain alone.  dconv_w sums over the batch and is left to the
    smaller cases above (the oracle would need all 16 rows of a head, minutes)."""
    import linear_attention_sequence_shortconv_b200 as prism

    w = synth.WORKLOADS["lm_130m"].replace(with_s0=True)
    inp = synth.make_inputs(w)
    gen = torch.Generator().manual_seed(31)
    dO = torch.randn((w.B, w.T, w.H, w.d_v), generator=gen).to(torch.bfloat16)
    dSf = torch.randn((w.B, w.H, w.d_v, w.d_k), generator=gen)
    d = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}
    g = prism.scan_bwd(d["q"], d["k"], d["v"], d["gamma"], d["beta"], d["u"], d["alpha"], d["gain"], d["conv_w"],
                       dO.cuda(), L=w.L, S0=d["S0"], lengths=d["lengths"], dS_final=dSf.cuda())
    torch.cuda.synchronize()
    assert prism.stream_status() == 0
    got = {n: t.cpu().numpy().astype(np.float64) for n, t in g.items()}
    x = synth.to_float64_numpy(inp)
    dO64, dSf64 = dO.double().numpy(), dSf.double().numpy()

    def chain_inputs(bs, h):
        c = {n: x[n][bs][:, :, h:h + 1] for n in ("q", "k", "v", "gamma", "beta", "u", "alpha", "gain")}
        c["conv_w"] = x["conv_w"][h:h + 1]
        c["S0"] = x["S0"][bs][:, h:h + 1]
        c["lengths"] = None if x["lengths"] is None else x["lengths"][bs]
        return c

    for b, h in ((0, 0), (15, 5)):
        ref = prism_seq_grad(**chain_inputs(slice(b, b + 1), h), dO=dO64[b:b + 1, :, h:h + 1],
                             dS_final=dSf64[b:b + 1, h:h + 1])
        for n, r in ref.items():
            if n == "conv_w":
                continue
            mine = got[n][b:b + 1, h:h + 1] if n == "S0" else got[n][b:b + 1, :, h:h + 1]
            assert _rel(mine, r) <= TOL, ((b, h), n, _rel(mine, r))
