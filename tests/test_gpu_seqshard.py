"""Sequence sharding on the GPU, one process: prism_state_affine against an fp64
matmul, and the phases of seqshard.py run for every segment in turn on the library's
kernels (the all-gathers become lists), against the oracle's scan of the whole,
unsharded sequence at the forward bars (2e-2 bf16, 1e-4 fp32)."""
import numpy as np
import pytest
import torch

import linear_attention_sequence_shortconv_b200 as prism
from linear_attention_sequence_shortconv_b200 import seqshard, synth
from oracle import max_abs_rel_err, prism_seq

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d_v,d_k", [(64, 128), (128, 128), (32, 16)])
def test_state_affine_matches_fp64(d_v, d_k):
    g = torch.Generator().manual_seed(d_v + d_k)
    S = torch.randn(3, 4, d_v, d_k, generator=g)
    M = torch.randn(3, 4, d_k, d_k, generator=g) / d_k ** 0.5
    N = torch.randn(3, 4, d_v, d_k, generator=g)
    ref = S.double() @ M.double() + N.double()
    Sd, Md, Nd = S.cuda(), M.cuda(), N.cuda()
    out = prism.state_affine(Sd, Md, Nd)
    no_n = prism.state_affine(Sd, Md)
    prism.state_affine(Sd, Md, Nd, out=Sd)  # in place over S
    torch.cuda.synchronize()
    err = (out.cpu().double() - ref).abs().max().item() / ref.abs().max().item()
    assert err < 1e-5
    assert torch.equal(out, Sd)  # same arithmetic, same order
    assert (no_n.cpu().double() - (S.double() @ M.double())).abs().max().item() < 1e-4


def _sharded_on_gpu(w, bounds, chain="linear"):
    inp = synth.make_inputs(w)
    d = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}
    W = w.W
    names = ("q", "k", "v", "gamma", "beta", "u", "alpha", "gain")
    segs = [seqshard.Segment(**{n: d[n][:, s:e].contiguous() for n in names}, start=s)
            for s, e in zip(bounds[:-1], bounds[1:])]
    ops = seqshard.LibraryOps()
    halos = [seqshard.halo_rows(s.v, W) for s in segs]
    hists = [seqshard.conv_history(halos[i - 1]) if i else None for i in range(len(segs))]
    lens = [seqshard.local_lengths(d["lengths"], s, s.v.shape[1]) for s in segs]
    maps = [seqshard.segment_map(s, d["conv_w"], w.L, ln, chain, w.chunk, ops, hs)
            for s, ln, hs in zip(segs, lens, hists)]
    outs, S_end = [], None
    for r, (sg, ln, hs) in enumerate(zip(segs, lens, hists)):
        S_start = seqshard.start_state(d["S0"], maps[:r], maps[0][1], ops)
        o, S_end = seqshard.scan_segment(sg, d["conv_w"], w.L, ln, chain, w.chunk, S_start, ops, hs)
        outs.append(o)
    torch.cuda.synchronize()
    assert prism.stream_status() == 0
    x = synth.to_float64_numpy(inp)
    o_ref, S_ref = prism_seq(**x, chain=chain)
    return torch.cat(outs, 1).float().cpu().numpy(), S_end.cpu().numpy(), o_ref, S_ref


def _rel_o(o, o_ref):
    """The forward bars' metric on outputs [B, T, H, d_v]: max-abs-relative error per
    (batch, head) slice, the largest over slices."""
    return max_abs_rel_err(o, o_ref)


def _rel_S(S, S_ref):
    """The same metric on states [B, H, d_v, d_k], one slice per (batch, head)."""
    return max_abs_rel_err(S, S_ref, slice_axes=(0, 1))


def test_sharded_bf16_tensor_core_segments():
    """Four segments of an LM-shaped head (d = 128, L = 4, W = 4, bf16: the tensor-core
    scan), segments of 128 tokens plus 3 history tokens (a ragged last chunk)."""
    w = synth.WORKLOADS["lm_130m"].replace(B=2, T=512, H=2, with_s0=True, seed=41)
    o, S, o_ref, S_ref = _sharded_on_gpu(w, [0, 128, 256, 384, 512])
    assert _rel_o(o, o_ref) <= 2e-2
    assert _rel_S(S, S_ref) <= 2e-2


def test_sharded_fp32_uneven_segments_ragged_lengths():
    w = synth.Workload("shard_fp32", B=3, T=150, H=2, d_k=64, d_v=64, L=3, chunk=64, W=4, dtype="fp32",
                       lengths_lo=40, with_s0=True, seed=42)
    o, S, o_ref, S_ref = _sharded_on_gpu(w, [0, 37, 100, 150], chain="gelu")
    assert _rel_o(o, o_ref) <= 1e-4
    assert _rel_S(S, S_ref) <= 1e-4


@pytest.mark.parametrize("P", [4, 8])
def test_segmented_bf16_tensor_core_segments(P):
    """scan_fwd_segmented on one device: each sequence cut into P segments that run side
    by side on the tensor-core scan (d = 128, L = 4, bf16), with S0 and ragged lengths,
    against the oracle's scan of the whole sequence."""
    w = synth.WORKLOADS["lm_130m"].replace(B=2, T=700, H=2, with_s0=True, lengths_lo=300, seed=43)
    inp = synth.make_inputs(w)
    d = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}
    o, S = seqshard.scan_fwd_segmented(d["q"], d["k"], d["v"], d["gamma"], d["beta"], d["u"], d["alpha"],
                                       d["gain"], d["conv_w"], w.L, P, S0=d["S0"], lengths=d["lengths"])
    torch.cuda.synchronize()
    assert prism.stream_status() == 0
    o_ref, S_ref = prism_seq(**synth.to_float64_numpy(inp))
    o = o.float().cpu().numpy()
    assert _rel_o(o, o_ref) <= 2e-2
    assert _rel_S(S.cpu().numpy(), S_ref) <= 2e-2
    lens = inp["lengths"].numpy()
    for b, n in enumerate(lens):
        assert np.all(o[b, n:] == 0)


@pytest.mark.parametrize("P", [4, 8])
def test_segmented_fp32_gelu_ragged(P):
    """The same on the fp32 build with the exact GELU chain (1e-4 bar), T not a multiple
    of P, and lengths that end inside early segments."""
    w = synth.Workload("seg_fp32", B=3, T=203, H=2, d_k=64, d_v=64, L=3, chunk=64, W=4, dtype="fp32",
                       lengths_lo=20, with_s0=True, seed=44)
    inp = synth.make_inputs(w)
    d = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}
    o, S = seqshard.scan_fwd_segmented(d["q"], d["k"], d["v"], d["gamma"], d["beta"], d["u"], d["alpha"],
                                       d["gain"], d["conv_w"], w.L, P, S0=d["S0"], lengths=d["lengths"],
                                       chain="gelu")
    torch.cuda.synchronize()
    assert prism.stream_status() == 0
    o_ref, S_ref = prism_seq(**synth.to_float64_numpy(inp), chain="gelu")
    assert _rel_o(o.cpu().numpy(), o_ref) <= 1e-4
    assert _rel_S(S.cpu().numpy(), S_ref) <= 1e-4
