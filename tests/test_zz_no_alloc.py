"""prism_scan_fwd_static: the scan with its scratch in a device-global array of the
library, so the call allocates nothing.  Its results must be bit-for-bit those of
prism_scan_fwd_ex with a caller-supplied workspace, also when two calls follow
each other and reuse the same scratch.
"""
import numpy as np
import pytest
import torch

import linear_attention_sequence_shortconv_b200 as prism
from linear_attention_sequence_shortconv_b200 import synth

FAKE = 0x10000  # 16-byte aligned, never dereferenced: these calls fail before any CUDA call


def _static_call(**kw):
    a = dict(B=2, T=64, H=2, d_k=64, d_v=64, L=4, W=4, chunk=64, dtype=0, chain=0)
    a.update(kw)
    return prism.lib().prism_scan_fwd_static(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None,
                                             a["B"], a["T"], a["H"], a["d_k"], a["d_v"], a["L"], a["W"], a["chunk"],
                                             a["dtype"], FAKE, None, None, a["chain"])


def test_every_shape_fits_the_static_scratch():
    # only a cut sequence uses scratch, and chains x segments never exceeds 148: no shape
    # needs more than 3 x 148 x 128^2 fp32 (27.75 MiB) of the array's 32 MiB, so the size
    # check of the entry point is a guard that no valid shape reaches
    for B, T, H in ((1, 65536, 8), (1, 1 << 20, 1), (2, 4096, 1), (74, 4096, 1), (16, 2048, 6)):
        assert prism.workspace_size(B, T, H, 128, 128, 8, 4, 64, 0) <= 32 << 20


def test_invalid_arguments_are_rejected_before_launch():
    assert _static_call(chain=5) == 1
    assert _static_call(B=0) == 1
    assert _static_call(d_k=48) == 2


def _run(fn, d, w, **kw):
    return fn(d["q"], d["k"], d["v"], d["gamma"], d["beta"], d["u"], d["alpha"], d["gain"], d["conv_w"],
              L=w.L, chunk=w.chunk, S0=d["S0"], lengths=d["lengths"], **kw)


@pytest.mark.gpu
def test_two_calls_in_a_row_match_the_workspace_entry_point():
    # a sequence long enough to be cut into segments (its maps and start states live in the
    # scratch), then a ragged batch that needs no scratch, then the long one again
    w1 = synth.WORKLOADS["long_ctx"].replace(T=4096, H=2, L=4, with_s0=True, seed=11)
    w2 = synth.WORKLOADS["recsys"].replace(B=5, T=200, lengths_lo=20, seed=12)
    w3 = w1.replace(seed=13)
    assert prism.workspace_size(w1.B, w1.T, w1.H, w1.d_k, w1.d_v, w1.L, w1.W, w1.chunk, 0) > 0
    runs = []
    for w in (w1, w2, w3):
        d = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in synth.make_inputs(w).items()}
        runs.append((w, d))
    # the static entry point twice in a row (the second call reuses the scratch)...
    got = [_run(prism.scan_fwd_static, d, w) for w, d in runs]
    # ...and the entry point with a caller-supplied workspace on the same inputs
    ref = [_run(prism.scan_fwd, d, w) for w, d in runs]
    torch.cuda.synchronize()
    for (o_s, S_s), (o_r, S_r) in zip(got, ref):
        assert torch.equal(o_s, o_r)
        assert torch.equal(S_s, S_r)
    assert prism.stream_status() == 0


@pytest.mark.gpu
def test_full_size_long_context_matches_and_allocates_nothing():
    w = synth.WORKLOADS["long_ctx"]
    assert 0 < prism.workspace_size(w.B, w.T, w.H, w.d_k, w.d_v, w.L, w.W, w.chunk, 0) <= 32 << 20
    d = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in synth.make_inputs(w).items()}
    o = torch.empty((w.B, w.T, w.H, w.d_v), dtype=torch.bfloat16, device="cuda")
    S = torch.empty((w.B, w.H, w.d_v, w.d_k), dtype=torch.float32, device="cuda")
    _run(prism.scan_fwd_static, d, w, o=o, S_final=S)  # first use loads the module and its array
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(2):
        _run(prism.scan_fwd_static, d, w, o=o, S_final=S)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    # the workspace path needs 28 MiB; nothing of that size may appear
    assert free0 - free1 < (4 << 20)
    o_r, S_r = _run(prism.scan_fwd, d, w)
    torch.cuda.synchronize()
    assert torch.equal(o, o_r)
    assert torch.equal(S, S_r)
