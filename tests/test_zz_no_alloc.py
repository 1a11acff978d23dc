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
                                             a["dtype"], FAKE, None, None, a["chain"], None)


def test_static_scratch_holds_the_layer_shapes():
    # the scratch holds the residual write vectors of the 130M-LM layer and of the recsys
    # layer; a long sequence with many directions needs more and is refused before launch
    cap = 192 << 20
    assert prism.workspace_size(16, 2048, 6, 128, 128, 4, 4, 64, 0) <= cap
    assert prism.workspace_size(128, 1024, 2, 64, 64, 4, 4, 64, 0) <= cap
    assert prism.workspace_size(1, 65536, 8, 128, 128, 8, 4, 64, 0) > cap
    assert _static_call(B=1, T=65536, H=8, d_k=128, d_v=128, L=8) == 3


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
def test_full_size_lm_layer_matches_and_allocates_nothing():
    w = synth.WORKLOADS["lm_130m"]
    assert 0 < prism.workspace_size(w.B, w.T, w.H, w.d_k, w.d_v, w.L, w.W, w.chunk, 0) <= 192 << 20
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
    # the workspace path needs 144 MiB; nothing of that size may appear
    assert free0 - free1 < (4 << 20)
    o_r, S_r = _run(prism.scan_fwd, d, w)
    torch.cuda.synchronize()
    assert torch.equal(o, o_r)
    assert torch.equal(S, S_r)
