"""The debug build (libprism_debug.so, compiled with PRISM_DEBUG_BOUNDS): its kernels check
the global indices they compute against their buffers' extents and record
PRISM_ERR_BOUNDS instead of faulting.  On valid inputs it must report nothing and give the
release build's results bit for bit, on every forward path: the tensor-core scan (plain,
in two halves, cut into segments, ragged rows), the fp32 chunk form, the token-by-token
kernel, the decode step, and both backward paths.  Its probe hook shows that a failed device-side check
reaches prism_stream_status.

The debug library is loaded in a child process (PRISM_DEBUG_BOUNDS=1 selects it), which
writes its outputs to a file that this process compares with the release library's.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from linear_attention_sequence_shortconv_b200 import synth

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = {
    # tensor-core scan, ragged tail and S0
    "tc_d128": synth.Workload("a", B=2, T=200, H=3, d_k=128, d_v=128, L=4, chunk=64, with_s0=True, seed=81),
    # tensor-core scan in two halves (10 chunks, chains leave SMs idle), ragged rows
    "tc_halves": synth.Workload("b", B=3, T=640, H=2, d_k=64, d_v=64, L=3, chunk=64, lengths_lo=300, seed=82),
    # tensor-core scan cut into segments (64 chunks over two chains)
    "tc_segments": synth.Workload("c", B=1, T=4096, H=2, d_k=128, d_v=128, L=4, chunk=64, with_s0=True, seed=83),
    # more chains than SMs, ragged rows (longest rows first), W = 8
    "tc_many_chains": synth.Workload("d", B=80, T=150, H=2, d_k=64, d_v=64, L=2, chunk=64, W=8, lengths_lo=1,
                                     seed=84),
    # fp32 chunk form
    "fp32_chunk": synth.Workload("e", B=2, T=100, H=2, d_k=32, d_v=32, L=3, chunk=32, dtype="fp32",
                                 lengths_lo=10, with_s0=True, seed=85),
    # token by token: bf16 at d = 32, and fp32 at d = 128
    "token_bf16": synth.Workload("f", B=2, T=90, H=2, d_k=32, d_v=32, L=3, chunk=32, seed=86),
    "token_fp32": synth.Workload("g", B=1, T=70, H=2, d_k=128, d_v=128, L=2, chunk=64, dtype="fp32", seed=87),
}


def _run_all():
    import linear_attention_sequence_shortconv_b200 as prism

    out = {}
    for name, w in CASES.items():
        d = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in synth.make_inputs(w).items()}
        for chain in ("linear", "gelu"):
            o, S = prism.scan_fwd(d["q"], d["k"], d["v"], d["gamma"], d["beta"], d["u"], d["alpha"], d["gain"],
                                  d["conv_w"], L=w.L, chunk=w.chunk, S0=d["S0"], lengths=d["lengths"], chain=chain)
            status = prism.stream_status()
            out[f"{name}_{chain}_o"] = o.float().cpu().numpy()
            out[f"{name}_{chain}_S"] = S.cpu().numpy()
            out[f"{name}_{chain}_status"] = np.array(status)
    # decode: a few tokens of two cases, the state and the ShortConv history carried in place
    for name in ("tc_d128", "fp32_chunk"):
        w = CASES[name]
        d = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in synth.make_inputs(w).items()}
        S = torch.zeros((w.B, w.H, w.d_v, w.d_k), dtype=torch.float32, device="cuda")
        hist = torch.zeros((w.B, w.H, w.W - 1, w.d_v), dtype=d["v"].dtype, device="cuda")
        for t in range(3):
            tok = {n: d[n][:, t].contiguous() for n in ("q", "k", "v", "gamma", "beta", "u", "alpha", "gain")}
            o = prism.decode_step(tok["q"], tok["k"], tok["v"], tok["gamma"], tok["beta"], tok["u"], tok["alpha"],
                                  tok["gain"], d["conv_w"], hist, S, L=w.L)
            out[f"decode_{name}_{t}_o"] = o.float().cpu().numpy()
        out[f"decode_{name}_status"] = np.array(prism.stream_status())
        out[f"decode_{name}_S"] = S.cpu().numpy()
        out[f"decode_{name}_hist"] = hist.float().cpu().numpy()
    # backward: the chunked path (d = 64, ragged rows) and the token-by-token one (fp32, d = 32)
    for name, w in (("bwd_chunked", synth.Workload("h", B=2, T=150, H=2, d_k=64, d_v=64, L=3, chunk=64,
                                                   lengths_lo=70, with_s0=True, seed=88)),
                    ("bwd_token", synth.Workload("i", B=1, T=60, H=2, d_k=32, d_v=32, L=3, chunk=32, dtype="fp32",
                                                 with_s0=True, seed=89))):
        inp = synth.make_inputs(w)
        d = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}
        dO = torch.randn((w.B, w.T, w.H, w.d_v), generator=torch.Generator().manual_seed(7)).to(inp["v"].dtype)
        g = prism.scan_bwd(d["q"], d["k"], d["v"], d["gamma"], d["beta"], d["u"], d["alpha"], d["gain"],
                           d["conv_w"], dO.cuda(), L=w.L, S0=d["S0"], lengths=d["lengths"])
        out[f"{name}_status"] = np.array(prism.stream_status())
        for n, t in g.items():
            out[f"{name}_{n}"] = t.cpu().numpy()
    return out


def _child(path):
    """Run in a process started with PRISM_DEBUG_BOUNDS=1: the probe hook, then every case."""
    import linear_attention_sequence_shortconv_b200 as prism

    L = prism.lib()
    assert L.prism_debug_bounds() == 1
    probe = {}
    for i, n in ((3, 4), (0, 1), (4, 4), (-1, 4)):
        assert L.prism_debug_bounds_probe(i, n, None) == 0
        probe[f"probe_{i}_{n}"] = np.array(prism.stream_status())
    out = _run_all()
    out.update(probe)
    np.savez(path, **out)


def test_debug_build_matches_release_and_reports_nothing(tmp_path):
    ref = _run_all()
    path = str(tmp_path / "debug.npz")
    env = dict(os.environ, PRISM_DEBUG_BOUNDS="1")
    code = f"import tests.test_gpu_debug_bounds as t; t._child({path!r})"
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    got = np.load(path)
    # the device-side check reports exactly the indices outside [0, n)
    assert int(got["probe_3_4"]) == 0 and int(got["probe_0_1"]) == 0
    assert int(got["probe_4_4"]) == 6 and int(got["probe_-1_4"]) == 6  # PRISM_ERR_BOUNDS
    for key, val in ref.items():
        if key.endswith("_status"):
            assert int(val) == 0 and int(got[key]) == 0, key
        else:
            assert np.array_equal(val, got[key]), key
