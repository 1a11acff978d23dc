"""Parity of the CUDA path (through the C ABI) against the fp64 CPU oracle.

Bars (max-abs-relative error, per (batch, head) slice): 2e-2 for bf16 inputs
and outputs with fp32 accumulation, 1e-4 for the fp32 build.  The oracle
consumes exactly the (already rounded) inputs the GPU sees.
"""
import numpy as np
import pytest
import torch

from linear_attention_sequence_shortconv_b200 import synth
from oracle import gdn_seq, max_abs_rel_err, prism_seq, residual_chain
from tests.helpers import TOL, gpu_run, oracle_run, rel_err

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS

# Reduced versions of every workload: several chunks, a ragged tail (T not a
# multiple of 64), and the same head sizes, L, W and dtypes as the full ones.
REDUCED = {
    "tiny_fp32": W["tiny_fp32"],
    "tiny_fp32_s0": W["tiny_fp32"].replace(with_s0=True, seed=1),
    "gdn_l1": W["gdn_l1"].replace(B=2, T=300, H=2),
    "recsys": W["recsys"].replace(B=6, T=333, lengths_lo=40),
    "lm_130m": W["lm_130m"].replace(B=2, T=200, H=3, with_s0=True),
    "long_ctx": W["long_ctx"].replace(T=150, H=2),
    "lm_fp32": W["lm_130m"].replace(B=1, T=130, H=2, dtype="fp32"),
    "d32_L16_W8": synth.Workload("d32", B=2, T=97, H=3, d_k=32, d_v=32, L=16, chunk=32, W=8),
    "dk64_dv128_W1": synth.Workload("mixed", B=1, T=77, H=2, d_k=64, d_v=128, L=3, chunk=64, W=1),
}


@pytest.mark.parametrize("name", list(REDUCED))
def test_parity_reduced(name):
    w = REDUCED[name]
    inp = synth.make_inputs(w)
    o, S = gpu_run(inp, w)
    o_ref, S_ref = oracle_run(inp, w)
    tol = TOL[w.dtype]
    assert max_abs_rel_err(o, o_ref) <= tol, name
    assert max_abs_rel_err(S, S_ref, slice_axes=(0, 1)) <= tol, name
    if w.lengths_lo is not None:
        lens = inp["lengths"].numpy()
        for b, n in enumerate(lens):
            assert np.all(o[b, n:] == 0)


def test_L1_full_config_equals_plain_gdn():
    """The L = 1 workload (B=4, H=4, T=1024, d=64, bf16) against the separately
    written gated-delta recurrence."""
    w = W["gdn_l1"]
    inp = synth.make_inputs(w)
    o, S = gpu_run(inp, w)
    x = synth.to_float64_numpy(inp)
    o_ref, S_ref = gdn_seq(x["q"], x["k"], x["v"], x["gamma"], x["beta"])
    assert max_abs_rel_err(o, o_ref) <= TOL["bf16"]
    assert max_abs_rel_err(S, S_ref, slice_axes=(0, 1)) <= TOL["bf16"]


@pytest.mark.parametrize("name,pairs", [
    ("lm_130m", [(0, 0), (7, 3), (15, 5)]),
    ("recsys", [(0, 0), (77, 1), (127, 0)]),
])
def test_parity_full_size_sampled(name, pairs):
    """Full-size workloads in the launch configuration the bench times; the
    oracle evaluates a sample of (batch, head) chains over the whole sequence."""
    w = W[name]
    inp = synth.make_inputs(w)
    o, S = gpu_run(inp, w)
    outs, states = oracle_run(inp, w, bh=pairs)
    for (b, h), o_ref, S_ref in zip(pairs, outs, states):
        assert rel_err(o[b, :, h], o_ref) <= TOL[w.dtype], (b, h)
        assert rel_err(S[b, h], S_ref) <= TOL[w.dtype], (b, h)


def test_long_context_full_size_final_state_sampled():
    """Long context (B=1, T=65536, H=8, d=128, L=8): outputs and the returned
    final state of one head against the oracle over all 65536 steps."""
    w = W["long_ctx"]
    inp = synth.make_inputs(w)
    o, S = gpu_run(inp, w)
    outs, states = oracle_run(inp, w, bh=[(0, 5)])
    assert rel_err(o[0, :, 5], outs[0]) <= TOL["bf16"]
    assert rel_err(S[0, 5], states[0]) <= TOL["bf16"]


# ---------------------------------------------------------------- cut sequences
SEGMENTED = {
    # 33 chunks over 2 chains: two segments, a ragged last chunk, S0, L = 8
    "two_segments": synth.Workload("seg2", B=1, T=2100, H=2, d_k=128, d_v=128, L=8, chunk=64, with_s0=True, seed=5),
    # two segments per row; row 0 ends inside the first one, so its second segment is empty
    "ragged": synth.Workload("segr", B=2, T=2600, H=1, d_k=128, d_v=128, L=4, chunk=64, with_s0=True, seed=6),
    # d = 64, one chain cut into four segments, the exact GELU chain
    "d64": synth.Workload("seg64", B=1, T=4096, H=1, d_k=64, d_v=64, L=3, chunk=64, seed=7),
}


@pytest.mark.parametrize("name", list(SEGMENTED))
def test_segmented_long_sequences(name):
    """Long sequences over few chains run as segments side by side (three scans and a fold
    of the per-segment state maps); outputs and final states against the token loop."""
    import linear_attention_sequence_shortconv_b200 as prism

    w = SEGMENTED[name]
    assert prism.workspace_size(w.B, w.T, w.H, w.d_k, w.d_v, w.L, w.W, w.chunk, 0) > 0  # the cut path
    inp = synth.make_inputs(w)
    if name == "ragged":
        inp["lengths"] = torch.tensor([700, 2600], dtype=torch.int32)
    chain = "gelu" if name == "d64" else "linear"
    o, S = gpu_run(inp, w, chain=chain)
    assert prism.stream_status() == 0
    o_ref, S_ref = oracle_run(inp, w, chain=chain)
    assert max_abs_rel_err(o, o_ref) <= TOL["bf16"]
    assert max_abs_rel_err(S, S_ref, slice_axes=(0, 1)) <= TOL["bf16"]
    if name == "ragged":
        assert np.all(o[0, 700:] == 0)


# ---------------------------------------------------------------- edge cases
@pytest.mark.parametrize("T", [1, 2, 3, 63, 64, 65])
def test_short_and_boundary_lengths(T):
    w = synth.Workload("edge", B=2, T=T, H=2, d_k=64, d_v=64, L=4, chunk=64, with_s0=True)
    inp = synth.make_inputs(w)
    o, S = gpu_run(inp, w)
    o_ref, S_ref = oracle_run(inp, w)
    assert max_abs_rel_err(o, o_ref) <= TOL["bf16"]
    assert max_abs_rel_err(S, S_ref, slice_axes=(0, 1)) <= TOL["bf16"]


def test_empty_and_full_rows_in_one_batch():
    """lengths = 0 (empty row: o = 0, S_final = S0), 1, T-1 and T in one batch."""
    w = synth.Workload("ragged", B=4, T=130, H=2, d_k=128, d_v=128, L=4, chunk=64, with_s0=True)
    inp = synth.make_inputs(w)
    inp["lengths"] = torch.tensor([0, 1, 129, 130], dtype=torch.int32)
    o, S = gpu_run(inp, w)
    o_ref, S_ref = oracle_run(inp, w)
    assert np.all(o[0] == 0)
    np.testing.assert_array_equal(S[0], inp["S0"][0].numpy())
    assert max_abs_rel_err(o, o_ref) <= TOL["bf16"]
    assert max_abs_rel_err(S, S_ref, slice_axes=(0, 1)) <= TOL["bf16"]


def test_bitwise_deterministic():
    w = W["lm_130m"].replace(B=3, T=257, H=2)
    inp = synth.make_inputs(w)
    o1, S1 = gpu_run(inp, w)
    o2, S2 = gpu_run(inp, w)
    assert np.array_equal(o1, o2) and np.array_equal(S1, S2)


def test_state_only_optional():
    w = REDUCED["lm_130m"]
    inp = synth.make_inputs(w)
    o1, _ = gpu_run(inp, w, want_state=False)
    o2, _ = gpu_run(inp, w)
    assert np.array_equal(o1, o2)


# ---------------------------------------------------------------- prologue
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_prologue_kernel(dtype):
    import linear_attention_sequence_shortconv_b200 as prism

    w = synth.Workload("pro", B=3, T=70, H=2, d_k=64, d_v=64, L=5, chunk=64, lengths_lo=10, dtype=dtype)
    inp = synth.make_inputs(w)
    d = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}
    rho = prism.prologue_fwd(d["v"], d["alpha"], d["gain"], d["conv_w"], L=w.L, lengths=d["lengths"])
    torch.cuda.synchronize()
    x = synth.to_float64_numpy(inp)
    ref = x["alpha"][..., None] * residual_chain(x["v"], x["conv_w"], x["gain"])
    valid = np.arange(w.T)[None, :] < x["lengths"][:, None]
    ref = np.where(valid[:, :, None, None, None], ref, 0.0)
    got = rho.cpu().numpy()
    assert np.abs(got - ref).max() <= 1e-5 * max(np.abs(ref).max(), 1.0)


# ---------------------------------------------------------------- host entry point
def test_host_entry_point_matches_device_entry_point():
    import linear_attention_sequence_shortconv_b200 as prism

    w = REDUCED["recsys"]
    inp = synth.make_inputs(w)
    o_dev, S_dev = gpu_run(inp, w)
    host = {n: (t.pin_memory() if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}
    host["o"] = torch.empty(o_dev.shape, dtype=torch.bfloat16).pin_memory()
    host["S_final"] = torch.empty(S_dev.shape, dtype=torch.float32).pin_memory()
    dev = {n: torch.empty_like(t, device="cuda") for n, t in host.items() if isinstance(t, torch.Tensor)}
    prism.scan_fwd_host(host, dev, L=w.L, chunk=w.chunk)
    torch.cuda.synchronize()
    assert np.array_equal(host["o"].float().numpy(), o_dev)
    assert np.array_equal(host["S_final"].numpy(), S_dev)


# ---------------------------------------------------------------- errors
def test_argument_errors_raise_before_launch():
    import linear_attention_sequence_shortconv_b200 as prism

    w = REDUCED["lm_130m"]
    inp = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in synth.make_inputs(w).items()}
    with pytest.raises(prism.PrismError) as e:
        prism.scan_fwd(inp["q"], inp["k"], inp["v"], inp["gamma"], inp["beta"], inp["u"], inp["alpha"],
                       inp["gain"], inp["conv_w"], L=w.L, chunk=48)
    assert e.value.code == 2
    misaligned = inp["q"].data_ptr() + 2
    rc = prism.lib().prism_scan_fwd(misaligned, inp["k"].data_ptr(), inp["v"].data_ptr(),
                                    inp["gamma"].data_ptr(), inp["beta"].data_ptr(), inp["u"].data_ptr(),
                                    inp["alpha"].data_ptr(), inp["gain"].data_ptr(), inp["conv_w"].data_ptr(),
                                    None, None, 1, 8, 1, 128, 128, 4, 4, 64, 0,
                                    inp["v"].data_ptr(), None, None, 0, None)
    assert rc == 2
    assert prism.stream_status() == 0


# ---------------------------------------------------------------- paths and device-side errors
def test_tensor_core_path_is_taken_for_the_benchmarked_shapes():
    import linear_attention_sequence_shortconv_b200 as prism

    for name in ("lm_130m", "recsys", "gdn_l1"):
        w = W[name]
        assert prism.uses_tensor_cores(w.d_k, w.d_v, w.L, w.W, w.chunk, prism.PRISM_BF16), name
    assert not prism.uses_tensor_cores(128, 128, 4, 4, 64, prism.PRISM_FP32)


def test_bounded_wait_timeout_is_reported_and_recovers():
    """A spin limit of one poll makes the chunk kernel's first wait give up: the
    kernel records PRISM_ERR_TIMEOUT, drains its own copies, frees TMEM and
    exits; the context stays usable and the next call is correct."""
    import linear_attention_sequence_shortconv_b200 as prism

    w = REDUCED["lm_130m"]
    inp = synth.make_inputs(w)
    prism.set_spin_limit(1)
    try:
        gpu_run(inp, w)
        assert prism.stream_status() == 5
    finally:
        prism.set_spin_limit(0)
    assert prism.stream_status() == 0
    o, S = gpu_run(inp, w)
    o_ref, S_ref = oracle_run(inp, w)
    assert max_abs_rel_err(o, o_ref) <= TOL["bf16"]


def test_full_size_bitwise_deterministic():
    """The benchmarked LM layer (96 chains x 32 chunks) twice: bitwise equal outputs and
    states.  A buffer reused before an asynchronous reader is done shows up here first."""
    w = W["lm_130m"]
    inp = synth.make_inputs(w)
    o1, S1 = gpu_run(inp, w)
    o2, S2 = gpu_run(inp, w)
    o3, S3 = gpu_run(inp, w)
    assert np.array_equal(o1, o2) and np.array_equal(o1, o3)
    assert np.array_equal(S1, S2) and np.array_equal(S1, S3)


# ---------------------------------------------------------------- strongly decaying chunks
@pytest.mark.parametrize("name", ["lm_130m", "recsys"])
@pytest.mark.parametrize("chain", ["linear", "gelu"])
def test_strongly_decaying_chunks(name, chain):
    """Chunks whose total log-decay is below -60 take the exact path of the chunk
    kernel (per-element e^{G_t - G_i}, the state-side decay applied to U instead of
    P).  Row 0: every other chunk strongly decaying; row 1: all of them; the other
    rows: the ordinary gates."""
    w = {"lm_130m": W["lm_130m"].replace(B=3, T=300, H=2, with_s0=True),
         "recsys": W["recsys"].replace(B=3, T=260, lengths_lo=None)}[name]
    inp = synth.make_inputs(w)
    g = inp["gamma"].clone()
    strong = torch.full_like(g[0, :64], 0.38).to(torch.bfloat16).float()  # 64 log(0.38) = -62
    for c0 in range(64, w.T, 128):
        n = min(64, w.T - c0)
        g[0, c0:c0 + n] = strong[:n]
    g[1] = torch.full_like(g[1], 0.38).to(torch.bfloat16).float()
    inp["gamma"] = g
    import linear_attention_sequence_shortconv_b200 as prism
    assert prism.uses_tensor_cores(w.d_k, w.d_v, w.L, w.W, w.chunk, prism.PRISM_BF16)
    o, S = gpu_run(inp, w, chain=chain)
    o_ref, S_ref = oracle_run(inp, w, chain=chain)
    assert max_abs_rel_err(o, o_ref) <= TOL["bf16"]
    assert max_abs_rel_err(S, S_ref, slice_axes=(0, 1)) <= TOL["bf16"]


def test_ragged_rows_exceeding_the_sms():
    """More chains than SMs with ragged lengths (the scan takes the rows longest first),
    every chain against the oracle, empty rows included."""
    w = synth.Workload("ragged160", B=80, T=150, H=2, d_k=64, d_v=64, L=3, chunk=64, lengths_lo=0,
                       with_s0=True, seed=31)
    inp = synth.make_inputs(w)
    inp["lengths"][::7] = 0
    o, S = gpu_run(inp, w)
    x = synth.to_float64_numpy(inp)
    o_ref, S_ref = prism_seq(**x)
    assert max_abs_rel_err(o, o_ref) <= TOL["bf16"]
    assert max_abs_rel_err(S, S_ref, slice_axes=(0, 1)) <= TOL["bf16"]
    for b, n in enumerate(inp["lengths"].tolist()):
        assert np.all(o[b, n:] == 0)


@pytest.mark.parametrize("d,L", [(128, 4), (64, 3)])
def test_two_halves_with_ragged_rows(d, L):
    """The scan in two launches (chains that leave SMs idle, 15 chunks), with rows that end
    inside the first half, inside the second, exactly at the split and an empty row: the
    hand-over of the end states between the launches, against the oracle."""
    w = synth.Workload("halves", B=5, T=900, H=2, d_k=d, d_v=d, L=L, chunk=64, with_s0=True, seed=37 + d)
    import linear_attention_sequence_shortconv_b200 as prism
    assert prism.scan_fwd_launches(w.B, w.T, w.H, d, d, L, w.W, 64, 0) == 4  # two halves
    inp = synth.make_inputs(w)
    inp["lengths"] = torch.tensor([900, 400, 0, 512, 777], dtype=torch.int32)
    o, S = gpu_run(inp, w)
    o_ref, S_ref = prism_seq(**synth.to_float64_numpy(inp))
    assert max_abs_rel_err(o, o_ref) <= TOL["bf16"]
    assert max_abs_rel_err(S, S_ref, slice_axes=(0, 1)) <= TOL["bf16"]
    for b, n in enumerate(inp["lengths"].tolist()):
        assert np.all(o[b, n:] == 0)
