"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol include/prism.h declares, and rejects bad arguments before it
touches the device."""
import ctypes
import os
import re

import pytest

import linear_attention_sequence_shortconv_b200 as prism
from linear_attention_sequence_shortconv_b200 import build as prism_build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "prism.h")


@pytest.fixture(scope="module")
def L():
    prism_build.build()
    return prism.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(prism_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(prism.EXPORTS)


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_version_matches_header(L):
    text = open(HEADER).read()
    ver = tuple(int(re.search(rf"#define PRISM_VERSION_{k}\s+(\d+)", text).group(1)) for k in ("MAJOR", "MINOR", "PATCH"))
    assert prism.version() == ver


def test_status_strings(L):
    for code in range(7):
        assert prism.status_string(code).startswith("PRISM")
    assert "BOUNDS" in prism.status_string(6)
    assert "unknown" in prism.status_string(99)


def test_debug_build_exports_the_same_symbols(L):
    # the bounds-checked debug build is a second library with the same ABI; it reports itself
    # through prism_debug_bounds (the release build: 0, and its probe hook is unsupported)
    D = ctypes.CDLL(prism_build.LIB_DEBUG)
    for name in declared_functions():
        assert hasattr(D, name), name
    D.prism_debug_bounds.restype = ctypes.c_int
    assert D.prism_debug_bounds() == 1
    assert L.prism_debug_bounds() == 0
    assert L.prism_debug_bounds_probe(5, 4, None) == 2  # PRISM_ERR_UNSUPPORTED, no CUDA call


FAKE = 0x10000  # 16-byte aligned, never dereferenced: every case below fails before any CUDA call


def call(lib_, workspace_ok=True, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, gamma=FAKE, beta=FAKE, u=FAKE, alpha=FAKE, gain=FAKE, conv_w=FAKE,
             S0=None, lengths=None, B=2, T=8, H=2, d_k=64, d_v=64, L=4, W=4, chunk=64, dtype=0,
             o=FAKE, S_final=None)
    a.update(kw)
    ws, ws_bytes = (FAKE, 1 << 40) if workspace_ok else (None, 0)
    return lib_.prism_scan_fwd(a["q"], a["k"], a["v"], a["gamma"], a["beta"], a["u"], a["alpha"], a["gain"],
                               a["conv_w"], a["S0"], a["lengths"], a["B"], a["T"], a["H"], a["d_k"], a["d_v"],
                               a["L"], a["W"], a["chunk"], a["dtype"], a["o"], a["S_final"], ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), 1), (dict(T=0), 1), (dict(H=-1), 1), (dict(L=0), 1), (dict(W=0), 1), (dict(dtype=7), 1),
    (dict(q=None), 1), (dict(o=None), 1), (dict(conv_w=None), 1), (dict(u=None), 1), (dict(alpha=None), 1),
    (dict(d_k=48), 2), (dict(d_v=256), 2), (dict(L=17), 2), (dict(W=9), 2), (dict(chunk=48), 2),
    (dict(chunk=128), 2), (dict(q=FAKE + 8), 2), (dict(gamma=FAKE + 4), 2), (dict(S_final=FAKE + 2), 2),
])
def test_invalid_arguments(L, kw, code):
    assert call(L, **kw) == code


def test_L1_needs_no_residual_inputs(L):
    # L = 1 ignores u/alpha/gain: with them NULL the checks pass up to the first
    # device query, so only check that NULL residual inputs are not rejected as
    # invalid when a size error is also present (the size error wins).
    assert call(L, L=1, u=None, alpha=None, gain=None, B=0) == 1


def _segments(B, T, H):
    """Segments per sequence of the tensor-core scan: long sequences (>= 32 chunks of 64)
    whose chains fill under half of a B200's 148 SMs are cut into segments of >= 16 chunks."""
    nc, chains = -(-T // 64), B * H
    if 2 * chains > 148 or nc < 32:
        return 1
    P = min(148 // chains, nc // 16)
    if P < 2:
        return 1
    cps = -(-nc // P)
    return -(-nc // cps)


def _ptil(B, T, H, D, L):
    """Bytes of the residual write vectors the tensor-core scan stages in the workspace:
    bf16, one d_v row per (token, head, direction), rounded up to 256."""
    n = B * T * H * (L - 1) * D * 2
    return -(-n // 256) * 256


def test_workspace_size_query(L):
    # the tensor-core scan stages the residual write vectors of every token (bf16, the
    # layout of gain); a cut sequence adds three fp32 states per segment (its two maps and
    # its start state); a scan run in two halves adds two fp32 states per chain
    lm = _ptil(16, 2048, 6, 128, 4) + 2 * 16 * 6 * 128 * 128 * 4
    assert prism.workspace_size(16, 2048, 6, 128, 128, 4, 4, 64, 0) == lm    # 130M-LM layer: two halves
    assert _ptil(16, 2048, 6, 128, 4) == 144 << 20
    assert prism.workspace_size(128, 1024, 2, 64, 64, 4, 4, 64, 0) == _ptil(128, 1024, 2, 64, 4)  # recsys: 256 chains
    assert prism.workspace_size(16, 2048, 6, 128, 128, 1, 4, 64, 0) == 0   # L = 1: no residual writes
    assert prism.workspace_size(16, 448, 6, 128, 128, 4, 4, 64, 0) == _ptil(16, 448, 6, 128, 4)  # 7 chunks: one launch
    P = _segments(1, 65536, 8)
    assert P == 18
    assert prism.workspace_size(1, 65536, 8, 128, 128, 8, 4, 64, 0) == \
        _ptil(1, 65536, 8, 128, 8) + 3 * 8 * P * 128 * 128 * 4
    assert prism.workspace_size(2, 4096, 1, 64, 64, 2, 4, 64, 0) == \
        _ptil(2, 4096, 1, 64, 2) + 3 * 2 * _segments(2, 4096, 1) * 64 * 64 * 4
    assert prism.workspace_size(1, 3, 1, 64, 64, 2, 4, 64, 0) == 512   # 384 bytes, rounded up to 256
    assert prism.workspace_size(16, 2048, 6, 128, 128, 4, 4, 64, 1) == 0   # fp32: token-by-token kernel
    assert prism.workspace_size(0, 64, 8, 128, 128, 4, 4, 64, 0) == 0       # invalid sizes


def test_launch_count_query(L):
    # residual-write launch + one scan; a cut sequence: three scans and a fold instead;
    # chains that leave SMs idle: two halves (two residual writes, two scans)
    assert prism.scan_fwd_launches(16, 2048, 6, 128, 128, 4, 4, 64, 0) == 4
    assert prism.scan_fwd_launches(128, 1024, 2, 64, 64, 4, 4, 64, 0) == 2
    assert prism.scan_fwd_launches(16, 448, 6, 128, 128, 4, 4, 64, 0) == 2
    assert prism.scan_fwd_launches(16, 2048, 6, 128, 128, 1, 4, 64, 0) == 1
    assert prism.scan_fwd_launches(1, 65536, 8, 128, 128, 8, 4, 64, 0) == 5
    assert prism.scan_fwd_launches(1, 65536, 8, 128, 128, 1, 4, 64, 0) == 4
    assert prism.scan_fwd_launches(16, 2048, 6, 128, 128, 4, 4, 64, 1) == 1   # token-by-token
    assert prism.scan_fwd_launches(16, 2048, 6, 128, 128, 4, 4, 32, 0) == 1
    assert prism.scan_fwd_launches(0, 2048, 6, 128, 128, 4, 4, 64, 0) == 0


def test_split_point_query():
    # the first of the two halves ends where the second half's residual write (on the SMs
    # the chains leave idle) should end about when the first scan does: x = 0.28 chains /
    # idle SMs, ceil(NC x / (1 + x)) chunks, clamped to [ceil(NC / 4), NC - 1]
    import math

    def model(B, T, H):
        nc, chains = -(-T // 64), B * H
        x = 0.28 * chains / (148 - chains)
        return max(-(-nc // 4), min(nc - 1, math.ceil(nc * x / (1 + x))))

    assert prism.scan_fwd_split_chunks(16, 2048, 6, 128, 128, 4, 4, 64, 0) == 11 == model(16, 2048, 6)
    assert prism.scan_fwd_split_chunks(31, 2048, 4, 64, 64, 3, 4, 64, 0) == model(31, 2048, 4) > 16
    assert prism.scan_fwd_split_chunks(1, 700, 4, 64, 64, 6, 8, 64, 0) == 3  # a quarter of 11 chunks
    for args in ((128, 1024, 2, 64, 64, 4, 4, 64, 0),      # more chains than idle SMs allow
                 (16, 448, 6, 128, 128, 4, 4, 64, 0),      # under 8 chunks
                 (16, 2048, 6, 128, 128, 1, 4, 64, 0),     # L = 1
                 (1, 65536, 8, 128, 128, 8, 4, 64, 0),     # cut into segments
                 (16, 2048, 6, 64, 64, 4, 4, 64, 1),       # fp32: a CUDA-core path
                 (0, 2048, 6, 128, 128, 4, 4, 64, 0)):     # invalid
        assert prism.scan_fwd_split_chunks(*args) == 0


def test_segment_states_stay_within_148_chains(L):
    # chains x segments never exceeds 148, so the segment (or hand-over) states never need
    # more than 3 x 148 x 128^2 fp32 beyond the residual write vectors
    worst = 0
    for B in (1, 2, 3, 5, 8, 37, 74):
        for H in (1, 2, 4, 8):
            for T in (64, 2047, 2048, 65536, 1 << 20):
                extra = prism.workspace_size(B, T, H, 128, 128, 8, 4, 64, 0) - _ptil(B, T, H, 128, 8)
                worst = max(worst, extra)
    assert 0 < worst <= 3 * 148 * 128 * 128 * 4


def test_missing_workspace_is_rejected_before_launch(L):
    # a cut sequence needs a workspace; without one the call fails before any launch
    assert L.prism_scan_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None,
                            1, 65536, 8, 128, 128, 8, 4, 64, 0, FAKE, None, None, 0, None) == 3


def test_prologue_invalid_arguments(L):
    rc = L.prism_prologue_fwd(FAKE, FAKE, FAKE, FAKE, None, 2, 8, 2, 64, 1, 4, 0, FAKE, None)
    assert rc == 1   # L must be >= 2
    rc = L.prism_prologue_fwd(FAKE, FAKE, FAKE, FAKE, None, 2, 8, 2, 64, 4, 4, 0, FAKE + 4, None)
    assert rc == 2   # misaligned output


def test_host_entry_invalid_arguments(L):
    args = [FAKE] * 11 + [FAKE] * 11 + [2, 8, 2, 64, 64, 4, 4, 64, 0] + [FAKE, FAKE, FAKE, FAKE, None, 0, None]
    bad = list(args)
    bad[0] = None      # host q
    assert L.prism_scan_fwd_host(*bad) == 1
    bad = list(args)
    bad[22] = 0        # B = 0
    assert L.prism_scan_fwd_host(*bad) == 1


def test_unknown_residual_chain_is_rejected(L):
    a = [FAKE] * 9 + [None, None, 2, 8, 2, 64, 64, 4, 4, 64, 0, FAKE, None, None, 0, None]
    for chain in (-1, 2, 7):
        assert L.prism_scan_fwd_ex(*a, chain, None) == 1
        assert L.prism_prologue_fwd_ex(FAKE, FAKE, FAKE, FAKE, None, 2, 8, 2, 64, 4, 4, 0, FAKE, None, chain) == 1
    with pytest.raises(ValueError):
        prism._lib._chain_code("tanh")


def test_conv_state_alignment_is_checked_before_launch(L):
    # B=2 T=8 H=2 d=64 L=4 W=4 bf16, no workspace: a misaligned history is rejected first
    a = [FAKE] * 9 + [None, None, 2, 8, 2, 64, 64, 4, 4, 64, 0, FAKE, None, None, 0, None, 0]
    assert L.prism_scan_fwd_ex(*a, FAKE + 4) == 2
    assert L.prism_scan_fwd_ex(*a, FAKE) == 3          # aligned: then the missing workspace
    w1 = list(a)
    w1[17] = 1                                          # W = 1: no history to read, ignored
    assert L.prism_scan_fwd_ex(*w1, FAKE + 4) == 3


def decode_call(lib_, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, gamma=FAKE, beta=FAKE, u=FAKE, alpha=FAKE, gain=FAKE, conv_w=FAKE,
             conv_state=FAKE, S=FAKE, B=2, H=2, d_k=64, d_v=64, L=4, W=4, dtype=0, chain=0, o=FAKE)
    a.update(kw)
    return lib_.prism_decode_step(a["q"], a["k"], a["v"], a["gamma"], a["beta"], a["u"], a["alpha"], a["gain"],
                                  a["conv_w"], a["conv_state"], a["S"], a["B"], a["H"], a["d_k"], a["d_v"],
                                  a["L"], a["W"], a["dtype"], a["chain"], a["o"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), 1), (dict(H=0), 1), (dict(L=0), 1), (dict(W=0), 1), (dict(dtype=3), 1), (dict(chain=2), 1),
    (dict(S=None), 1), (dict(o=None), 1), (dict(conv_state=None), 1), (dict(u=None), 1), (dict(gain=None), 1),
    (dict(d_k=48), 2), (dict(d_v=256), 2), (dict(L=17), 2), (dict(W=9), 2), (dict(S=FAKE + 4), 2),
    (dict(conv_state=FAKE + 2), 2),
])
def test_decode_invalid_arguments(L, kw, code):
    assert decode_call(L, **kw) == code


def test_decode_optional_inputs(L):
    # W = 1 needs no history and L = 1 no residual inputs: with those NULL the only
    # error left is the size error planted here.
    assert decode_call(L, W=1, conv_state=None, L=1, u=None, alpha=None, gain=None, B=0) == 1


def bwd_call(lib_, ws_ok=True, **kw):
    a = dict(B=2, T=8, H=2, d_k=64, d_v=64, L=4, W=4, dtype=0, chain=0, q=FAKE, dO=FAKE, dq=FAKE, du=FAKE)
    a.update(kw)
    ws, wsb = (FAKE, 1 << 40) if ws_ok else (None, 0)
    return lib_.prism_scan_bwd(a["q"], FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, a["dO"], None,
                               a["B"], a["T"], a["H"], a["d_k"], a["d_v"], a["L"], a["W"], a["dtype"], a["chain"],
                               a["dq"], FAKE, FAKE, FAKE, FAKE, a["du"], FAKE, FAKE, FAKE, FAKE, ws, wsb, None)


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), 1), (dict(L=0), 1), (dict(chain=3), 1), (dict(dtype=5), 1), (dict(dO=None), 1), (dict(dq=None), 1),
    (dict(du=None), 1), (dict(d_k=48), 2), (dict(L=17), 2), (dict(q=FAKE + 4), 2), (dict(ws_ok=False), 3),
])
def test_backward_invalid_arguments(L, kw, code):
    assert bwd_call(L, **kw) == code


def test_backward_workspace_size(L):
    al = lambda x: (x + 255) // 256 * 256
    # token-by-token path (d_k != d_v here): every state S_t (fp32) + dconv_w partials +
    # per-token row-block sums, each 256-byte aligned
    B, T, H, dk, dv, Lc, W = 2, 10, 3, 64, 32, 4, 4
    nv = (Lc + 1) * dk + (Lc + 1)
    expect = al(B * H * T * dv * dk * 4) + al(B * H * dv * W * 4) + al(B * T * H * 1 * nv * 4)
    assert prism.lib().prism_scan_bwd_workspace_size(B, T, H, dk, dv, Lc, W, 0) == expect
    # chunked path (d_k = d_v = 64, L <= 4): boundary states (NC + 1 per chain), H_n (NC per
    # chain), psi, gk, gu per token, <H_n, S_{n+1}> row partials, per-chunk dconv partials
    B, T, H, d, Lc, W = 2, 130, 3, 64, 4, 4
    NC = 3
    expect = (al(B * H * (NC + 1) * d * d * 4) + al(B * H * NC * d * d * 4) + al(B * T * H * d * 4) * 2 +
              al(B * T * H * (Lc - 1) * d * 4) + al(B * H * NC * d * 4) + al(B * NC * H * d * W * 4))
    assert prism.lib().prism_scan_bwd_workspace_size(B, T, H, d, d, Lc, W, 0) == expect
    # far smaller than recording every state: 9.6 MB against 134 MB at T = 2048, B = H = 1, d = 128
    assert prism.lib().prism_scan_bwd_workspace_size(1, 2048, 1, 128, 128, 4, 4, 0) < 10_000_000


def test_state_affine_rejects_bad_arguments_before_any_launch(L):
    F = 0x10000  # never dereferenced: every call below fails before a CUDA call
    f = L.prism_state_affine
    assert f(None, F, F, F, 4, 64, 64, None) == 1          # S missing
    assert f(F, None, F, F, 4, 64, 64, None) == 1          # M missing
    assert f(F, F, F, None, 4, 64, 64, None) == 1          # out missing
    assert f(F, F, F, F, 0, 64, 64, None) == 1             # no (batch, head)
    assert f(F, F + 64, F, F + 64, 4, 64, 64, None) == 1   # out aliases M
    assert f(F, F, F, F + 64, 4, 48, 64, None) == 2        # d_v not a supported head size
    assert f(F, F, F, F + 64, 70000, 64, 64, None) == 2    # more (batch, head) pairs than one grid axis
    # out overlapping an input anywhere but exactly at S or N: read after write, rejected
    S, M, N = 0x100000, 0x200000, 0x300000  # 64 KB regions: BH = 1, d = 128, fp32
    assert f(S, M, N, S + 256, 1, 128, 128, None) == 1      # out inside S at an offset
    assert f(S, M, N, N + 64, 1, 128, 128, None) == 1       # out inside N at an offset
    assert f(S, M, N, M - 4096, 1, 128, 128, None) == 1     # out's tail covers the start of M
    assert f(S, M, None, S - 65536 + 16, 1, 128, 128, None) == 1  # out's tail covers the start of S
