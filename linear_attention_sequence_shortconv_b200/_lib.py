"""ctypes binding of ``libprism.so`` (argument marshalling only).

Every step of the scan runs in the library's CUDA kernels; this module only
checks tensor dtypes/devices, allocates outputs with torch and passes raw
pointers plus torch's current stream.  There is no CPU fallback: if the
library is missing or the tensors are not on a CUDA device, the calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# PRISM_DEBUG_BOUNDS=1 in the environment loads the debug build (bounds-checked kernels)
DEBUG_BOUNDS = os.environ.get("PRISM_DEBUG_BOUNDS", "0") not in ("", "0")
LIB_PATH = os.path.join(_PKG, "libprism_debug.so" if DEBUG_BOUNDS else "libprism.so")

PRISM_BF16 = 0
PRISM_FP32 = 1
PRISM_CHAIN_LINEAR = 0
PRISM_CHAIN_GELU = 1
STATUS = {
    0: "PRISM_OK",
    1: "PRISM_ERR_INVALID_ARG",
    2: "PRISM_ERR_UNSUPPORTED",
    3: "PRISM_ERR_WORKSPACE",
    4: "PRISM_ERR_CUDA",
    5: "PRISM_ERR_TIMEOUT",
    6: "PRISM_ERR_BOUNDS",
}

# Every symbol include/prism.h declares.
EXPORTS = (
    "prism_scan_fwd",
    "prism_scan_fwd_ex",
    "prism_scan_fwd_workspace_size",
    "prism_scan_fwd_host",
    "prism_scan_fwd_static",
    "prism_prologue_fwd",
    "prism_prologue_fwd_ex",
    "prism_decode_step",
    "prism_scan_bwd",
    "prism_scan_bwd_workspace_size",
    "prism_state_affine",
    "prism_scan_fwd_uses_tensor_cores",
    "prism_scan_fwd_launches",
    "prism_scan_fwd_split_chunks",
    "prism_stream_status",
    "prism_set_spin_limit",
    "prism_set_split_event",
    "prism_status_string",
    "prism_version",
    "prism_debug_bounds",
    "prism_debug_bounds_probe",
)


class PrismError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)} ({status_string(code)})")


_lib = None


def lib() -> ctypes.CDLL:
    """Load the library once (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m linear_attention_sequence_shortconv_b200.build` (needs nvcc)")
    L = ctypes.CDLL(LIB_PATH)
    vp, fp, i32p = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
    ci, cs = ctypes.c_int, ctypes.c_size_t
    L.prism_scan_fwd.argtypes = [vp, vp, vp, fp, fp, vp, fp, vp, fp, fp, i32p,
                                 ci, ci, ci, ci, ci, ci, ci, ci, ci, vp, fp, vp, cs, vp]
    L.prism_scan_fwd.restype = ci
    L.prism_scan_fwd_ex.argtypes = L.prism_scan_fwd.argtypes + [ci, vp]
    L.prism_scan_fwd_ex.restype = ci
    L.prism_scan_fwd_workspace_size.argtypes = [ci] * 9
    L.prism_scan_fwd_workspace_size.restype = cs
    L.prism_scan_fwd_host.argtypes = ([vp] * 11 + [vp] * 11 + [ci] * 9 + [vp, vp, vp, vp, vp, cs, vp])
    L.prism_scan_fwd_host.restype = ci
    L.prism_scan_fwd_static.argtypes = [vp, vp, vp, fp, fp, vp, fp, vp, fp, fp, i32p,
                                        ci, ci, ci, ci, ci, ci, ci, ci, ci, vp, fp, vp, ci, vp]
    L.prism_scan_fwd_static.restype = ci
    L.prism_prologue_fwd.argtypes = [vp, fp, vp, fp, i32p, ci, ci, ci, ci, ci, ci, ci, fp, vp]
    L.prism_prologue_fwd.restype = ci
    L.prism_prologue_fwd_ex.argtypes = L.prism_prologue_fwd.argtypes + [ci]
    L.prism_prologue_fwd_ex.restype = ci
    L.prism_decode_step.argtypes = [vp] * 11 + [ci] * 8 + [vp, vp]
    L.prism_decode_step.restype = ci
    L.prism_scan_bwd_workspace_size.argtypes = [ci] * 8
    L.prism_scan_bwd_workspace_size.restype = cs
    L.prism_scan_bwd.argtypes = [vp] * 13 + [ci] * 9 + [vp] * 11 + [cs, vp]
    L.prism_scan_bwd.restype = ci
    L.prism_state_affine.argtypes = [fp, fp, fp, fp, ci, ci, ci, vp]
    L.prism_state_affine.restype = ci
    L.prism_scan_fwd_uses_tensor_cores.argtypes = [ci] * 6
    L.prism_scan_fwd_uses_tensor_cores.restype = ci
    L.prism_scan_fwd_launches.argtypes = [ci] * 9
    L.prism_scan_fwd_launches.restype = ci
    L.prism_scan_fwd_split_chunks.argtypes = [ci] * 9
    L.prism_scan_fwd_split_chunks.restype = ci
    L.prism_stream_status.argtypes = [vp]
    L.prism_stream_status.restype = ci
    L.prism_set_spin_limit.argtypes = [ctypes.c_longlong]
    L.prism_set_spin_limit.restype = None
    L.prism_set_split_event.argtypes = [vp]
    L.prism_set_split_event.restype = None
    L.prism_status_string.argtypes = [ci]
    L.prism_status_string.restype = ctypes.c_char_p
    L.prism_version.argtypes = []
    L.prism_version.restype = ci
    L.prism_debug_bounds.argtypes = []
    L.prism_debug_bounds.restype = ci
    L.prism_debug_bounds_probe.argtypes = [ctypes.c_longlong, ctypes.c_longlong, vp]
    L.prism_debug_bounds_probe.restype = ci
    _lib = L
    return L


def status_string(code: int) -> str:
    return lib().prism_status_string(int(code)).decode()


def version() -> Tuple[int, int, int]:
    v = lib().prism_version()
    return (v >> 16) & 0xFF, (v >> 8) & 0xFF, v & 0xFF


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return PRISM_BF16
    if t.dtype == torch.float32:
        return PRISM_FP32
    raise TypeError(f"q/k/v/u/gain must be bfloat16 or float32, got {t.dtype}")


CHAINS = {"linear": PRISM_CHAIN_LINEAR, "gelu": PRISM_CHAIN_GELU}


def _chain_code(chain: str) -> int:
    if chain not in CHAINS:
        raise ValueError(f"chain must be one of {sorted(CHAINS)}, got {chain!r}")
    return CHAINS[chain]


def _check(t: Optional[torch.Tensor], name: str, dtype=None, required=True, shape=None, device=None):
    """Validate one tensor argument: CUDA, contiguous, dtype, and (when given) the exact
    shape and the device every other argument of the call is on."""
    if t is None:
        if required:
            raise ValueError(f"{name} is required")
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, but the call's tensors are on {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _call_device(first: torch.Tensor, stream) -> torch.device:
    """The device a call runs on: that of its first tensor argument.  The library launches
    on the current CUDA device, so every entry point below runs inside
    ``torch.cuda.device(dev)``; a stream passed in must belong to the same device."""
    if not isinstance(first, torch.Tensor) or not first.is_cuda:
        raise ValueError("the first tensor argument must be a CUDA tensor (the library has no CPU path)")
    dev = first.device
    if stream is not None and stream.device != dev:
        raise ValueError(f"stream belongs to {stream.device}, but the call's tensors are on {dev}")
    return dev


def workspace_size(B, T, H, d_k, d_v, L, W, chunk, dtype_code) -> int:
    return int(lib().prism_scan_fwd_workspace_size(B, T, H, d_k, d_v, L, W, chunk, dtype_code))


def _scan_checks(q, k, v, gamma, beta, u, alpha, gain, conv_w, L, S0, lengths, o, S_final, want_state,
                 stream, conv_state=None):
    """Argument checks shared by scan_fwd and scan_fwd_static; returns the sizes, the
    device and the (allocated when missing) outputs."""
    dev = _call_device(q, stream)
    dt = q.dtype
    code = _dtype_code(q)
    if q.dim() != 4 or v.dim() != 4 or conv_w.dim() != 3:
        raise ValueError("q, k, v must be [B, T, H, d] and conv_w [H, d_v, W]")
    B, T, H, d_k = q.shape
    d_v = v.shape[-1]
    W = conv_w.shape[-1]
    m = L - 1
    _check(q, "q", dt, device=dev)
    _check(k, "k", dt, shape=(B, T, H, d_k), device=dev)
    _check(v, "v", dt, shape=(B, T, H, d_v), device=dev)
    _check(gamma, "gamma", torch.float32, shape=(B, T, H), device=dev)
    _check(beta, "beta", torch.float32, shape=(B, T, H), device=dev)
    _check(conv_w, "conv_w", torch.float32, shape=(H, d_v, W), device=dev)
    if L > 1:
        _check(u, "u", dt, shape=(B, T, H, m, d_k), device=dev)
        _check(gain, "gain", dt, shape=(B, T, H, m, d_v), device=dev)
        _check(alpha, "alpha", torch.float32, shape=(B, T, H, m), device=dev)
    _check(S0, "S0", torch.float32, required=False, shape=(B, H, d_v, d_k), device=dev)
    _check(lengths, "lengths", torch.int32, required=False, shape=(B,), device=dev)
    if W > 1:
        _check(conv_state, "conv_state", dt, required=False, shape=(B, H, W - 1, d_v), device=dev)
    if o is None:
        o = torch.empty((B, T, H, d_v), dtype=dt, device=dev)
    else:
        _check(o, "o", dt, shape=(B, T, H, d_v), device=dev)
    if want_state:
        if S_final is None:
            S_final = torch.empty((B, H, d_v, d_k), dtype=torch.float32, device=dev)
        else:
            _check(S_final, "S_final", torch.float32, shape=(B, H, d_v, d_k), device=dev)
    return (B, T, H, d_k, d_v, W, code), dev, o, S_final


def scan_fwd(q, k, v, gamma, beta, u, alpha, gain, conv_w, L: int, chunk: int = 64,
             S0=None, lengths=None, want_state: bool = True, o=None, S_final=None,
             workspace=None, stream=None, chain: str = "linear", conv_state=None):
    """PRISM mixer forward on CUDA tensors; returns (o, S_final or None).

    ``chain`` picks the residual chain step: "linear" r <- (1 - g) r, or "gelu"
    r <- r - GELU(g r) (exact erf GELU; ``gain`` then holds the predictor p).

    Shapes as in include/prism.h: q, k [B,T,H,d_k]; v [B,T,H,d_v]; gamma, beta
    [B,T,H] fp32; u [B,T,H,L-1,d_k]; alpha [B,T,H,L-1] fp32; gain [B,T,H,L-1,d_v];
    conv_w [H,d_v,W] fp32; S0 [B,H,d_v,d_k] fp32 or None; lengths [B] int32 or None;
    conv_state [B,H,W-1,d_v] (the I/O dtype) or None: the values of v before token 0,
    oldest first, that the first ShortConv anchors read (None: zeros).
    Every tensor must be on one CUDA device; the call runs on that device.
    """
    chain_code = _chain_code(chain)
    (B, T, H, d_k, d_v, W, code), dev, o, S_final = _scan_checks(
        q, k, v, gamma, beta, u, alpha, gain, conv_w, L, S0, lengths, o, S_final, want_state, stream, conv_state)
    with torch.cuda.device(dev):
        ws_bytes = workspace_size(B, T, H, d_k, d_v, L, W, chunk, code)
        if ws_bytes and workspace is None:
            workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        if workspace is not None:
            _check(workspace, "workspace", torch.uint8, device=dev)
        rc = lib().prism_scan_fwd_ex(
            _ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta),
            _ptr(u if L > 1 else None), _ptr(alpha if L > 1 else None), _ptr(gain if L > 1 else None),
            _ptr(conv_w), _ptr(S0), _ptr(lengths),
            B, T, H, d_k, d_v, L, W, chunk, code,
            _ptr(o), _ptr(S_final if want_state else None),
            _ptr(workspace), workspace.numel() if workspace is not None else 0, _stream_handle(stream),
            chain_code, _ptr(conv_state if W > 1 else None))
    if rc != 0:
        raise PrismError(rc, "prism_scan_fwd_ex")
    return o, (S_final if want_state else None)


def scan_fwd_static(q, k, v, gamma, beta, u, alpha, gain, conv_w, L: int, chunk: int = 64,
                    S0=None, lengths=None, want_state: bool = True, o=None, S_final=None,
                    stream=None, chain: str = "linear", conv_state=None):
    """scan_fwd through prism_scan_fwd_static: no workspace argument, and the library
    allocates nothing (its scratch is a device-global array); returns (o, S_final)."""
    chain_code = _chain_code(chain)
    (B, T, H, d_k, d_v, W, code), dev, o, S_final = _scan_checks(
        q, k, v, gamma, beta, u, alpha, gain, conv_w, L, S0, lengths, o, S_final, want_state, stream, conv_state)
    with torch.cuda.device(dev):
        rc = lib().prism_scan_fwd_static(
            _ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta),
            _ptr(u if L > 1 else None), _ptr(alpha if L > 1 else None), _ptr(gain if L > 1 else None),
            _ptr(conv_w), _ptr(S0), _ptr(lengths),
            B, T, H, d_k, d_v, L, W, chunk, code,
            _ptr(o), _ptr(S_final if want_state else None), _stream_handle(stream), chain_code,
            _ptr(conv_state if W > 1 else None))
    if rc != 0:
        raise PrismError(rc, "prism_scan_fwd_static")
    return o, (S_final if want_state else None)


def scan_fwd_host(host: dict, dev: dict, L: int, chunk: int = 64, stream=None):
    """The host-buffer entry point: ``host`` holds pinned CPU tensors (inputs and
    the outputs ``o``/``S_final``), ``dev`` CUDA tensors of the same shapes (and
    optionally ``workspace``, allocated here when missing).  Enqueues H2D copies,
    the scan and D2H copies on ``stream``; does not sync."""
    names = ("q", "k", "v", "gamma", "beta", "u", "alpha", "gain", "conv_w", "S0", "lengths")
    q = host["q"]
    B, T, H, d_k = q.shape
    d_v = host["v"].shape[-1]
    W = host["conv_w"].shape[-1]
    code = _dtype_code(q)
    device = _call_device(dev["o"], stream)
    for n in names + ("o", "S_final"):
        h = host.get(n)
        if h is None:
            continue
        if h.is_cuda or not h.is_contiguous():
            raise ValueError(f"host[{n!r}] must be a contiguous CPU tensor (pinned for asynchronous copies)")
        _check(dev.get(n), f"dev[{n!r}]", h.dtype, shape=h.shape, device=device)
    ws_bytes = workspace_size(B, T, H, d_k, d_v, L, W, chunk, code)
    ws = dev.get("workspace")
    with torch.cuda.device(device):
        if ws_bytes and ws is None:
            ws = torch.empty(ws_bytes, dtype=torch.uint8, device=device)
        if ws is not None:
            _check(ws, "dev['workspace']", torch.uint8, device=device)
        rc = lib().prism_scan_fwd_host(
            *[_ptr(host.get(n)) for n in names],
            *[_ptr(dev.get(n) if host.get(n) is not None else None) for n in names],
            B, T, H, d_k, d_v, L, W, chunk, code,
            _ptr(dev["o"]), _ptr(dev.get("S_final")), _ptr(host["o"]), _ptr(host.get("S_final")),
            _ptr(ws), ws.numel() if ws is not None else 0, _stream_handle(stream))
    if rc != 0:
        raise PrismError(rc, "prism_scan_fwd_host")


def prologue_fwd(v, alpha, gain, conv_w, L: int, lengths=None, stream=None, chain: str = "linear"):
    """rho_{t,l} = alpha_{t,l} r_{t,l} as [B,T,H,L-1,d_v] fp32 (CUDA)."""
    chain_code = _chain_code(chain)
    dev = _call_device(v, stream)
    code = _dtype_code(v)
    _check(v, "v", device=dev)
    B, T, H, d_v = v.shape
    W = conv_w.shape[-1]
    _check(gain, "gain", v.dtype, shape=(B, T, H, L - 1, d_v), device=dev)
    _check(alpha, "alpha", torch.float32, shape=(B, T, H, L - 1), device=dev)
    _check(conv_w, "conv_w", torch.float32, shape=(H, d_v, W), device=dev)
    _check(lengths, "lengths", torch.int32, required=False, shape=(B,), device=dev)
    rho = torch.empty((B, T, H, L - 1, d_v), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        rc = lib().prism_prologue_fwd_ex(_ptr(v), _ptr(alpha), _ptr(gain), _ptr(conv_w), _ptr(lengths),
                                         B, T, H, d_v, L, W, code, _ptr(rho), _stream_handle(stream), chain_code)
    if rc != 0:
        raise PrismError(rc, "prism_prologue_fwd_ex")
    return rho


def decode_step(q, k, v, gamma, beta, u, alpha, gain, conv_w, conv_state, S, L: int, o=None,
                stream=None, chain: str = "linear"):
    """One recurrent step for every (b, h) on CUDA tensors; returns o [B,H,d_v].

    q, k [B,H,d_k]; v [B,H,d_v]; gamma, beta [B,H] fp32; u [B,H,L-1,d_k]; alpha
    [B,H,L-1] fp32; gain [B,H,L-1,d_v]; conv_w [H,d_v,W] fp32.  ``conv_state``
    [B,H,W-1,d_v] (v's dtype; None when W = 1) and ``S`` [B,H,d_v,d_k] fp32 are
    updated in place.
    """
    chain_code = _chain_code(chain)
    dev = _call_device(q, stream)
    dt = q.dtype
    code = _dtype_code(q)
    B, H, d_k = q.shape
    d_v = v.shape[-1]
    W = conv_w.shape[-1]
    m = L - 1
    _check(q, "q", dt, device=dev)
    _check(k, "k", dt, shape=(B, H, d_k), device=dev)
    _check(v, "v", dt, shape=(B, H, d_v), device=dev)
    _check(gamma, "gamma", torch.float32, shape=(B, H), device=dev)
    _check(beta, "beta", torch.float32, shape=(B, H), device=dev)
    _check(conv_w, "conv_w", torch.float32, shape=(H, d_v, W), device=dev)
    _check(S, "S", torch.float32, shape=(B, H, d_v, d_k), device=dev)
    if L > 1:
        _check(u, "u", dt, shape=(B, H, m, d_k), device=dev)
        _check(gain, "gain", dt, shape=(B, H, m, d_v), device=dev)
        _check(alpha, "alpha", torch.float32, shape=(B, H, m), device=dev)
    _check(conv_state, "conv_state", dt, required=W > 1, shape=(B, H, W - 1, d_v), device=dev)
    if o is None:
        o = torch.empty((B, H, d_v), dtype=dt, device=dev)
    else:
        _check(o, "o", dt, shape=(B, H, d_v), device=dev)
    with torch.cuda.device(dev):
        rc = lib().prism_decode_step(
            _ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta),
            _ptr(u if L > 1 else None), _ptr(alpha if L > 1 else None), _ptr(gain if L > 1 else None),
            _ptr(conv_w), _ptr(conv_state if W > 1 else None), _ptr(S),
            B, H, d_k, d_v, L, W, code, chain_code, _ptr(o), _stream_handle(stream))
    if rc != 0:
        raise PrismError(rc, "prism_decode_step")
    return o


def state_affine(S, M, N=None, out=None, stream=None):
    """out = S M + N per (batch, head) on CUDA fp32 tensors: S, N [..., d_v, d_k], M
    [..., d_k, d_k] with the same leading dimensions (the composition step of per-segment
    state maps).  N may be None (zero); out may be S or N."""
    dev = _call_device(S, stream)
    _check(S, "S", torch.float32, device=dev)
    _check(M, "M", torch.float32, device=dev)
    _check(N, "N", torch.float32, required=False, device=dev)
    d_v, d_k = S.shape[-2], S.shape[-1]
    if tuple(M.shape) != tuple(S.shape[:-2]) + (d_k, d_k):
        raise ValueError(f"M must be {tuple(S.shape[:-2]) + (d_k, d_k)}, got {tuple(M.shape)}")
    if N is not None and tuple(N.shape) != tuple(S.shape):
        raise ValueError(f"N must be {tuple(S.shape)}, got {tuple(N.shape)}")
    if out is None:
        out = torch.empty_like(S)
    else:
        _check(out, "out", torch.float32, shape=S.shape, device=dev)
    BH = S.numel() // (d_v * d_k)
    with torch.cuda.device(dev):
        rc = lib().prism_state_affine(_ptr(S), _ptr(M), _ptr(N), _ptr(out), BH, d_v, d_k, _stream_handle(stream))
    if rc != 0:
        raise PrismError(rc, "prism_state_affine")
    return out


def scan_bwd(q, k, v, gamma, beta, u, alpha, gain, conv_w, dO, L: int, S0=None, lengths=None, dS_final=None,
             workspace=None, stream=None, chain: str = "linear"):
    """Gradients of <o, dO> + <S_final, dS_final> on CUDA tensors (fp32); returns a dict
    with keys q, k, v, gamma, beta, conv_w, S0 and (L > 1) u, alpha, gain."""
    chain_code = _chain_code(chain)
    (B, T, H, d_k, d_v, W, code), dev, _, _ = _scan_checks(
        q, k, v, gamma, beta, u, alpha, gain, conv_w, L, S0, lengths, dO, None, False, stream)
    _check(dS_final, "dS_final", torch.float32, required=False, shape=(B, H, d_v, d_k), device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    g = {"q": torch.empty(q.shape, **f32), "k": torch.empty(k.shape, **f32), "v": torch.empty(v.shape, **f32),
         "gamma": torch.empty(gamma.shape, **f32), "beta": torch.empty(beta.shape, **f32),
         "conv_w": torch.empty(conv_w.shape, **f32), "S0": torch.empty((B, H, d_v, d_k), **f32)}
    if L > 1:
        g["u"] = torch.empty(u.shape, **f32)
        g["alpha"] = torch.empty(alpha.shape, **f32)
        g["gain"] = torch.empty(gain.shape, **f32)
    ws_bytes = int(lib().prism_scan_bwd_workspace_size(B, T, H, d_k, d_v, L, W, code))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    else:
        _check(workspace, "workspace", torch.uint8, device=dev)
    with torch.cuda.device(dev):
        rc = lib().prism_scan_bwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta),
            _ptr(u if L > 1 else None), _ptr(alpha if L > 1 else None), _ptr(gain if L > 1 else None),
            _ptr(conv_w), _ptr(S0), _ptr(lengths), _ptr(dO), _ptr(dS_final),
            B, T, H, d_k, d_v, L, W, code, chain_code,
            _ptr(g["q"]), _ptr(g["k"]), _ptr(g["v"]), _ptr(g["gamma"]), _ptr(g["beta"]),
            _ptr(g.get("u")), _ptr(g.get("alpha")), _ptr(g.get("gain")), _ptr(g["conv_w"]), _ptr(g["S0"]),
            _ptr(workspace), workspace.numel(), _stream_handle(stream))
    if rc != 0:
        raise PrismError(rc, "prism_scan_bwd")
    return g


def uses_tensor_cores(d_k, d_v, L, W, chunk, dtype_code) -> bool:
    """True if prism_scan_fwd runs these sizes on the tcgen05 chunk kernel."""
    return bool(lib().prism_scan_fwd_uses_tensor_cores(d_k, d_v, L, W, chunk, dtype_code))


def scan_fwd_launches(B, T, H, d_k, d_v, L, W, chunk, dtype_code) -> int:
    """Kernel launches one prism_scan_fwd call with these sizes issues."""
    return int(lib().prism_scan_fwd_launches(B, T, H, d_k, d_v, L, W, chunk, dtype_code))


def scan_fwd_split_chunks(B, T, H, d_k, d_v, L, W, chunk, dtype_code) -> int:
    """Chunks in the first scan launch when the forward runs in two halves, else 0."""
    return int(lib().prism_scan_fwd_split_chunks(B, T, H, d_k, d_v, L, W, chunk, dtype_code))


def set_split_event(event) -> None:
    """Measurement hook: the next tensor-core forward with L > 1 records ``event`` (a
    torch.cuda.Event that has been recorded once, so that it exists) between its
    residual-write launch and its scan.  None clears it."""
    lib().prism_set_split_event(None if event is None else ctypes.c_void_p(event.cuda_event))


def stream_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return int(lib().prism_stream_status(_stream_handle(stream)))


def set_spin_limit(limit: int) -> None:
    lib().prism_set_spin_limit(int(limit))
