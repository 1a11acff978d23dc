"""PRISM sequence-mixer scan for NVIDIA B200 (sm_100a).

The compute lives in ``libprism.so`` (hand-written CUDA kernels behind the C
ABI of include/prism.h); this package is its thin Python binding plus the
seeded synthetic input generator.  Build the library with
``python -m linear_attention_sequence_shortconv_b200.build``.
"""
from ._lib import (  # noqa: F401
    EXPORTS,
    PRISM_BF16,
    PRISM_FP32,
    PRISM_CHAIN_GELU,
    PRISM_CHAIN_LINEAR,
    PrismError,
    lib,
    decode_step,
    prologue_fwd,
    scan_bwd,
    scan_fwd,
    scan_fwd_host,
    scan_fwd_static,
    set_spin_limit,
    state_affine,
    status_string,
    stream_status,
    uses_tensor_cores,
    scan_fwd_launches,
    scan_fwd_split_chunks,
    set_split_event,
    version,
    workspace_size,
)
