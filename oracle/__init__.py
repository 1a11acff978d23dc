"""CPU oracle for the PRISM sequence-mixer scan (fp64).

TEST INFRASTRUCTURE: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import it.  The library never does.
"""
from .prism_oracle import (  # noqa: F401
    affine_maps,
    gdn_seq,
    gelu,
    max_abs_rel_err,
    prism_chunked,
    prism_decode_step,
    prism_seq,
    residual_chain,
    residual_write,
    shortconv_anchor,
)
