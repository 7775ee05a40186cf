"""fp64 CPU oracle of the Mamba selective scan, the selective state update and
the causal conv front-end of the block's input path.

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check and by the
benchmark's CPU-baseline leg, never by the product package. It shares no code
with the CUDA path. See ``mamba_oracle.c`` for what it computes and which
passage of the Mamba pages each step follows.
"""
from .oracle import (  # noqa: F401
    build_oracle,
    causal_conv,
    conv_scan,
    load_oracle,
    scan,
    scan_bwd,
    scan_mt,
    ssd,
    ssd_chunk_cb,
    state_update,
    softplus,
    silu,
)
