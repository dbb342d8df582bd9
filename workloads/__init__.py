"""Seeded synthetic inputs for paged latent attention.

This package builds inputs only: page tables, row lengths and random bf16
tensors.  It holds none of the attention arithmetic, and both the oracle-side
tests and the CUDA-side tests/bench draw their inputs from it.
"""

from .configs import (  # noqa: F401
    CONFIG_NAMES,
    MlaInputs,
    make_config,
    make_custom,
    SM_SCALE,
)
