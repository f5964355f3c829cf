"""Block-sparse exact softmax attention for B200 (sm_100a).

The computation runs in ``libbsa.so`` (CUDA kernels behind the C ABI of
``include/bsa.h``); this package is its thin Python binding.  Importing it does
not load the library; the first call does, and fails loudly if it is missing.
"""

from ._binding import (  # noqa: F401
    BsaError,
    Mask,
    Stages,
    Workspace,
    attn_bwd,
    attn_fwd,
    header_functions,
    launch_count,
    lib,
    plan_build,
    workspace_size,
)
