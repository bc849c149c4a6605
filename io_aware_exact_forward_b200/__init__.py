"""io_aware_exact_forward_b200 -- exact IO-aware attention for B200 (sm_100a).

The computation lives in libfa.so (hand-written CUDA kernels behind the C ABI
of include/fa.h); this package only marshals torch tensors into that ABI.
"""

from ._binding import (  # noqa: F401
    FAError,
    LIB_PATH,
    SIGNATURES,
    STATUS,
    backward,
    backward_dropout,
    backward_workspace_bytes,
    check,
    decode_merge,
    decode_splitkv,
    decode_splitkv_noalloc,
    decode_splitkv_partial,
    decode_workspace_bytes,
    forward,
    forward_dropout,
    forward_fp8,
    load_library,
    selftest_bounded_wait,
)
from .context_parallel import decode_splitkv_cp  # noqa: F401,E402
