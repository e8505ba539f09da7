"""BASED hot path on B200: causal Taylor linear attention + sliding-window attention,
plus the short gated convolution (BaseConv) mixer.

The computation lives in libbased.so (hand-written sm_100a CUDA kernels behind
the C ABI of include/based.h); this package is its ctypes binding. Importing it
does not need a GPU; calling an op does.
"""

from .binding import (  # noqa: F401
    BasedError,
    SYMBOLS,
    feature_dim,
    packed_dim,
    get_last_error,
    la_backward,
    la_backward_workspace,
    la_decode_step,
    la_decode_step_decay,
    la_prefill,
    la_prefill_decay,
    la_prefill_noalloc,
    la_prefill_workspace,
    lib,
    library_path,
    status_string,
    swa_decode,
    baseconv_prefill,
    baseconv_decode,
    swa_prefill,
)

__version__ = "0.1.0"
