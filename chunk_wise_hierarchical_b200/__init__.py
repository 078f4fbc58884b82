"""HiLS-Attention forward pass on NVIDIA B200 (sm_100a).

The product is the C-ABI library libhils.so (CUDA kernels under csrc/, ABI in
include/hils.h).  This package is its thin Python binding: torch tensors in,
raw device pointers out, nothing computed in Python.
"""
from ._abi import (  # noqa: F401
    HilsError,
    Prefill,
    Decode,
    attend,
    attend_selected,
    backward,
    new_workspace,
    OP_SELECT,
    OP_ATTEND,
    OP_DECODE,
    OP_ATTEND_SELECTED,
    OP_BACKWARD,
    decode,
    decode_static,
    device_status,
    set_wait_limit,
    DEFAULT_WAIT_LIMIT,
    select,
    summarize,
    summarize_paged,
    workspace_size,
    make_shape,
    lib,
    LIB_PATH,
    EXPORTED,
)
