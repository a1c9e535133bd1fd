"""Paged decode attention for NVIDIA B200 (sm_100a).

The library is ``libpa370.so`` (C ABI in ``include/pa.h``): CUDA kernels for
the paged KV write, the copy-on-write block copy and split-context decode
attention with a log-sum-exp merge, plus a host block manager. This package
is its Python binding; PyTorch supplies device memory and streams only.
"""
from .abi import (  # noqa: F401
    BlockManager,
    OutOfBlocks,
    PAError,
    pa_copy_blocks,
    pa_decode,
    pa_decode_default_partition,
    pa_decode_workspace_size,
    pa_device_status,
    pa_reshape_and_cache,
    pa_slot_mapping,
)
