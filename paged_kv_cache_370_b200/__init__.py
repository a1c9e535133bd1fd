"""Paged decode attention for NVIDIA B200 (sm_100a).

The library is ``libpa370.so`` (C ABI in ``include/pa.h``): CUDA kernels for
the paged KV write, the copy-on-write block copy and paged decode attention,
plus a host block manager. This package is its Python binding; PyTorch
supplies device memory and streams only.

Names are resolved from ``abi`` on first use, so that ``build`` can run
before the library exists; using any of them without the library raises.
"""
_EXPORTS = (
    "BlockManager", "OutOfBlocks", "PAError", "pa_copy_blocks", "pa_decode", "pa_decode_append",
    "pa_decode_append_launches",
    "pa_decode_default_partition", "pa_decode_launches", "pa_decode_static_workspace",
    "pa_decode_workspace_size", "pa_device_status", "pa_reshape_and_cache", "pa_slot_mapping",
    "SwapSpace", "pa_swap_out", "pa_swap_in", "pa_decode_window", "pa_decode_append_window",
    "pa_decode_window_launches", "pa_decode_append_window_launches", "pa_prefill", "pa_decode_append_overlapped",
)

__all__ = list(_EXPORTS)


def __getattr__(name):
    if name in _EXPORTS:
        from . import abi
        return getattr(abi, name)
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")
