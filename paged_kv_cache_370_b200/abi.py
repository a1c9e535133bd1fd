"""Thin Python binding of libpa370.so (argument marshalling only).

Every function here has the name of the C entry point it calls (see
``include/pa.h`` for the contract). Device operations take CUDA torch tensors,
derive the sizes the C call needs from their shapes, and pass raw pointers
and the current CUDA stream; all work runs in the library's kernels. There
is no fallback: if ``libpa370.so`` is missing or cannot be loaded, importing
this module raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import LIB_PATH

PA_OK = 0
PA_ERR_INVALID = -1
PA_ERR_OUT_OF_BLOCKS = -2
PA_ERR_STATE = -3
PA_ERR_CUDA = -4
PA_ERR_UNSUPPORTED = -5

PA_F16 = 0
PA_BF16 = 1

PA_DEVERR_BLOCK_ID = 1
PA_DEVERR_SLOT = 2
PA_DEVERR_COPY_PAIR = 4
PA_DEVERR_CONTEXT_LEN = 8
PA_DEVERR_TIMEOUT = 16

PA_STATIC_WORKSPACE_BYTES = 16 << 20


class PAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


class OutOfBlocks(PAError):
    pass


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with "
                          "`python -m paged_kv_cache_370_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, i, i64, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    sigs = {
        "pa_reshape_and_cache": (i, [P, P, P, i, P, P, i, i, i, i, i, P]),
        "pa_copy_blocks": (i, [P, P, P, i, i, i, i, i, i, P]),
        "pa_decode_workspace_size": (sz, [i, i, i, i, i, i]),
        "pa_decode": (i, [P, P, P, P, P, i, P, i, i, i, i, i, i, i, f, i, P, sz, i, P]),
        "pa_decode_default_partition": (i, [i, i, i]),
        "pa_decode_launches": (i, [i, i, i, i, i, i, i, i]),
        "pa_decode_grid_ctas": (i, [i, i, i, i, i, i, i, i]),
        "pa_debug_wait_test": (i, [i, ctypes.c_longlong]),
        "pa_decode_append": (i, [P, P, P, P, P, P, P, P, i, P, i, i, i, i, i, i, i, f, i, P, sz,
                                 i, P]),
        "pa_decode_append_launches": (i, [i, i, i, i, i, i, i, i]),
        "pa_decode_append_overlapped": (i, [P, P, P, P, P, P, P, P, i, P, i, i, i, i, i, i, i, f,
                                            i, P, sz, i, P]),
        "pa_decode_window": (i, [P, P, P, P, P, i, P, i, i, i, i, i, i, i, f, i, i, P, sz, i, P]),
        "pa_decode_window_launches": (i, [i, i, i, i, i, i, i, i, i]),
        "pa_decode_append_window_launches": (i, [i, i, i, i, i, i, i, i, i]),
        "pa_prefill": (i, [P, P, P, P, P, i, P, P, i, i, i, i, i, i, i, i, i, f, i, i, P]),
        "pa_decode_append_window": (i, [P, P, P, P, P, P, P, P, i, P, i, i, i, i, i, i, i, f, i, i,
                                        P, sz, i, P]),
        "pa_decode_append_window_overlapped": (i, [P, P, P, P, P, P, P, P, i, P, i, i, i, i, i, i,
                                                   i, f, i, i, P, sz, i, P]),
        "pa_decode_static_workspace": (i, [P, P, P, P, P, i, P, i, i, i, i, i, i, i, f, i, i, P]),
        "pa_device_status": (i, [P, P]),
        "pa_hbm_read": (i, [P, sz, P, i, P]),
        "pa_status_string": (ctypes.c_char_p, [i]),
        "pa_slot_mapping": (i, [P, i, P, i, i, P]),
        "pa_alloc_create": (i, [i, i, P]),
        "pa_alloc_destroy": (None, [P]),
        "pa_alloc_add_seq": (i, [P, i64, i]),
        "pa_alloc_fork": (i, [P, i64, i64]),
        "pa_alloc_append_slot": (i, [P, i64, P, P, P]),
        "pa_alloc_seq_slots": (i, [P, i64, i, i, P]),
        "pa_alloc_free_seq": (i, [P, i64]),
        "pa_alloc_slide_window": (i, [P, i64, i, P]),
        "pa_alloc_set_host_blocks": (i, [P, i]),
        "pa_swap_space_create": (i, [i, i, i, i, i, P]),
        "pa_swap_space_destroy": (None, [P]),
        "pa_swap_space_pools": (i, [P, P, P]),
        "pa_swap_out": (i, [P, P, P, i, P, i, P]),
        "pa_swap_in": (i, [P, P, P, i, P, i, P]),
        "pa_alloc_swap_out": (i, [P, P, i, P, i, P]),
        "pa_alloc_swap_in": (i, [P, P, i, P, i, P]),
        "pa_alloc_is_swapped": (i, [P, i64, P]),
        "pa_alloc_host_free": (i, [P, P]),
        "pa_alloc_add_seq_cached": (i, [P, i64, P, i, P]),
        "pa_alloc_cached_blocks": (i, [P, P, P]),
        "pa_alloc_reset_prefix_cache": (i, [P]),
        "pa_alloc_block_table": (i, [P, i64, P, i, P, P]),
        "pa_alloc_fill_tables": (i, [P, P, i, P, i, ctypes.c_int32, P]),
        "pa_alloc_ref_count": (i, [P, ctypes.c_int32, P]),
        "pa_alloc_stats": (i, [P, P, P, P]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


_lib = _load()


def lib() -> ctypes.CDLL:
    return _lib


def status_string(status: int) -> str:
    return _lib.pa_status_string(status).decode()


def _check(status: int, what: str):
    if status == PA_ERR_OUT_OF_BLOCKS:
        raise OutOfBlocks(status, what)
    if status != PA_OK:
        raise PAError(status, what)


# ------------------------------------------------------------------------------ device helpers
def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return PA_BF16
    if t.dtype == torch.float16:
        return PA_F16
    raise TypeError(f"unsupported dtype {t.dtype}; expected float16 or bfloat16")


def _dev_ptr(t, what: str):
    if t is None:
        return None
    if not t.is_cuda:
        raise TypeError(f"{what} must be a CUDA tensor")
    if not t.is_contiguous():
        raise TypeError(f"{what} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(_torch().cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def pa_reshape_and_cache(k_new, v_new, slot_mapping, k_cache, v_cache, stream=None):
    """Store k_new/v_new [T, Hkv, D] at slot_mapping[T] (int64) in the pools
    [num_blocks, Hkv, block_size, D]."""
    nb, hkv, bs, d = k_cache.shape
    st = _lib.pa_reshape_and_cache(_dev_ptr(k_new, "k_new"), _dev_ptr(v_new, "v_new"),
                                   _dev_ptr(slot_mapping, "slot_mapping"), int(slot_mapping.numel()),
                                   _dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"), nb,
                                   hkv, bs, d, _dtype_code(k_cache), _stream(stream))
    _check(st, "pa_reshape_and_cache")


def pa_copy_blocks(k_cache, v_cache, block_pairs, stream=None):
    """Copy whole blocks (src -> dst) for every row of block_pairs [P, 2] (int64)."""
    nb, hkv, bs, d = k_cache.shape
    n = int(block_pairs.shape[0]) if block_pairs.numel() else 0
    st = _lib.pa_copy_blocks(_dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"),
                             _dev_ptr(block_pairs, "block_pairs"), n, nb, hkv, bs, d,
                             _dtype_code(k_cache), _stream(stream))
    _check(st, "pa_copy_blocks")


class SwapSpace:
    """Pinned, device-mapped host memory for ``num_host_blocks`` KV blocks
    (pa_swap_space_*). ``k_host`` / ``v_host`` are numpy views of the two host
    pools, [num_host_blocks, num_kv_heads, block_size, head_dim] of 16-bit words."""

    def __init__(self, num_host_blocks: int, num_kv_heads: int, block_size: int, head_dim: int,
                 dtype: str):
        code = {"f16": PA_F16, "bf16": PA_BF16}[dtype]
        h = ctypes.c_void_p()
        _check(_lib.pa_swap_space_create(num_host_blocks, num_kv_heads, block_size, head_dim, code,
                                         ctypes.byref(h)), "pa_swap_space_create")
        self._h = h
        self.shape = (num_host_blocks, num_kv_heads, block_size, head_dim)
        kp, vp = ctypes.c_void_p(), ctypes.c_void_p()
        _check(_lib.pa_swap_space_pools(h, ctypes.byref(kp), ctypes.byref(vp)), "pa_swap_space_pools")
        n = int(np.prod(self.shape))
        self.k_host = np.ctypeslib.as_array((ctypes.c_uint16 * n).from_address(kp.value)).reshape(self.shape)
        self.v_host = np.ctypeslib.as_array((ctypes.c_uint16 * n).from_address(vp.value)).reshape(self.shape)

    def close(self):
        if self._h:
            self.k_host = self.v_host = None
            _lib.pa_swap_space_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # noqa: BLE001 -- interpreter shutdown
            pass


def pa_swap_out(space: SwapSpace, k_cache, v_cache, block_pairs, stream=None):
    """Copy device blocks to host blocks for every (device, host) row of block_pairs."""
    n = int(block_pairs.shape[0]) if block_pairs.numel() else 0
    st = _lib.pa_swap_out(space._h, _dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"),
                          int(k_cache.shape[0]), _dev_ptr(block_pairs, "block_pairs"), n,
                          _stream(stream))
    _check(st, "pa_swap_out")


def pa_swap_in(space: SwapSpace, k_cache, v_cache, block_pairs, stream=None):
    """Copy host blocks to device blocks for every (host, device) row of block_pairs."""
    n = int(block_pairs.shape[0]) if block_pairs.numel() else 0
    st = _lib.pa_swap_in(space._h, _dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"),
                         int(k_cache.shape[0]), _dev_ptr(block_pairs, "block_pairs"), n,
                         _stream(stream))
    _check(st, "pa_swap_in")


def pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                             partition_tokens=0) -> int:
    return int(_lib.pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                             max_context_len, partition_tokens))


def pa_decode_launches(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                       max_context_len, partition_tokens=0) -> int:
    """Kernels one pa_decode call with these arguments launches."""
    return int(_lib.pa_decode_launches(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                       num_blocks, max_context_len, partition_tokens))


def pa_decode_default_partition(num_seqs, num_kv_heads, max_context_len) -> int:
    return int(_lib.pa_decode_default_partition(num_seqs, num_kv_heads, max_context_len))


def pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len, scale,
              workspace=None, partition_tokens=0, stream=None):
    """Paged decode attention: out[B, Hq, D] from q[B, Hq, D], the pools, int32
    block_tables[B, max_blocks_per_seq] and int32 context_lens[B]."""
    B, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = _lib.pa_decode(_dev_ptr(out, "out"), _dev_ptr(q, "q"), _dev_ptr(k_cache, "k_cache"),
                        _dev_ptr(v_cache, "v_cache"), _dev_ptr(block_tables, "block_tables"),
                        int(block_tables.shape[1]), _dev_ptr(context_lens, "context_lens"),
                        int(max_context_len), B, hq, hkv, d, bs, nb, float(scale),
                        _dtype_code(q), _dev_ptr(workspace, "workspace"), ws_bytes,
                        int(partition_tokens), _stream(stream))
    _check(st, "pa_decode")


def pa_decode_window(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len, scale,
                     window, workspace=None, partition_tokens=0, stream=None):
    """pa_decode over each sequence's last ``window`` positions only."""
    B, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = _lib.pa_decode_window(_dev_ptr(out, "out"), _dev_ptr(q, "q"), _dev_ptr(k_cache, "k_cache"),
                               _dev_ptr(v_cache, "v_cache"), _dev_ptr(block_tables, "block_tables"),
                               int(block_tables.shape[1]), _dev_ptr(context_lens, "context_lens"),
                               int(max_context_len), B, hq, hkv, d, bs, nb, float(scale),
                               int(window), _dtype_code(q), _dev_ptr(workspace, "workspace"),
                               ws_bytes, int(partition_tokens), _stream(stream))
    _check(st, "pa_decode_window")


def pa_prefill(out, q, k_cache, v_cache, block_tables, context_lens, q_start, max_q_len,
               max_context_len, scale, window=0, stream=None):
    """Paged prefill attention: out[T, Hq, D] for the query tokens q[T, Hq, D] of every
    sequence (rows q_start[b]:q_start[b+1], the sequence's last positions), causal."""
    T, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    st = _lib.pa_prefill(_dev_ptr(out, "out"), _dev_ptr(q, "q"), _dev_ptr(k_cache, "k_cache"),
                         _dev_ptr(v_cache, "v_cache"), _dev_ptr(block_tables, "block_tables"),
                         int(block_tables.shape[1]), _dev_ptr(context_lens, "context_lens"),
                         _dev_ptr(q_start, "q_start"), int(context_lens.shape[0]), T,
                         int(max_q_len), int(max_context_len), hq, hkv, d, bs, nb, float(scale),
                         int(window), _dtype_code(q), _stream(stream))
    _check(st, "pa_prefill")


def pa_decode_window_launches(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                              num_blocks, max_context_len, window, partition_tokens=0) -> int:
    """Kernels one pa_decode_window call with these arguments launches."""
    return int(_lib.pa_decode_window_launches(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                              block_size, num_blocks, max_context_len, window,
                                              partition_tokens))


def pa_decode_append_window_launches(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                     num_blocks, max_context_len, window,
                                     partition_tokens=0) -> int:
    """Kernels one pa_decode_append_window call with these arguments launches."""
    return int(_lib.pa_decode_append_window_launches(num_seqs, num_q_heads, num_kv_heads,
                                                     head_dim, block_size, num_blocks,
                                                     max_context_len, window, partition_tokens))


def pa_decode_append_window(out, q, k_new, v_new, slot_mapping, k_cache, v_cache, block_tables,
                            context_lens, max_context_len, scale, window, workspace=None,
                            partition_tokens=0, stream=None, overlapped=False):
    """pa_decode_append over each sequence's last ``window`` positions only
    (``overlapped``: pa_decode_append_window_overlapped, the programmatic early
    start of pa_decode_append_overlapped, under the same contract)."""
    B, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    fn = _lib.pa_decode_append_window_overlapped if overlapped else _lib.pa_decode_append_window
    st = fn(
        _dev_ptr(out, "out"), _dev_ptr(q, "q"), _dev_ptr(k_new, "k_new"), _dev_ptr(v_new, "v_new"),
        _dev_ptr(slot_mapping, "slot_mapping"), _dev_ptr(k_cache, "k_cache"),
        _dev_ptr(v_cache, "v_cache"), _dev_ptr(block_tables, "block_tables"),
        int(block_tables.shape[1]), _dev_ptr(context_lens, "context_lens"), int(max_context_len),
        B, hq, hkv, d, bs, nb, float(scale), int(window), _dtype_code(q),
        _dev_ptr(workspace, "workspace"), ws_bytes, int(partition_tokens), _stream(stream))
    _check(st, "pa_decode_append_window")


def pa_decode_append(out, q, k_new, v_new, slot_mapping, k_cache, v_cache, block_tables,
                     context_lens, max_context_len, scale, workspace=None, partition_tokens=0,
                     stream=None):
    """One decode step: store k_new/v_new [B, Hkv, D] at slot_mapping[B] (the token at
    position context_lens[b] - 1), then attend, as pa_reshape_and_cache + pa_decode."""
    B, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = _lib.pa_decode_append(
        _dev_ptr(out, "out"), _dev_ptr(q, "q"), _dev_ptr(k_new, "k_new"), _dev_ptr(v_new, "v_new"),
        _dev_ptr(slot_mapping, "slot_mapping"), _dev_ptr(k_cache, "k_cache"),
        _dev_ptr(v_cache, "v_cache"), _dev_ptr(block_tables, "block_tables"),
        int(block_tables.shape[1]), _dev_ptr(context_lens, "context_lens"), int(max_context_len),
        B, hq, hkv, d, bs, nb, float(scale), _dtype_code(q), _dev_ptr(workspace, "workspace"),
        ws_bytes, int(partition_tokens), _stream(stream))
    _check(st, "pa_decode_append")


def pa_decode_append_overlapped(out, q, k_new, v_new, slot_mapping, k_cache, v_cache,
                                block_tables, context_lens, max_context_len, scale,
                                workspace=None, partition_tokens=0, stream=None):
    """pa_decode_append whose kernel may start during the preceding kernel's tail; the
    lengths, tables and slots must not be written by that preceding kernel."""
    B, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = _lib.pa_decode_append_overlapped(
        _dev_ptr(out, "out"), _dev_ptr(q, "q"), _dev_ptr(k_new, "k_new"), _dev_ptr(v_new, "v_new"),
        _dev_ptr(slot_mapping, "slot_mapping"), _dev_ptr(k_cache, "k_cache"),
        _dev_ptr(v_cache, "v_cache"), _dev_ptr(block_tables, "block_tables"),
        int(block_tables.shape[1]), _dev_ptr(context_lens, "context_lens"), int(max_context_len),
        B, hq, hkv, d, bs, nb, float(scale), _dtype_code(q), _dev_ptr(workspace, "workspace"),
        ws_bytes, int(partition_tokens), _stream(stream))
    _check(st, "pa_decode_append_overlapped")


def pa_decode_append_launches(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                              num_blocks, max_context_len, partition_tokens=0) -> int:
    return int(_lib.pa_decode_append_launches(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                              block_size, num_blocks, max_context_len,
                                              partition_tokens))


def pa_decode_static_workspace(out, q, k_cache, v_cache, block_tables, context_lens,
                               max_context_len, scale, partition_tokens=0, stream=None):
    """pa_decode for callers that cannot allocate device memory: the split-context
    scratch is the library's fixed device array (PA_STATIC_WORKSPACE_BYTES), shared
    by every call. Raises PAError(PA_ERR_UNSUPPORTED) if the call needs more."""
    B, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    st = _lib.pa_decode_static_workspace(
        _dev_ptr(out, "out"), _dev_ptr(q, "q"), _dev_ptr(k_cache, "k_cache"),
        _dev_ptr(v_cache, "v_cache"), _dev_ptr(block_tables, "block_tables"),
        int(block_tables.shape[1]), _dev_ptr(context_lens, "context_lens"), int(max_context_len),
        B, hq, hkv, d, bs, nb, float(scale), _dtype_code(q), int(partition_tokens),
        _stream(stream))
    _check(st, "pa_decode_static_workspace")


def pa_decode_grid_ctas(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                        max_context_len, partition_tokens=0) -> int:
    """CTAs of the even-split kernel such a pa_decode call launches (0: the
    partition kernel runs instead)."""
    return int(_lib.pa_decode_grid_ctas(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                        block_size, num_blocks, max_context_len,
                                        partition_tokens))


def pa_debug_wait_test(enable: bool, consumer_wait_ns: int = 0):
    """Test hook: later decode launches make their bounded data waits run out
    (no copies issued); see include/pa.h. enable=False restores normal launches."""
    _check(_lib.pa_debug_wait_test(1 if enable else 0, int(consumer_wait_ns)),
           "pa_debug_wait_test")


def pa_hbm_read(buf, sink, ctas_per_sm=4, stream=None):
    """Read the device buffer ``buf`` once as a read-only stream (a measurement
    utility); ``sink`` (one int32 on the device) receives the XOR of its 32-bit words."""
    nbytes = buf.numel() * buf.element_size()
    _check(_lib.pa_hbm_read(_dev_ptr(buf, "buf"), nbytes, _dev_ptr(sink, "sink"),
                            int(ctas_per_sm), _stream(stream)), "pa_hbm_read")


def pa_device_status(stream=None) -> int:
    """Read and clear the device-side error word (synchronises the stream)."""
    code = ctypes.c_int32(0)
    _check(_lib.pa_device_status(_stream(stream), ctypes.byref(code)), "pa_device_status")
    return code.value


# -------------------------------------------------------------------------------- host helpers
def _np_ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def pa_slot_mapping(block_tables: np.ndarray, counts, block_size: int) -> np.ndarray:
    """Slots of positions [0, counts[b]) of every sequence, sequence-major (int64)."""
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cnt = np.ascontiguousarray(counts, dtype=np.int32)
    out = np.empty(int(cnt.sum()), dtype=np.int64)
    _check(_lib.pa_slot_mapping(_np_ptr(bt), bt.shape[1], _np_ptr(cnt), len(cnt), block_size,
                                _np_ptr(out)), "pa_slot_mapping")
    return out


class BlockManager:
    """Host block manager: free list, reference counts, copy-on-write (pa_alloc_*)."""

    def __init__(self, num_blocks: int, block_size: int):
        h = ctypes.c_void_p()
        _check(_lib.pa_alloc_create(num_blocks, block_size, ctypes.byref(h)), "pa_alloc_create")
        self._h = h
        self.num_blocks = num_blocks
        self.block_size = block_size

    def close(self):
        if self._h:
            _lib.pa_alloc_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # noqa: BLE001 -- interpreter shutdown
            pass

    def add_seq(self, seq_id: int, num_tokens: int):
        _check(_lib.pa_alloc_add_seq(self._h, seq_id, num_tokens), "pa_alloc_add_seq")

    def add_seq_cached(self, seq_id: int, tokens) -> int:
        """A new sequence holding the prompt ``tokens`` (token ids), sharing the
        leading full blocks whose whole prefix is cached; returns how many
        positions are already in the pool (the caller writes the rest)."""
        tok = np.ascontiguousarray(np.asarray(tokens, dtype=np.int32).reshape(-1))
        n = ctypes.c_int(0)
        _check(_lib.pa_alloc_add_seq_cached(self._h, seq_id, _np_ptr(tok) if len(tok) else None,
                                            len(tok), ctypes.byref(n)),
               "pa_alloc_add_seq_cached")
        return n.value

    def cached_blocks(self) -> tuple[int, int]:
        """(blocks holding a cached prefix, of which free)."""
        c, f = ctypes.c_int(0), ctypes.c_int(0)
        _check(_lib.pa_alloc_cached_blocks(self._h, ctypes.byref(c), ctypes.byref(f)),
               "pa_alloc_cached_blocks")
        return c.value, f.value

    def reset_prefix_cache(self):
        _check(_lib.pa_alloc_reset_prefix_cache(self._h), "pa_alloc_reset_prefix_cache")

    def fork(self, parent: int, child: int):
        _check(_lib.pa_alloc_fork(self._h, parent, child), "pa_alloc_fork")

    def append_slot(self, seq_id: int):
        slot, src, dst = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        _check(_lib.pa_alloc_append_slot(self._h, seq_id, ctypes.byref(slot), ctypes.byref(src),
                                         ctypes.byref(dst)), "pa_alloc_append_slot")
        return slot.value, src.value, dst.value

    def seq_slots(self, seq_id: int, start: int, count: int) -> np.ndarray:
        out = np.empty(count, dtype=np.int64)
        _check(_lib.pa_alloc_seq_slots(self._h, seq_id, start, count, _np_ptr(out)),
               "pa_alloc_seq_slots")
        return out

    def free_seq(self, seq_id: int):
        _check(_lib.pa_alloc_free_seq(self._h, seq_id), "pa_alloc_free_seq")

    def slide_window(self, seq_id: int, window: int) -> int:
        """Release the blocks wholly before the last ``window`` positions; returns
        how many went back on the free list."""
        freed = ctypes.c_int(0)
        _check(_lib.pa_alloc_slide_window(self._h, seq_id, window, ctypes.byref(freed)),
               "pa_alloc_slide_window")
        return freed.value

    def set_host_blocks(self, num_host_blocks: int):
        """Give the manager a host swap space of ``num_host_blocks`` blocks."""
        _check(_lib.pa_alloc_set_host_blocks(self._h, num_host_blocks), "pa_alloc_set_host_blocks")

    def _swap(self, fn, name, seq_ids):
        ids = np.ascontiguousarray(np.asarray(list(seq_ids), dtype=np.int64))
        cap = 0
        for s in ids.tolist():
            cap += len(self.block_table(int(s)))
        pairs = np.zeros((max(cap, 1), 2), dtype=np.int64)
        n = ctypes.c_int(0)
        _check(fn(self._h, _np_ptr(ids), len(ids), _np_ptr(pairs), cap, ctypes.byref(n)), name)
        return pairs[: n.value].copy()

    def swap_out(self, seq_ids) -> np.ndarray:
        """Move a group of sequences to the host swap space; returns the
        (device block, host block) pairs to copy (pa_swap_out)."""
        return self._swap(_lib.pa_alloc_swap_out, "pa_alloc_swap_out", seq_ids)

    def swap_in(self, seq_ids) -> np.ndarray:
        """Bring a swapped group back; returns (host block, device block) pairs
        to copy (pa_swap_in)."""
        return self._swap(_lib.pa_alloc_swap_in, "pa_alloc_swap_in", seq_ids)

    def is_swapped(self, seq_id: int) -> bool:
        v = ctypes.c_int(0)
        _check(_lib.pa_alloc_is_swapped(self._h, seq_id, ctypes.byref(v)), "pa_alloc_is_swapped")
        return bool(v.value)

    def host_free(self) -> int:
        v = ctypes.c_int(0)
        _check(_lib.pa_alloc_host_free(self._h, ctypes.byref(v)), "pa_alloc_host_free")
        return v.value

    def block_table(self, seq_id: int) -> list[int]:
        nb, nt = ctypes.c_int(), ctypes.c_int()
        _check(_lib.pa_alloc_block_table(self._h, seq_id, None, 0, ctypes.byref(nb),
                                         ctypes.byref(nt)), "pa_alloc_block_table")
        out = np.empty(max(nb.value, 1), dtype=np.int32)
        _check(_lib.pa_alloc_block_table(self._h, seq_id, _np_ptr(out), len(out), None, None),
               "pa_alloc_block_table")
        return out[:nb.value].tolist()

    def seq_len(self, seq_id: int) -> int:
        nt = ctypes.c_int()
        _check(_lib.pa_alloc_block_table(self._h, seq_id, None, 0, None, ctypes.byref(nt)),
               "pa_alloc_block_table")
        return nt.value

    def fill_tables(self, seq_ids, max_blocks_per_seq: int, pad: int = 0):
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        tables = np.empty((len(ids), max_blocks_per_seq), dtype=np.int32)
        lens = np.empty(len(ids), dtype=np.int32)
        _check(_lib.pa_alloc_fill_tables(self._h, _np_ptr(ids), len(ids), _np_ptr(tables),
                                         max_blocks_per_seq, pad, _np_ptr(lens)),
               "pa_alloc_fill_tables")
        return tables, lens

    def ref_count(self, block: int) -> int:
        r = ctypes.c_int()
        _check(_lib.pa_alloc_ref_count(self._h, block, ctypes.byref(r)), "pa_alloc_ref_count")
        return r.value

    def stats(self):
        """(free blocks, token slots in use, allocated slots not holding a token)."""
        fb, ut, wt = ctypes.c_int(), ctypes.c_int64(), ctypes.c_int64()
        _check(_lib.pa_alloc_stats(self._h, ctypes.byref(fb), ctypes.byref(ut), ctypes.byref(wt)),
               "pa_alloc_stats")
        return fb.value, ut.value, wt.value

    def num_free(self) -> int:
        return self.stats()[0]
