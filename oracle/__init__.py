"""The CPU oracle for paged decode attention -- TEST INFRASTRUCTURE ONLY.

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
may import this package. The product library never does: it shares no code
with the oracle, and the product path fails loudly when its CUDA library is
missing instead of falling back here.

``oracle.c`` holds the fp64 arithmetic (plain loops, no blocking or fusion);
this module compiles it with gcc into ``liboracle.so`` beside the source and
wraps its entry points for NumPy arrays. ``allocator_model`` is a plain
Python model of the block manager (free list, reference counts,
copy-on-write).

Every function here is pinned by ``tests/test_oracle_pins.py`` to facts
that do not come from the oracle itself (the pages' worked example, closed
forms, library routines, brute force).
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

DTYPE_CODE = {"f16": 0, "bf16": 1}

_lib = None


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` (gcc, OpenMP, strict fp)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
               "-shared", "-std=c11", "-Wall", "-o", tmp, SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


def _load(path: str):
    """Load a compiled oracle library and declare its C signatures."""
    L = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i, f, i64 = ctypes.c_int, ctypes.c_float, ctypes.c_int64
    L.oracle_f16_to_double.restype = ctypes.c_double
    L.oracle_f16_to_double.argtypes = [ctypes.c_uint16]
    L.oracle_bf16_to_double.restype = ctypes.c_double
    L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
    L.oracle_slot.restype = i64
    L.oracle_slot.argtypes = [P, i64, i]
    L.oracle_reshape_and_cache.restype = i
    L.oracle_reshape_and_cache.argtypes = [P, P, P, i, P, P, i, i, i, i]
    L.oracle_copy_blocks.restype = i
    L.oracle_copy_blocks.argtypes = [P, P, P, i, i, i, i, i]
    L.oracle_decode.restype = i
    L.oracle_decode.argtypes = [P, P, P, P, P, i, P, i, i, i, i, i, i, f, i, i]
    L.oracle_decode_one.restype = i
    L.oracle_decode_one.argtypes = [P, P, P, P, P, i, i, i, i, i, i, f, i]
    L.oracle_decode_partitioned.restype = i
    L.oracle_decode_partitioned.argtypes = [P, P, P, P, P, i, P, i, i, i, i, i, i, f, i,
                                            i, i, P, P, P, i]
    L.oracle_max_threads.restype = i
    L.oracle_decode_window.restype = i
    L.oracle_decode_window.argtypes = [P, P, P, P, P, i, P, i, i, i, i, i, i, f, i, i, i]
    L.oracle_swap_blocks.restype = i
    L.oracle_swap_blocks.argtypes = [P, P, i, P, P, i, P, i, i, i, i]
    L.oracle_prefill.restype = i
    L.oracle_prefill.argtypes = [P, P, P, P, P, i, P, P, i, i, i, i, i, i, f, i, i, i]
    L.oracle_max_threads.argtypes = []
    return L


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = _load(LIB)
    return _lib


@contextlib.contextmanager
def using(path: str):
    """Route every wrapper of this module through another build of the oracle
    (the mutation tests compile deliberately broken copies of oracle.c)."""
    global _lib
    saved = _lib
    _lib = _load(path)
    _widen_tables.clear()
    try:
        yield _lib
    finally:
        _lib = saved
        _widen_tables.clear()


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _need(a: np.ndarray, dtype) -> np.ndarray:
    if a.dtype != dtype or not a.flags.c_contiguous:
        raise TypeError(f"expected C-contiguous {np.dtype(dtype)} array, got {a.dtype}")
    return a


class OracleError(RuntimeError):
    pass


def _check(rc: int, what: str):
    if rc != 0:
        raise OracleError(f"{what} failed with status {rc}")


def f16_to_double(bits: int) -> float:
    return lib().oracle_f16_to_double(bits)


def bf16_to_double(bits: int) -> float:
    return lib().oracle_bf16_to_double(bits)


_widen_tables: dict = {}


def widen(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Exact fp64 values of 16-bit patterns, via the oracle's own decoders."""
    if dtype not in _widen_tables:
        fn = lib().oracle_bf16_to_double if dtype == "bf16" else lib().oracle_f16_to_double
        _widen_tables[dtype] = np.array([fn(i) for i in range(1 << 16)], dtype=np.float64)
    flat = np.asarray(bits, dtype=np.uint16).ravel()
    return _widen_tables[dtype][flat].reshape(np.shape(bits))


def slot(table_row: np.ndarray, pos: int, block_size: int) -> int:
    row = _need(np.asarray(table_row, dtype=np.int32), np.int32)
    return int(lib().oracle_slot(_ptr(row), pos, block_size))


def slots_for(table_row: np.ndarray, positions, block_size: int) -> np.ndarray:
    row = _need(np.ascontiguousarray(table_row, dtype=np.int32), np.int32)
    return np.array([lib().oracle_slot(_ptr(row), int(p), block_size) for p in positions],
                    dtype=np.int64)


def empty_pool(num_blocks: int, num_kv_heads: int, block_size: int, head_dim: int) -> np.ndarray:
    """A zeroed K or V pool [num_blocks, num_kv_heads, block_size, head_dim] of 16-bit patterns."""
    return np.zeros((num_blocks, num_kv_heads, block_size, head_dim), dtype=np.uint16)


def reshape_and_cache(k_new, v_new, slot_mapping, k_cache, v_cache):
    nb, hkv, bs, d = k_cache.shape
    k_new = _need(k_new, np.uint16)
    v_new = _need(v_new, np.uint16)
    slot_mapping = _need(slot_mapping, np.int64)
    _need(k_cache, np.uint16)
    _need(v_cache, np.uint16)
    rc = lib().oracle_reshape_and_cache(_ptr(k_new), _ptr(v_new), _ptr(slot_mapping),
                                        len(slot_mapping), _ptr(k_cache), _ptr(v_cache), nb, hkv,
                                        bs, d)
    _check(rc, "oracle_reshape_and_cache")


def copy_blocks(k_cache, v_cache, block_pairs):
    nb, hkv, bs, d = k_cache.shape
    pairs = _need(np.ascontiguousarray(block_pairs, dtype=np.int64).reshape(-1, 2), np.int64)
    rc = lib().oracle_copy_blocks(_ptr(_need(k_cache, np.uint16)), _ptr(_need(v_cache, np.uint16)),
                                  _ptr(pairs), len(pairs), nb, hkv, bs, d)
    _check(rc, "oracle_copy_blocks")


def swap_blocks(dst_k, dst_v, src_k, src_v, block_pairs):
    """dst pools [block] = src pools [block] for each (src, dst) pair (K and V)."""
    nd, hkv, bs, d = dst_k.shape
    ns = src_k.shape[0]
    assert src_k.shape[1:] == dst_k.shape[1:]
    pairs = _need(np.ascontiguousarray(block_pairs, dtype=np.int64).reshape(-1, 2), np.int64)
    rc = lib().oracle_swap_blocks(_ptr(_need(dst_k, np.uint16)), _ptr(_need(dst_v, np.uint16)), nd,
                                  _ptr(_need(src_k, np.uint16)), _ptr(_need(src_v, np.uint16)), ns,
                                  _ptr(pairs), len(pairs), hkv, bs, d)
    _check(rc, "oracle_swap_blocks")


def decode(q, k_cache, v_cache, block_tables, context_lens, scale, dtype, num_threads=0):
    """fp64 outputs [B, Hq, D] of paged decode attention (unrounded)."""
    B, hq, d = q.shape
    nb, hkv, bs, d2 = k_cache.shape
    assert d == d2
    out = np.zeros((B, hq, d), dtype=np.float64)
    bt = _need(np.ascontiguousarray(block_tables, dtype=np.int32), np.int32)
    cl = _need(np.ascontiguousarray(context_lens, dtype=np.int32), np.int32)
    rc = lib().oracle_decode(_ptr(out), _ptr(_need(q, np.uint16)), _ptr(_need(k_cache, np.uint16)),
                             _ptr(_need(v_cache, np.uint16)), _ptr(bt), bt.shape[1], _ptr(cl), B,
                             hq, hkv, d, bs, nb, float(scale), DTYPE_CODE[dtype], num_threads)
    _check(rc, "oracle_decode")
    return out


def decode_window(q, k_cache, v_cache, block_tables, context_lens, scale, dtype, window,
                  num_threads=0):
    """fp64 outputs [B, Hq, D] of sliding-window decode: each sequence attends to
    its last ``window`` positions (``window`` <= 0: all of them)."""
    B, hq, d = q.shape
    nb, hkv, bs, d2 = k_cache.shape
    assert d == d2
    out = np.zeros((B, hq, d), dtype=np.float64)
    bt = _need(np.ascontiguousarray(block_tables, dtype=np.int32), np.int32)
    cl = _need(np.ascontiguousarray(context_lens, dtype=np.int32), np.int32)
    rc = lib().oracle_decode_window(_ptr(out), _ptr(_need(q, np.uint16)),
                                    _ptr(_need(k_cache, np.uint16)),
                                    _ptr(_need(v_cache, np.uint16)), _ptr(bt), bt.shape[1],
                                    _ptr(cl), B, hq, hkv, d, bs, nb, float(scale),
                                    DTYPE_CODE[dtype], int(window), num_threads)
    _check(rc, "oracle_decode_window")
    return out


def prefill(q, k_cache, v_cache, block_tables, context_lens, q_start, scale, dtype, window=0,
            num_threads=0):
    """fp64 outputs [T, Hq, D] of paged prefill attention: the query rows of
    sequence b are q[q_start[b]:q_start[b+1]], its last positions; each attends
    causally (and within ``window`` if > 0)."""
    T, hq, d = q.shape
    nb, hkv, bs, d2 = k_cache.shape
    assert d == d2
    out = np.zeros((T, hq, d), dtype=np.float64)
    bt = _need(np.ascontiguousarray(block_tables, dtype=np.int32), np.int32)
    cl = _need(np.ascontiguousarray(context_lens, dtype=np.int32), np.int32)
    qs = _need(np.ascontiguousarray(q_start, dtype=np.int32), np.int32)
    assert len(qs) == len(cl) + 1 and qs[-1] == T
    rc = lib().oracle_prefill(_ptr(out), _ptr(_need(q, np.uint16)), _ptr(_need(k_cache, np.uint16)),
                              _ptr(_need(v_cache, np.uint16)), _ptr(bt), bt.shape[1], _ptr(cl),
                              _ptr(qs), len(cl), hq, hkv, d, bs, nb, float(scale),
                              DTYPE_CODE[dtype], int(window), num_threads)
    _check(rc, "oracle_prefill")
    return out


def decode_one(q_row, k_cache, v_cache, table_row, context_len, kv_head, scale, dtype):
    nb, hkv, bs, d = k_cache.shape
    out = np.zeros(d, dtype=np.float64)
    row = _need(np.ascontiguousarray(table_row, dtype=np.int32), np.int32)
    qr = _need(np.ascontiguousarray(q_row, dtype=np.uint16), np.uint16)
    rc = lib().oracle_decode_one(_ptr(out), _ptr(qr), _ptr(_need(k_cache, np.uint16)),
                                 _ptr(_need(v_cache, np.uint16)), _ptr(row), int(context_len),
                                 int(kv_head), hkv, d, bs, nb, float(scale), DTYPE_CODE[dtype])
    _check(rc, "oracle_decode_one")
    return out


def decode_partitioned(q, k_cache, v_cache, block_tables, context_lens, scale, dtype,
                       partition_tokens, return_partials=False, num_threads=0):
    B, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    cl = _need(np.ascontiguousarray(context_lens, dtype=np.int32), np.int32)
    bt = _need(np.ascontiguousarray(block_tables, dtype=np.int32), np.int32)
    max_parts = max(1, -(-int(cl.max()) // partition_tokens)) if B else 1
    out = np.zeros((B, hq, d), dtype=np.float64)
    pm = np.zeros((B, hq, max_parts)) if return_partials else None
    pl = np.zeros((B, hq, max_parts)) if return_partials else None
    pa = np.zeros((B, hq, max_parts, d)) if return_partials else None
    rc = lib().oracle_decode_partitioned(_ptr(out), _ptr(_need(q, np.uint16)),
                                         _ptr(_need(k_cache, np.uint16)),
                                         _ptr(_need(v_cache, np.uint16)), _ptr(bt), bt.shape[1],
                                         _ptr(cl), B, hq, hkv, d, bs, nb, float(scale),
                                         DTYPE_CODE[dtype], partition_tokens, max_parts, _ptr(pm),
                                         _ptr(pl), _ptr(pa), num_threads)
    _check(rc, "oracle_decode_partitioned")
    if return_partials:
        return out, pm, pl, pa
    return out


def max_threads() -> int:
    return int(lib().oracle_max_threads())


# ----------------------------------------------------------------------------------------------
# Placement helpers: put a synth.DecodeBatch's logical rows into an oracle-side pool.


def place_history(batch, k_cache, v_cache, include_new: bool = True):
    """Write the logical K/V rows of every sequence of ``batch`` into the pools
    at the slots the oracle computes from the block tables. With
    ``include_new`` False the last position of each sequence is left out
    (it is the token the decode step itself writes)."""
    for b in range(batch.num_seqs):
        n = int(batch.context_lens[b]) - (0 if include_new else 1)
        if n <= 0:
            continue
        rows = np.arange(int(batch.seq_start[b]), int(batch.seq_start[b]) + n)
        slots = slots_for(batch.block_tables[b], range(n), batch.block_size)
        reshape_and_cache(np.ascontiguousarray(batch.k[rows]), np.ascontiguousarray(batch.v[rows]),
                          slots, k_cache, v_cache)


def new_token_slots(batch) -> np.ndarray:
    """Slot of each sequence's last position (where the step's token goes)."""
    return np.array([slot(batch.block_tables[b], int(batch.context_lens[b]) - 1, batch.block_size)
                     if batch.context_lens[b] > 0 else -1 for b in range(batch.num_seqs)],
                    dtype=np.int64)
