"""Byte accounting of paged decode attention (the roofline numerators).

``kv_bytes_per_token`` is the K+V footprint of one token over a model's
layers: 2 (K and V) x layers x kv_heads x head_dim x element bytes. The pages
give two instances: 128 KiB per token for Llama-3.1-8B and 2 MiB per 16-token
block of 32 layers (page "08. PagedAttention：把 KV Cache 分页管理", section
"浪费降到了多少"), and about 800 KB per token for OPT-13B (page
"PagedAttention 核心思想解析", section 1).

``decode_step_bytes`` counts the algorithmic bytes one decode step must move:
the K and V rows of exactly context_len tokens per (sequence, kv head) --
every step reads the whole history (third page, section "它没有解决什么") --
plus the queries, the outputs, the block-table entries actually used and the
context lengths. Bytes the kernels move beyond that (the split-context
scratch, the new tokens' write) are reported separately.
"""
from __future__ import annotations

import numpy as np


def kv_bytes_per_token(num_layers: int, num_kv_heads: int, head_dim: int, elem_bytes: int) -> int:
    return 2 * num_layers * num_kv_heads * head_dim * elem_bytes


def blocks_needed(context_lens, block_size: int) -> np.ndarray:
    lens = np.asarray(context_lens, dtype=np.int64)
    return (lens + block_size - 1) // block_size


def decode_step_bytes(context_lens, num_q_heads: int, num_kv_heads: int, head_dim: int,
                      block_size: int, elem_bytes: int = 2) -> dict:
    lens = np.asarray(context_lens, dtype=np.int64)
    B = len(lens)
    kv = 2 * int(lens.sum()) * num_kv_heads * head_dim * elem_bytes
    q = B * num_q_heads * head_dim * elem_bytes
    out = q
    tables = int(blocks_needed(lens, block_size).sum()) * 4
    ctx = B * 4
    return {"kv": kv, "q": q, "out": out, "block_tables": tables, "context_lens": ctx,
            "total": kv + q + out + tables + ctx}


def tail_overread_bytes(context_lens, num_kv_heads: int, head_dim: int, block_size: int,
                        elem_bytes: int = 2) -> int:
    """K and V bytes of the unfilled tail rows of each sequence's last block, which a
    kernel that copies whole blocks reads beyond the algorithmic bytes."""
    lens = np.asarray(context_lens, dtype=np.int64)
    tail = blocks_needed(lens, block_size) * block_size - lens
    return int(2 * tail.sum() * num_kv_heads * head_dim * elem_bytes)


def split_scratch_bytes(context_lens, num_q_heads: int, head_dim: int, partition_tokens: int) -> int:
    """Workspace bytes written and read back for sequences split into more than
    one partition: (head_dim + 2) fp32 per (sequence, q head, partition), twice."""
    lens = np.asarray(context_lens, dtype=np.int64)
    parts = (lens + partition_tokens - 1) // partition_tokens
    parts = np.where(parts > 1, parts, 0)
    return int(2 * parts.sum() * num_q_heads * (head_dim + 2) * 4)


def new_token_bytes(num_tokens: int, num_kv_heads: int, head_dim: int, elem_bytes: int = 2) -> int:
    """The KV write of a step: each new token's K and V rows read once and written once."""
    return 2 * 2 * num_tokens * num_kv_heads * head_dim * elem_bytes


def stream_split_scratch_bytes(context_lens, num_kv_heads: int, group: int, head_dim: int,
                               num_ctas: int, tile: int = 64) -> int:
    """Workspace bytes the even-split kernel moves for one call: the work is the
    list of (sequence, kv head) segments in order, each cut into tiles of ``tile``
    tokens (an empty sequence still has one tile), and CTA c takes tiles
    [c*W/n, (c+1)*W/n). A segment whose tiles belong to more than one CTA leaves
    one piece per such CTA -- (head_dim + 2) fp32 for each of its ``group`` q
    heads -- written once and read back once by the merge, plus a 4-byte counter
    read and written per piece."""
    lens = np.asarray(context_lens, dtype=np.int64)
    n = int(num_ctas)
    if n <= 0 or lens.size == 0:
        return 0
    per_seg = np.maximum(1, (lens + tile - 1) // tile)
    seg = np.repeat(per_seg, num_kv_heads)           # sequences in order, kv heads inner
    first = np.concatenate([[0], np.cumsum(seg)[:-1]])
    W = int(seg.sum())
    owner = lambda x: ((x + 1) * n - 1) // W           # noqa: E731 -- CTA holding tile x
    ca, cb = owner(first), owner(first + seg - 1)
    starts = (np.arange(n + 1, dtype=np.int64) * W) // n
    has = (starts[1:] > starts[:-1]).astype(np.int64)  # CTAs that own any tile
    cum = np.concatenate([[0], np.cumsum(has)])
    pieces = cum[cb + 1] - cum[ca]
    pieces = np.where(pieces > 1, pieces, 0)
    return int(pieces.sum() * (2 * group * (head_dim + 2) * 4 + 8))


def unique_kv_bytes(block_tables, context_lens, block_size: int, num_kv_heads: int,
                    head_dim: int, elem_bytes: int = 2) -> int:
    """K and V bytes of every physical block a batch reads, each block counted once:
    rows [0, r) of a block, r the most any sequence reads from it (blocks shared
    by several sequences -- a forked prompt -- are counted once, not per reader)."""
    lens = np.asarray(context_lens, dtype=np.int64)
    rows = {}
    for b, n in enumerate(lens):
        nblk = int(-(-int(n) // block_size))
        for i in range(nblk):
            blk = int(block_tables[b][i])
            r = min(block_size, int(n) - i * block_size)
            rows[blk] = max(rows.get(blk, 0), r)
    return int(2 * sum(rows.values()) * num_kv_heads * head_dim * elem_bytes)
