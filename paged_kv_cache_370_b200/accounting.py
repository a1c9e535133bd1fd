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
