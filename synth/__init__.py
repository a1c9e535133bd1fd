"""Seeded synthetic inputs for paged decode attention.

This module draws every random input of a decode step and nothing else:
context lengths, the physical block ids that fill each sequence's block
table, the queries, and the *logical* K/V history of every sequence (one
row per token position, in position order). It never maps a position to
a block or a slot, never touches a KV pool and computes no attention: the
CUDA path and the CPU oracle each place the logical rows into their own
pool with their own code.

Values are drawn as float32 N(0, 1) with ``numpy.random.default_rng`` and
rounded to the storage type with round-to-nearest-even, so both sides read
the same 16-bit patterns. Arrays of 16-bit floats are returned as
``uint16`` bit patterns.

Workload shapes follow the pages' examples: Llama-3.1-8B (32 q heads,
8 KV heads, head_dim 128, 16-token blocks; page "08. PagedAttention：把 KV
Cache 分页管理", section "浪费降到了多少") and OPT-13B (40 heads of 128;
page intelliparadigm "PagedAttention 核心思想解析", section 1), block size
16 and a 65,536-block pool (same page, section 6.1 configuration example).
"""
from __future__ import annotations

from dataclasses import dataclass, field
import math

import numpy as np

F16 = "f16"
BF16 = "bf16"

SEED_BASE = 370_000


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def f32_to_f16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to IEEE binary16 (nearest, ties to even); return bits."""
    return np.ascontiguousarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)


def round_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == BF16:
        return f32_to_bf16_bits(x)
    if dtype == F16:
        return f32_to_f16_bits(x)
    raise ValueError(f"unknown dtype {dtype!r}")


def _normal_bits(rng: np.random.Generator, shape, dtype: str) -> np.ndarray:
    """N(0,1) float32 draws rounded to ``dtype``; drawn in slabs to bound memory."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    slab = 1 << 24
    for s in range(0, n, slab):
        e = min(n, s + slab)
        out[s:e] = round_bits(rng.standard_normal(e - s, dtype=np.float32), dtype)
    return out.reshape(shape)


def scale_for(head_dim: int) -> np.float32:
    """The softmax scale 1/sqrt(d) of the attention formula, as float32."""
    return np.float32(1.0 / math.sqrt(head_dim))


@dataclass
class DecodeBatch:
    """One batch of sequences, each with a block table and a logical K/V history.

    ``context_lens[b]`` counts every token of sequence ``b`` including the
    one this step appends (its last position). ``k``/``v`` hold the
    logical rows of all sequences back to back: sequence ``b`` owns rows
    ``seq_start[b] : seq_start[b + 1]`` in position order. Each row of
    ``block_tables`` is filled with distinct physical ids over its whole
    width; a sequence only ever uses a prefix of its row.
    """

    name: str
    dtype: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    max_blocks_per_seq: int
    context_lens: np.ndarray  # int32 [B]
    block_tables: np.ndarray  # int32 [B, max_blocks_per_seq]
    q: np.ndarray             # uint16 [B, Hq, D]
    k: np.ndarray             # uint16 [sum(lens), Hkv, D]
    v: np.ndarray             # uint16 [sum(lens), Hkv, D]
    seq_start: np.ndarray     # int64 [B + 1]
    scale: np.float32
    meta: dict = field(default_factory=dict)

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0

    @property
    def total_tokens(self) -> int:
        return int(self.seq_start[-1])

    def rows(self, b: int) -> slice:
        return slice(int(self.seq_start[b]), int(self.seq_start[b + 1]))

    def new_token_rows(self) -> np.ndarray:
        """Row index of each sequence's last position (the token this step writes)."""
        return self.seq_start[1:] - 1

    def history_rows(self) -> np.ndarray:
        """Row indices of every position except each sequence's last one."""
        keep = np.ones(self.total_tokens, dtype=bool)
        keep[self.new_token_rows()] = False
        return np.nonzero(keep)[0]


def _table_width(max_len: int, block_size: int) -> int:
    # capacity of a table row: enough entries for the longest allowed context
    return max(1, -(-max_len // block_size))


def _assemble(name, rng, dtype, lens, Hq, Hkv, D, bs, nb, table_ids, width, meta=None,
              kv=None, q=None) -> DecodeBatch:
    B = len(lens)
    lens = np.asarray(lens, dtype=np.int32)
    seq_start = np.zeros(B + 1, dtype=np.int64)
    np.cumsum(lens, out=seq_start[1:])
    total = int(seq_start[-1])
    if q is None:
        q = _normal_bits(rng, (B, Hq, D), dtype)
    if kv is None:
        k = _normal_bits(rng, (total, Hkv, D), dtype)
        v = _normal_bits(rng, (total, Hkv, D), dtype)
    else:
        k, v = kv
    tables = np.asarray(table_ids, dtype=np.int32).reshape(B, width)
    return DecodeBatch(name=name, dtype=dtype, num_seqs=B, num_q_heads=Hq,
                       num_kv_heads=Hkv, head_dim=D, block_size=bs, num_blocks=nb,
                       max_blocks_per_seq=width, context_lens=lens, block_tables=tables,
                       q=q, k=k, v=v, seq_start=seq_start, scale=scale_for(D),
                       meta=dict(meta or {}))


def tiny(seed: int = SEED_BASE + 1) -> DecodeBatch:
    """4 sequences, lengths {1, 7, 16, 33}, 16-token blocks in a 16-block pool,
    4 q heads = 4 KV heads, head_dim 64, fp16; block ids are the leading
    entries of a seeded permutation of the pool, handed out in order."""
    rng = np.random.default_rng(seed)
    lens = [1, 7, 16, 33]
    bs, nb = 16, 16
    width = _table_width(max(lens), bs)
    ids = rng.permutation(nb)[: len(lens) * width]
    return _assemble("tiny", rng, F16, lens, 4, 4, 64, bs, nb, ids, width)


def llama8b(seed: int = SEED_BASE + 2, variant: int = 0, num_variants: int = 1,
            num_seqs: int = 64, num_blocks: int = 65536) -> DecodeBatch:
    """Llama-3.1-8B-shaped single-layer decode batch: 64 sequences, 32 q / 8 KV
    heads, head_dim 128, bf16, 16-token blocks, lengths uniform in
    [128, 2048], one 65,536-block pool. ``variant`` selects one of
    ``num_variants`` batches that draw disjoint block ids from the same
    pool (so several batches can live in one pool at once). A smaller
    ``num_blocks`` shrinks the pool (for profiler captures) without changing
    the batch's lengths or values."""
    bs, nb, lo, hi = 16, num_blocks, 128, 2048
    width = _table_width(hi, bs)
    pool_rng = np.random.default_rng(seed)
    perm = pool_rng.permutation(nb)
    need = num_seqs * width
    if need * num_variants > nb:
        raise ValueError("not enough physical blocks for the requested variants")
    ids = perm[variant * need:(variant + 1) * need]
    rng = np.random.default_rng(seed + 7919 * (variant + 1))
    lens = rng.integers(lo, hi + 1, size=num_seqs)
    return _assemble("llama8b", rng, BF16, lens, 32, 8, 128, bs, nb, ids, width,
                     meta={"variant": variant})


def long_skew(seed: int = SEED_BASE + 3, num_seqs: int = 8, lo: int = 8192,
              hi: int = 32768, spikes: int = 4, spike_factor: float = 8.0) -> DecodeBatch:
    """Long-context decode: 8 sequences with lengths uniform in [8192, 32768],
    32 q / 8 KV heads, head_dim 128, bf16, 16-token blocks, 65,536-block
    pool. In every (sequence, KV head) ``spikes`` seeded key rows are
    multiplied by 8 (exact in bf16) to stress the running softmax max."""
    bs, nb = 16, 65536
    width = _table_width(hi, bs)
    rng = np.random.default_rng(seed)
    ids = rng.choice(nb, size=num_seqs * width, replace=False)
    lens = rng.integers(lo, hi + 1, size=num_seqs)
    batch = _assemble("long_skew", rng, BF16, lens, 32, 8, 128, bs, nb, ids, width)
    spike_rows = np.zeros((num_seqs, batch.num_kv_heads, spikes), dtype=np.int64)
    for b in range(num_seqs):
        for g in range(batch.num_kv_heads):
            pos = rng.choice(int(lens[b]), size=spikes, replace=False)
            spike_rows[b, g] = pos
            rows = batch.seq_start[b] + pos
            vals = _bits_to_f32(batch.k[rows, g, :], BF16) * np.float32(spike_factor)
            batch.k[rows, g, :] = f32_to_bf16_bits(vals)
    batch.meta["spike_positions"] = spike_rows
    return batch


def mixed_lengths(seed: int = SEED_BASE + 5, num_seqs: int = 256, lo: int = 16,
                  hi: int = 4096) -> np.ndarray:
    """Log-uniform context lengths floor(exp(U(ln lo, ln hi)))."""
    rng = np.random.default_rng(seed)
    u = rng.uniform(math.log(lo), math.log(hi), size=num_seqs)
    return np.floor(np.exp(u)).astype(np.int32)


def mixed_sweep(block_size: int, seed: int = SEED_BASE + 5, num_seqs: int = 256,
                token_capacity: int = 1 << 20, base: DecodeBatch | None = None) -> DecodeBatch:
    """Mixed serving batch for one block size of the sweep {8,16,32,64,256}:
    256 sequences with log-uniform lengths in [16, 4096], 32 q / 8 KV heads,
    head_dim 128, bf16. The logical K/V and q are drawn once (pass ``base``
    to reuse them) and only the block tables change with the block size;
    the pool holds ``token_capacity / block_size`` blocks."""
    lens = mixed_lengths(seed, num_seqs)
    nb = token_capacity // block_size
    width = _table_width(4096, block_size)
    id_rng = np.random.default_rng(seed * 1000 + block_size)
    ids = id_rng.permutation(nb)[: num_seqs * width]
    if base is None:
        rng = np.random.default_rng(seed)
        rng.uniform(size=num_seqs)  # keep the value stream independent of the lengths draw
        return _assemble(f"mixed_bs{block_size}", rng, BF16, lens, 32, 8, 128, block_size, nb,
                         ids, width, meta={"block_size": block_size})
    return _assemble(f"mixed_bs{block_size}", None, BF16, lens, 32, 8, 128, block_size, nb,
                     ids, width, meta={"block_size": block_size}, kv=(base.k, base.v), q=base.q)


@dataclass
class SharedPromptScript:
    """Inputs of the shared-prompt (parallel sampling / beam) workload.

    For every prompt ``i`` there are four branches, in this order:
    ``P0`` (the parent that holds the prompt), ``P1``/``P2`` (forked from
    ``P0`` right after the prompt), and ``P3`` (forked from ``P1`` after
    ``P1`` generated ``n_before_fork[i]`` tokens, a count that is not a
    multiple of the block size, so ``P1``'s last block is shared while only
    partly filled). ``P0`` and ``P2`` then generate ``n_after[i, 0]`` and
    ``n_after[i, 1]`` tokens. The decode step appends one new token to
    each of the 64 branches in branch order.

    Token rows: ``prompt_k[i]`` [prompt_len, H, D]; ``gen_k[i][j]`` rows of
    branch-local history (j = 0: P0's, 1: P1's before the fork, 2: P2's);
    ``new_k`` [64, H, D] the step's token per branch. Same for v.
    """

    dtype: str
    num_prompts: int
    prompt_len: int
    num_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    n_before_fork: np.ndarray   # int32 [P]
    n_after: np.ndarray         # int32 [P, 2]  (P0, P2)
    prompt_k: np.ndarray
    prompt_v: np.ndarray
    gen_k: list
    gen_v: list
    new_k: np.ndarray
    new_v: np.ndarray
    q: np.ndarray               # uint16 [64, H, D]
    scale: np.float32


def shared_prompt(seed: int = SEED_BASE + 4, num_prompts: int = 16, prompt_len: int = 512,
                  num_heads: int = 40, head_dim: int = 128, block_size: int = 16,
                  num_blocks: int = 4096, max_private: int = 200) -> SharedPromptScript:
    """OPT-13B-shaped shared-prompt decode: 16 prompts of 512 tokens, 40 q heads
    = 40 KV heads, head_dim 128, fp16, 16-token blocks, a 4,096-block pool;
    four branches per prompt with up to 200 private tokens each."""
    rng = np.random.default_rng(seed)
    n_before = np.empty(num_prompts, dtype=np.int32)
    for i in range(num_prompts):
        while True:
            n = int(rng.integers(1, max_private))
            if n % block_size:
                break
        n_before[i] = n
    n_after = rng.integers(0, max_private, size=(num_prompts, 2)).astype(np.int32)
    H, D = num_heads, head_dim
    pk = _normal_bits(rng, (num_prompts, prompt_len, H, D), F16)
    pv = _normal_bits(rng, (num_prompts, prompt_len, H, D), F16)
    gen_k, gen_v = [], []
    for i in range(num_prompts):
        counts = (int(n_after[i, 0]), int(n_before[i]), int(n_after[i, 1]))
        gen_k.append([_normal_bits(rng, (c, H, D), F16) for c in counts])
        gen_v.append([_normal_bits(rng, (c, H, D), F16) for c in counts])
    nseq = 4 * num_prompts
    new_k = _normal_bits(rng, (nseq, H, D), F16)
    new_v = _normal_bits(rng, (nseq, H, D), F16)
    q = _normal_bits(rng, (nseq, H, D), F16)
    return SharedPromptScript(dtype=F16, num_prompts=num_prompts, prompt_len=prompt_len,
                              num_heads=H, head_dim=D, block_size=block_size,
                              num_blocks=num_blocks, n_before_fork=n_before, n_after=n_after,
                              prompt_k=pk, prompt_v=pv, gen_k=gen_k, gen_v=gen_v,
                              new_k=new_k, new_v=new_v, q=q, scale=scale_for(D))


def _bits_to_f32(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Widen 16-bit patterns to float32 (exact) -- used only to apply the
    exact x8 spike to bf16 keys before re-rounding."""
    if dtype == BF16:
        return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return bits.view(np.float16).astype(np.float32)


def small_random(seed: int, num_seqs: int, lens, num_q_heads: int, num_kv_heads: int,
                 head_dim: int, block_size: int, num_blocks: int, dtype: str,
                 width: int | None = None) -> DecodeBatch:
    """A generic small batch for tests: given lengths, a pool of ``num_blocks``
    and a table width, block ids are a seeded permutation of the pool."""
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, dtype=np.int32)
    if width is None:
        width = _table_width(int(lens.max()) if len(lens) else 1, block_size)
    if num_seqs * width > num_blocks:
        raise ValueError("pool too small for full-width tables")
    ids = rng.permutation(num_blocks)[: num_seqs * width]
    return _assemble("small", rng, dtype, lens, num_q_heads, num_kv_heads, head_dim, block_size,
                     num_blocks, ids, width)


# ------------------------------------------------------------------------------------ prefill
def prefill_random(seed: int, lens, q_lens, num_q_heads: int, num_kv_heads: int, head_dim: int,
                   block_size: int, num_blocks: int, dtype: str, width: int | None = None,
                   name: str = "prefill") -> DecodeBatch:
    """A prefill (or chunked-prefill) batch: sequence b holds lens[b] positions of
    which the last q_lens[b] are this step's query tokens. ``q`` is [T, Hq, D]
    with T = sum(q_lens), rows in sequence order; ``meta['q_start']`` (int32
    [B + 1]) delimits each sequence's rows. K/V rows cover every position (the
    new tokens' included: they are written to the pool before attending)."""
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, dtype=np.int32)
    q_lens = np.asarray(q_lens, dtype=np.int32)
    assert len(lens) == len(q_lens) and np.all(q_lens <= lens) and np.all(q_lens >= 0)
    if width is None:
        width = _table_width(int(lens.max()) if len(lens) else 1, block_size)
    if len(lens) * width > num_blocks:
        raise ValueError("pool too small for full-width tables")
    ids = rng.permutation(num_blocks)[: len(lens) * width]
    q_start = np.zeros(len(lens) + 1, dtype=np.int32)
    np.cumsum(q_lens, out=q_start[1:])
    q = _normal_bits(rng, (int(q_start[-1]), num_q_heads, head_dim), dtype)
    return _assemble(name, rng, dtype, lens, num_q_heads, num_kv_heads, head_dim, block_size,
                     num_blocks, ids, width, meta={"q_start": q_start, "q_lens": q_lens}, q=q)


def llama8b_prefill(seed: int = SEED_BASE + 7, num_blocks: int = 65536) -> DecodeBatch:
    """Chunked prefill on the Llama-3.1-8B shapes (32 q / 8 KV heads, head_dim
    128, bf16, 16-token blocks): 16 sequences, each with a history uniform in
    [0, 1536] positions and a chunk of 512 new query tokens."""
    rng = np.random.default_rng(seed)
    hist = rng.integers(0, 1537, size=16)
    q_lens = np.full(16, 512, dtype=np.int32)
    lens = (hist + q_lens).astype(np.int32)
    return prefill_random(seed + 1, lens, q_lens, 32, 8, 128, 16, num_blocks, BF16,
                          width=_table_width(2048, 16), name="llama8b_prefill")
