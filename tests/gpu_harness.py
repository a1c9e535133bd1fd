"""Run a synthetic decode workload through the CUDA path (via the C ABI) and
through the oracle, on the same seeded inputs. Test-only plumbing: the CUDA
side uses only the library (pa_slot_mapping, BlockManager, the kernels); the
oracle side uses only ``oracle``."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from oracle.allocator_model import BlockManagerModel
from paged_kv_cache_370_b200 import abi
from paged_kv_cache_370_b200.step import DecodeStep

TORCH_DT = {"f16": torch.float16, "bf16": torch.bfloat16}
NAN_BITS = {"f16": 0x7E00, "bf16": 0x7FC0}


def to_dev(bits: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device).view(TORCH_DT[dtype])


def to_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def poisoned_pool(shape, dtype, device="cuda") -> torch.Tensor:
    bits = NAN_BITS[dtype] - (1 << 16) if NAN_BITS[dtype] >= 1 << 15 else NAN_BITS[dtype]
    return torch.full(shape, bits, dtype=torch.int16, device=device).view(TORCH_DT[dtype])


def widen_out(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).cpu().numpy()


# ------------------------------------------------------------------------- random-table batches
class GpuBatch:
    """A synth.DecodeBatch on the device: history written with pa_reshape_and_cache
    at slots from pa_slot_mapping, and a DecodeStep that writes each sequence's
    last token and decodes."""

    def __init__(self, batch, partition_tokens: int = 0, device="cuda", tables=None,
                 fused: bool = False, window: int = 0, step_tables=None):
        self.batch = batch
        bs, dt = batch.block_size, batch.dtype
        shape = (batch.num_blocks, batch.num_kv_heads, bs, batch.head_dim)
        self.k_cache = poisoned_pool(shape, dt, device)
        self.v_cache = poisoned_pool(shape, dt, device)
        self.tables_np = batch.block_tables if tables is None else tables
        slots = abi.pa_slot_mapping(self.tables_np, batch.context_lens, bs)
        hist = batch.history_rows()
        k_all = to_dev(batch.k, dt, device)
        v_all = to_dev(batch.v, dt, device)
        if len(hist):
            hidx = torch.from_numpy(hist).to(device)
            abi.pa_reshape_and_cache(k_all[hidx].contiguous(), v_all[hidx].contiguous(),
                                     torch.from_numpy(slots[hist]).to(device), self.k_cache,
                                     self.v_cache)
        # the step's new token: one per sequence; empty sequences get a padding slot
        B = batch.num_seqs
        new_k = torch.zeros((B, batch.num_kv_heads, batch.head_dim), dtype=TORCH_DT[dt],
                            device=device)
        new_v = torch.zeros_like(new_k)
        new_slots = np.full(B, -1, dtype=np.int64)
        has = batch.context_lens > 0
        rows = batch.new_token_rows()[has]
        if len(rows):
            ridx = torch.from_numpy(rows).to(device)
            sel = torch.from_numpy(np.nonzero(has)[0]).to(device)
            new_k[sel] = k_all[ridx]
            new_v[sel] = v_all[ridx]
            new_slots[has] = slots[rows]
        del k_all, v_all
        self.step = DecodeStep(
            k_cache=self.k_cache, v_cache=self.v_cache, q=to_dev(batch.q, dt, device),
            k_new=new_k, v_new=new_v, slot_mapping=torch.from_numpy(new_slots).to(device),
            block_tables=torch.from_numpy(np.ascontiguousarray(
                self.tables_np if step_tables is None else step_tables)).to(device),
            context_lens=torch.from_numpy(batch.context_lens).to(device),
            max_context_len=max(batch.max_context_len, 1), scale=float(batch.scale),
            partition_tokens=partition_tokens, fused=fused, window=window)

    def run(self):
        out = self.step.run()
        torch.cuda.synchronize()
        return out

    def slot_rows(self, slots: np.ndarray):
        """Pool rows at the given slots, [n, Hkv, D] bits (K, V)."""
        bs = self.batch.block_size
        s = torch.from_numpy(slots).to(self.k_cache.device)
        blk, off = s // bs, s % bs
        return to_bits(self.k_cache[blk, :, off, :]), to_bits(self.v_cache[blk, :, off, :])


def oracle_pools(batch, tables=None, full=True):
    """Oracle-side pools for ``batch``: history placed with the oracle's slots,
    then the step's new tokens written by oracle.reshape_and_cache. With
    ``full`` the pools start from the same poison pattern as the device pools
    (for whole-pool comparison); otherwise from lazily allocated zeros."""
    shape = (batch.num_blocks, batch.num_kv_heads, batch.block_size, batch.head_dim)
    if full:
        kp = np.full(shape, NAN_BITS[batch.dtype], dtype=np.uint16)
        vp = np.full(shape, NAN_BITS[batch.dtype], dtype=np.uint16)
    else:
        kp = np.zeros(shape, dtype=np.uint16)
        vp = np.zeros(shape, dtype=np.uint16)
    b2 = batch if tables is None else _with_tables(batch, tables)
    oracle.place_history(b2, kp, vp, include_new=False)
    has = batch.context_lens > 0
    if has.any():
        rows = batch.new_token_rows()[has]
        slots = oracle.new_token_slots(b2)[has]
        oracle.reshape_and_cache(np.ascontiguousarray(batch.k[rows]),
                                 np.ascontiguousarray(batch.v[rows]), slots, kp, vp)
    return kp, vp


def _with_tables(batch, tables):
    import copy
    b2 = copy.copy(batch)
    b2.block_tables = tables
    return b2


def oracle_decode(batch, kp, vp, tables=None):
    t = batch.block_tables if tables is None else tables
    return oracle.decode(batch.q, kp, vp, t, batch.context_lens, batch.scale, batch.dtype)


# --------------------------------------------------------------------- shared-prompt workload
def _seq_id(i, j):
    return 4 * i + j


def _shared_prompt_ops(script, mgr, append):
    """Drive a block manager (product or model) through the workload's history.
    Returns the history rows [(slot, k_row, v_row)] in write order."""
    rows_k, rows_v, slots = [], [], []
    P, L = script.num_prompts, script.prompt_len
    for i in range(P):
        p0, p1, p2, p3 = (_seq_id(i, j) for j in range(4))
        mgr.add_seq(p0, L)
        slots.extend(mgr.seq_slots(p0, 0, L))
        rows_k.append(script.prompt_k[i])
        rows_v.append(script.prompt_v[i])
        mgr.fork(p0, p1)
        mgr.fork(p0, p2)
        for seq, j in ((p1, 1),):
            for t in range(int(script.n_before_fork[i])):
                s, src, _ = append(seq)
                assert src == -1
                slots.append(s)
            rows_k.append(script.gen_k[i][j])
            rows_v.append(script.gen_v[i][j])
        mgr.fork(p1, p3)
        for seq, j, n in ((p0, 0, script.n_after[i, 0]), (p2, 2, script.n_after[i, 1])):
            for t in range(int(n)):
                s, src, _ = append(seq)
                assert src == -1
                slots.append(s)
            rows_k.append(script.gen_k[i][j])
            rows_v.append(script.gen_v[i][j])
    return (np.asarray(slots, dtype=np.int64), np.concatenate(rows_k), np.concatenate(rows_v))


def _step_appends(script, append):
    pairs, slots = [], []
    for i in range(script.num_prompts):
        for j in range(4):
            s, src, dst = append(_seq_id(i, j))
            slots.append(s)
            if src >= 0:
                pairs.append((src, dst))
    return np.asarray(slots, dtype=np.int64), np.asarray(pairs, dtype=np.int64).reshape(-1, 2)


SHARED_TABLE_WIDTH = 48


def shared_prompt_gpu(script, device="cuda", fused=False):
    bs, H, D = script.block_size, script.num_heads, script.head_dim
    mgr = abi.BlockManager(script.num_blocks, bs)
    shape = (script.num_blocks, H, bs, D)
    kc, vc = poisoned_pool(shape, script.dtype, device), poisoned_pool(shape, script.dtype, device)
    hslots, hk, hv = _shared_prompt_ops(script, mgr, mgr.append_slot)
    abi.pa_reshape_and_cache(to_dev(hk, script.dtype, device), to_dev(hv, script.dtype, device),
                             torch.from_numpy(hslots).to(device), kc, vc)
    nslots, pairs = _step_appends(script, mgr.append_slot)
    ids = [_seq_id(i, j) for i in range(script.num_prompts) for j in range(4)]
    tables, lens = mgr.fill_tables(ids, SHARED_TABLE_WIDTH, pad=0)
    step = DecodeStep(k_cache=kc, v_cache=vc, q=to_dev(script.q, script.dtype, device),
                      k_new=to_dev(script.new_k, script.dtype, device),
                      v_new=to_dev(script.new_v, script.dtype, device),
                      slot_mapping=torch.from_numpy(nslots).to(device),
                      block_tables=torch.from_numpy(tables).to(device),
                      context_lens=torch.from_numpy(lens).to(device),
                      max_context_len=int(lens.max()), scale=float(script.scale),
                      copy_pairs=torch.from_numpy(pairs).to(device), fused=fused)
    return mgr, step, tables, lens, pairs


class _ModelAdapter:
    def __init__(self, model):
        self.m = model

    def __getattr__(self, k):
        return getattr(self.m, k)


def shared_prompt_oracle(script):
    bs, H, D = script.block_size, script.num_heads, script.head_dim
    model = BlockManagerModel(script.num_blocks, bs)
    shape = (script.num_blocks, H, bs, D)
    kp = np.full(shape, NAN_BITS[script.dtype], dtype=np.uint16)
    vp = np.full(shape, NAN_BITS[script.dtype], dtype=np.uint16)
    hslots, hk, hv = _shared_prompt_ops(script, model, model.append_slot)
    oracle.reshape_and_cache(hk, hv, hslots, kp, vp)
    nslots, pairs = _step_appends(script, model.append_slot)
    oracle.copy_blocks(kp, vp, pairs)
    oracle.reshape_and_cache(np.ascontiguousarray(script.new_k), np.ascontiguousarray(script.new_v),
                             nslots, kp, vp)
    ids = [_seq_id(i, j) for i in range(script.num_prompts) for j in range(4)]
    tables = np.zeros((len(ids), SHARED_TABLE_WIDTH), dtype=np.int32)
    lens = np.zeros(len(ids), dtype=np.int32)
    for r, s in enumerate(ids):
        t = model.block_table(s)
        tables[r, :len(t)] = t
        lens[r] = model.lens[s]
    out = oracle.decode(script.q, kp, vp, tables, lens, script.scale, script.dtype)
    return model, kp, vp, tables, lens, pairs, out
