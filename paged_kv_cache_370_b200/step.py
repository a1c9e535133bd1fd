"""One decode step of a batch through the C ABI.

A decode step, in the order the pages give it: copy-on-write block copies for
sequences about to write into a shared block ("PagedAttention 核心思想解析",
section 2.3), the slot-indexed write of each sequence's new K/V ("08.
PagedAttention：把 KV Cache 分页管理", section "为什么叫 PagedAttention"), and
paged attention of each sequence's query over its whole history ("大语言模型
推理内存管理算法 paged attention", section 5).

``DecodeStep`` holds device tensors (PyTorch provides the memory) and launches
the library's kernels on the current stream. ``HostDecodeStep`` is the same
step fed from pinned host buffers: it copies the step's inputs to the device,
runs the step and copies the output back, all stream-ordered.
"""
from __future__ import annotations

import torch

from . import abi


class DecodeStep:
    def __init__(self, *, k_cache, v_cache, q, k_new, v_new, slot_mapping, block_tables,
                 context_lens, max_context_len: int, scale: float, partition_tokens: int = 0,
                 copy_pairs=None, out=None):
        self.k_cache, self.v_cache = k_cache, v_cache
        self.q, self.k_new, self.v_new = q, k_new, v_new
        self.slot_mapping = slot_mapping
        self.block_tables, self.context_lens = block_tables, context_lens
        self.max_context_len = int(max_context_len)
        self.scale = float(scale)
        self.partition_tokens = int(partition_tokens)
        self.copy_pairs = copy_pairs
        self.out = torch.empty_like(q) if out is None else out
        B, hq, d = q.shape
        hkv = k_cache.shape[1]
        nbytes = abi.pa_decode_workspace_size(B, hq, hkv, d, self.max_context_len,
                                              self.partition_tokens)
        self.workspace = (torch.empty(max(nbytes, 16) // 4 + 4, dtype=torch.float32,
                                      device=q.device) if nbytes else None)
        pt = self.partition_tokens or abi.pa_decode_default_partition(B, hkv, self.max_context_len)
        self.partition = pt
        self.max_parts = max(1, -(-self.max_context_len // pt))

    def launches(self) -> int:
        """Kernels one run() launches."""
        n = 2 + (1 if self.max_parts > 1 else 0)
        if self.copy_pairs is not None and self.copy_pairs.numel():
            n += 1
        return n

    def copy(self, stream=None):
        if self.copy_pairs is not None and self.copy_pairs.numel():
            abi.pa_copy_blocks(self.k_cache, self.v_cache, self.copy_pairs, stream)

    def write(self, stream=None):
        abi.pa_reshape_and_cache(self.k_new, self.v_new, self.slot_mapping, self.k_cache,
                                 self.v_cache, stream)

    def attend(self, stream=None):
        abi.pa_decode(self.out, self.q, self.k_cache, self.v_cache, self.block_tables,
                      self.context_lens, self.max_context_len, self.scale, self.workspace,
                      self.partition_tokens, stream)

    def run(self, stream=None):
        self.copy(stream)
        self.write(stream)
        self.attend(stream)
        return self.out


class HostDecodeStep:
    """A DecodeStep whose per-step inputs and output live in pinned host memory.

    The KV pools stay resident on the device (they are the cache); every run()
    copies q, the new K/V, the slots, the block tables, the lengths and any
    copy pairs host->device, runs the step and copies the output back."""

    def __init__(self, *, k_cache, v_cache, q, k_new, v_new, slot_mapping, block_tables,
                 context_lens, max_context_len: int, scale: float, partition_tokens: int = 0,
                 copy_pairs=None):
        dev = k_cache.device

        def pin(t):
            return t.detach().to("cpu").contiguous().pin_memory()

        self.h_in = {"q": pin(q), "k_new": pin(k_new), "v_new": pin(v_new),
                     "slot_mapping": pin(slot_mapping), "block_tables": pin(block_tables),
                     "context_lens": pin(context_lens)}
        if copy_pairs is not None and copy_pairs.numel():
            self.h_in["copy_pairs"] = pin(copy_pairs)
        self.d_in = {k: torch.empty_like(v, device=dev) for k, v in self.h_in.items()}
        self.step = DecodeStep(k_cache=k_cache, v_cache=v_cache, q=self.d_in["q"],
                               k_new=self.d_in["k_new"], v_new=self.d_in["v_new"],
                               slot_mapping=self.d_in["slot_mapping"],
                               block_tables=self.d_in["block_tables"],
                               context_lens=self.d_in["context_lens"],
                               max_context_len=max_context_len, scale=scale,
                               partition_tokens=partition_tokens,
                               copy_pairs=self.d_in.get("copy_pairs"))
        self.h_out = torch.empty(tuple(q.shape), dtype=q.dtype).pin_memory()

    @property
    def h2d_bytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in self.h_in.values())

    @property
    def d2h_bytes(self) -> int:
        return self.h_out.numel() * self.h_out.element_size()

    def launches(self) -> int:
        return self.step.launches()

    def run(self, stream=None):
        for k, h in self.h_in.items():
            self.d_in[k].copy_(h, non_blocking=True)
        out = self.step.run(stream)
        self.h_out.copy_(out, non_blocking=True)
        return self.h_out
