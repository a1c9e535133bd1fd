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
                 copy_pairs=None, out=None, fused: bool = False, window: int = 0,
                 overlapped: bool = False):
        """``fused``: write the new tokens inside the decode (pa_decode_append);
        k_new/v_new then hold one token per sequence, at position len - 1.
        ``window`` > 0: attend to each sequence's last ``window`` positions only
        (pa_decode_window / pa_decode_append_window)."""
        self.fused = fused
        self.window = int(window)
        # fused steps only: the kernel may start during the preceding kernel's tail
        # (pa_decode_append_overlapped); the lengths, tables and slots must not be
        # written by that kernel
        self.overlapped = overlapped
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
        # zero-filled once: pa_decode keeps its counters zero between calls
        self.workspace = (torch.zeros(max(nbytes, 16) // 4 + 4, dtype=torch.float32,
                                      device=q.device) if nbytes else None)
        nb, _, bs, _ = k_cache.shape
        self.decode_launches = abi.pa_decode_launches(B, hq, hkv, d, bs, nb,
                                                      self.max_context_len,
                                                      self.partition_tokens)
        self.append_launches = abi.pa_decode_append_launches(B, hq, hkv, d, bs, nb,
                                                             self.max_context_len,
                                                             self.partition_tokens)
        if self.window > 0:  # the partition kernel (and merge), after a separate write
            self.decode_launches = abi.pa_decode_window_launches(B, hq, hkv, d,
                                                                 self.max_context_len,
                                                                 self.window,
                                                                 self.partition_tokens)
            self.append_launches = 1 + self.decode_launches
        self.partition = self.partition_tokens or abi.pa_decode_default_partition(
            B, hkv, self.max_context_len)

    def launches(self) -> int:
        """Kernels one run() launches."""
        n = self.append_launches if self.fused else 1 + self.decode_launches
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
        if self.window > 0:
            abi.pa_decode_window(self.out, self.q, self.k_cache, self.v_cache, self.block_tables,
                                 self.context_lens, self.max_context_len, self.scale, self.window,
                                 self.workspace, self.partition_tokens, stream)
            return
        abi.pa_decode(self.out, self.q, self.k_cache, self.v_cache, self.block_tables,
                      self.context_lens, self.max_context_len, self.scale, self.workspace,
                      self.partition_tokens, stream)

    def append(self, stream=None):
        if self.window > 0:
            abi.pa_decode_append_window(self.out, self.q, self.k_new, self.v_new,
                                        self.slot_mapping, self.k_cache, self.v_cache,
                                        self.block_tables, self.context_lens,
                                        self.max_context_len, self.scale, self.window,
                                        self.workspace, self.partition_tokens, stream)
            return
        fn = abi.pa_decode_append_overlapped if self.overlapped else abi.pa_decode_append
        fn(self.out, self.q, self.k_new, self.v_new, self.slot_mapping, self.k_cache,
           self.v_cache, self.block_tables, self.context_lens, self.max_context_len, self.scale,
           self.workspace, self.partition_tokens, stream)

    def run(self, stream=None):
        self.copy(stream)
        if self.fused:
            self.append(stream)
        else:
            self.write(stream)
            self.attend(stream)
        return self.out


class HostDecodeStep:
    """A DecodeStep whose per-step inputs and output live in pinned host memory.

    The KV pools stay resident on the device (they are the cache). The step's
    inputs -- q, the new K/V, the slots, the block tables, the lengths and any
    copy pairs -- are packed back to back (16-byte aligned) in one pinned host
    buffer, so every run() is one host->device copy, the step's kernels, and one
    device->host copy of the output."""

    def __init__(self, *, k_cache, v_cache, q, k_new, v_new, slot_mapping, block_tables,
                 context_lens, max_context_len: int, scale: float, partition_tokens: int = 0,
                 copy_pairs=None, fused: bool = False, window: int = 0):
        dev = k_cache.device
        parts = {"q": q, "k_new": k_new, "v_new": v_new, "slot_mapping": slot_mapping,
                 "block_tables": block_tables, "context_lens": context_lens}
        if copy_pairs is not None and copy_pairs.numel():
            parts["copy_pairs"] = copy_pairs
        offsets, total = {}, 0
        for name, t in parts.items():
            offsets[name] = total
            total += -(-t.numel() * t.element_size() // 16) * 16
        self.h_in = torch.empty(total, dtype=torch.uint8).pin_memory()
        self.d_in = torch.empty(total, dtype=torch.uint8, device=dev)
        views = {}
        for name, t in parts.items():
            n = t.numel() * t.element_size()
            src = t.detach().contiguous().view(torch.uint8).reshape(-1).cpu()
            self.h_in[offsets[name]:offsets[name] + n].copy_(src)
            views[name] = self.d_in[offsets[name]:offsets[name] + n].view(t.dtype).view(t.shape)
        self.step = DecodeStep(k_cache=k_cache, v_cache=v_cache, q=views["q"],
                               k_new=views["k_new"], v_new=views["v_new"],
                               slot_mapping=views["slot_mapping"],
                               block_tables=views["block_tables"],
                               context_lens=views["context_lens"],
                               max_context_len=max_context_len, scale=scale,
                               partition_tokens=partition_tokens,
                               copy_pairs=views.get("copy_pairs"), fused=fused, window=window)
        self.h_out = torch.empty(tuple(q.shape), dtype=q.dtype).pin_memory()

    @property
    def h2d_bytes(self) -> int:
        return self.h_in.numel()

    @property
    def d2h_bytes(self) -> int:
        return self.h_out.numel() * self.h_out.element_size()

    def launches(self) -> int:
        return self.step.launches()

    def run(self):
        self.d_in.copy_(self.h_in, non_blocking=True)
        out = self.step.run()
        self.h_out.copy_(out, non_blocking=True)
        return self.h_out
