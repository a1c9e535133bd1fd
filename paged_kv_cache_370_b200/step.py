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
``HostStepPipeline`` runs many host-fed steps with their copies hidden under
other steps' kernels.
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
        # (pa_decode_append_overlapped, pa_decode_append_window_overlapped); the
        # lengths, tables and slots must not be written by that kernel
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
        if self.window > 0:
            self.decode_launches = abi.pa_decode_window_launches(
                B, hq, hkv, d, bs, nb, self.max_context_len, self.window, self.partition_tokens)
            self.append_launches = abi.pa_decode_append_window_launches(
                B, hq, hkv, d, bs, nb, self.max_context_len, self.window, self.partition_tokens)
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
                                        self.workspace, self.partition_tokens, stream,
                                        overlapped=self.overlapped)
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
                 copy_pairs=None, fused: bool = False, window: int = 0,
                 overlapped: bool = False):
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
                               copy_pairs=views.get("copy_pairs"), fused=fused, window=window,
                               overlapped=overlapped)
        self.h_out = torch.empty(tuple(q.shape), dtype=q.dtype).pin_memory()
        self._in_ready = torch.cuda.Event()
        self._done = torch.cuda.Event()

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

    def enqueue(self, copy_in, compute, copy_out):
        """The same step spread over three streams so that consecutive steps overlap:
        the upload on ``copy_in``, the kernels on ``compute`` once the upload landed,
        the download on ``copy_out`` once the kernels finished. Steps enqueued one
        after another on the same three streams pipeline: the next step's upload and
        the previous step's download run under this step's kernels, while the
        kernels themselves stay in order on ``compute`` (each step reads the pools
        the previous one wrote). The caller must not enqueue the same step again
        before its previous use completed (its buffers are reused); ``h_out`` holds
        the result once ``copy_out`` has passed this point."""
        with torch.cuda.stream(copy_in):
            self.d_in.copy_(self.h_in, non_blocking=True)
            self._in_ready.record(copy_in)
        compute.wait_event(self._in_ready)
        with torch.cuda.stream(compute):
            self.step.run()
            self._done.record(compute)
        copy_out.wait_event(self._done)
        with torch.cuda.stream(copy_out):
            self.h_out.copy_(self.step.out, non_blocking=True)
        return self.h_out

    def upload(self):
        self.d_in.copy_(self.h_in, non_blocking=True)

    def download(self):
        self.h_out.copy_(self.step.out, non_blocking=True)


class HostStepPipeline:
    """Host-fed steps run back to back with every copy under some step's kernels.

    The steps come in sets (rounds), each a list of HostDecodeStep with buffers of
    its own. Each round has three CUDA graphs: the uploads of its steps' inputs,
    its steps' kernels, and the downloads of its steps' outputs. ``run`` /
    ``run_order`` replay rounds on three streams so that the next round's uploads
    and the previous round's downloads run while a round's kernels do. Because the
    graph of kernels has no copy nodes in it, each decode kernel keeps its
    programmatic dependency on the one before it (the early start of an
    ``overlapped`` step). Rounds' kernels run in order on the caller's stream, so
    the steps see the pools in the order given.

    Only the first round's uploads and the last round's downloads are not hidden,
    so a short run is best served by rounds that grow from one step and shrink
    back to one (``ramp_sizes``); a long one by two rounds taking turns.

    A round's buffers are reused when it comes again: its uploads wait for its
    previous kernels to finish, and its kernels for its previous downloads."""

    def __init__(self, rounds):
        if len(rounds) < 1 or not all(rounds):
            raise ValueError("non-empty rounds of HostDecodeStep are needed")
        self.rounds = [list(r) for r in rounds]
        n = len(self.rounds)
        self.s_in = torch.cuda.Stream()
        self.s_out = torch.cuda.Stream()
        self._graphs = None
        self._up = [torch.cuda.Event() for _ in range(n)]
        self._comp = [torch.cuda.Event() for _ in range(n)]
        self._down = [torch.cuda.Event() for _ in range(n)]

    @staticmethod
    def ramp_sizes(num_steps: int, cap: int = 16, kernel_us: float = 55.0,
                   upload_us: float = 16.0, download_us: float = 10.0,
                   boundary_us: float = 10.0) -> list[int]:
        """Round sizes for one pass of num_steps host-fed steps. A round's uploads
        run under the kernels of the round before it and its downloads under those
        of the round after it, so consecutive sizes may grow at most by the ratio
        of a step's kernel time to its upload time and shrink at most by the ratio
        to its download time (defaults: the Llama-3.1-8B-shaped batch, ~55 us of
        kernels, ~16 and ~10 us of PCIe per step). What stays exposed is the first
        round's uploads, the last round's downloads and a gap at each round
        boundary; the sizes (at most ``cap``) minimise that sum."""
        # (copies slower than the kernels cannot be hidden whatever the sizes: then
        # rounds may still keep their size)
        grow = max(1.0, kernel_us / max(upload_us, 1e-9))
        shrink = max(1.0, kernel_us / max(download_us, 1e-9))
        if num_steps <= 0:
            return []
        sizes = range(1, min(cap, num_steps) + 1)
        # best[(left, prev)]: (cost, rest) of finishing `left` steps after a round of `prev`
        best = {}

        def solve(left, prev):
            key = (left, prev)
            if key in best:
                return best[key]
            out = (download_us * prev, [])  # prev is the last round
            if left > 0:
                out = (float("inf"), None)
                for s in sizes:
                    if s > left or s > grow * prev or prev > shrink * s:
                        continue
                    c, rest = solve(left - s, s)
                    if rest is not None and c + boundary_us < out[0]:
                        out = (c + boundary_us, [s] + rest)
            best[key] = out
            return out

        cands = []
        for s0 in sizes:
            c, rest = solve(num_steps - s0, s0)
            if rest is not None:
                cands.append((upload_us * s0 + c, [s0] + rest))
        return min(cands)[1]

    @property
    def steps_per_round(self):
        return [len(r) for r in self.rounds]

    def launches(self, round_index: int) -> int:
        return sum(h.launches() for h in self.rounds[round_index])

    def capture(self):
        """Capture the six graphs (after one eager pass that warms every launch path)."""
        cur = torch.cuda.current_stream()
        side = torch.cuda.Stream()
        side.wait_stream(cur)
        phases = []
        with torch.cuda.stream(side):
            for r in self.rounds:
                for h in r:
                    h.upload()
                for h in r:
                    h.step.run()
                for h in r:
                    h.download()
            torch.cuda.synchronize()
            for r in self.rounds:
                gs = []
                for fn in (lambda r=r: [h.upload() for h in r],
                           lambda r=r: [h.step.run() for h in r],
                           lambda r=r: [h.download() for h in r]):
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=side):
                        fn()
                    gs.append(g)
                phases.append(gs)
        cur.wait_stream(side)
        torch.cuda.synchronize()
        self._graphs = phases
        # nothing is in flight: every round's buffers are free
        for e in self._comp + self._down:
            e.record(cur)

    def graph(self, order):
        """One CUDA graph of the rounds ``order`` lists, enqueued as ``run_order``
        enqueues them: uploads on one side stream, kernels on the capturing stream,
        downloads on another, joined by events inside the graph. Replaying it costs
        one launch from the host, however short the rounds (``run_order`` needs a few
        host calls per round, which can take longer than a short round's kernels).
        The rounds' per-phase graphs need not have been captured; run each step once
        before (e.g. ``capture`` or ``run_order``) so that every launch path is warm."""
        cur = torch.cuda.current_stream()
        cs, s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        g = torch.cuda.CUDAGraph()
        comp, down = {}, {}
        cs.wait_stream(cur)
        with torch.cuda.graph(g, stream=cs):
            s_in.wait_stream(cs)
            s_out.wait_stream(cs)
            for x in order:
                r = self.rounds[x]
                if x in comp:  # this set's buffers: free once its previous kernels ran
                    s_in.wait_event(comp[x])
                with torch.cuda.stream(s_in):
                    for h in r:
                        h.upload()
                up = torch.cuda.Event()
                up.record(s_in)
                cs.wait_event(up)
                if x in down:  # and once its previous outputs were read back
                    cs.wait_event(down[x])
                for h in r:
                    h.step.run()
                comp[x] = torch.cuda.Event()
                comp[x].record(cs)
                s_out.wait_event(comp[x])
                with torch.cuda.stream(s_out):
                    for h in r:
                        h.download()
                down[x] = torch.cuda.Event()
                down[x].record(s_out)
            cs.wait_stream(s_in)
            cs.wait_stream(s_out)
        cur.wait_stream(cs)
        torch.cuda.synchronize()
        return g

    def run(self, n_rounds: int):
        """Enqueue ``n_rounds`` rounds (the sets in turn) on the current stream and
        the two copy streams; on return the current stream is ordered after every
        copy. Results are in each step's ``h_out`` once the stream passes."""
        self.run_order([i % len(self.rounds) for i in range(n_rounds)])

    def run_order(self, order):
        """Enqueue the rounds whose indices ``order`` lists, in that order (as ``run``)."""
        if self._graphs is None:
            self.capture()
        cs = torch.cuda.current_stream()
        self.s_in.wait_stream(cs)
        self.s_out.wait_stream(cs)
        for x in order:
            up, comp, down = self._graphs[x]
            self.s_in.wait_event(self._comp[x])
            with torch.cuda.stream(self.s_in):
                up.replay()
            self._up[x].record(self.s_in)
            cs.wait_event(self._up[x])
            cs.wait_event(self._down[x])
            comp.replay()
            self._comp[x].record(cs)
            self.s_out.wait_event(self._comp[x])
            with torch.cuda.stream(self.s_out):
                down.replay()
            self._down[x].record(self.s_out)
        cs.wait_stream(self.s_in)
        cs.wait_stream(self.s_out)
