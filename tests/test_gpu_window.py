"""Sliding-window decode on a B200 against the oracle's window decode.

Every case also checks what the window leaves behind is never touched: the
pool rows before each sequence's window hold NaN, and the table entries of
blocks wholly before it name a block outside the pool (what a released entry
may hold) -- a read of either would show in the output or in the device
error word.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_harness import GpuBatch, NAN_BITS, oracle_pools, widen_out
from paged_kv_cache_370_b200 import abi
from tolerance import assert_close

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU machines too; every test here needs the GPU
    pytest.skip("no CUDA device", allow_module_level=True)


def _lo(n, w):
    return n - w if 0 < w < n else 0


def _forget(batch, window):
    """Tables whose entries before each window name a block outside the pool."""
    t = np.array(batch.block_tables, dtype=np.int32, copy=True)
    for b in range(batch.num_seqs):
        t[b, :_lo(int(batch.context_lens[b]), window) // batch.block_size] = batch.num_blocks + 7
    return t


def _poison_before_window(g, batch, window):
    bs = batch.block_size
    nan = NAN_BITS[batch.dtype]
    nan = nan - (1 << 16) if nan >= 1 << 15 else nan
    for b in range(batch.num_seqs):
        lo = _lo(int(batch.context_lens[b]), window)
        if lo == 0:
            continue
        t = np.arange(lo)
        blk = torch.from_numpy(batch.block_tables[b][t // bs].astype(np.int64)).cuda()
        off = torch.from_numpy(t % bs).cuda()
        g.k_cache.view(torch.int16)[blk, :, off, :] = nan
        g.v_cache.view(torch.int16)[blk, :, off, :] = nan


def _window_case(batch, window, partition_tokens=0, fused=False, sample=None):
    g = GpuBatch(batch, partition_tokens=partition_tokens, fused=fused, window=window,
                 step_tables=_forget(batch, window))
    _poison_before_window(g, batch, window)
    out = widen_out(g.run())
    code = abi.pa_device_status()
    assert code == 0, f"device error word {code:#x}: something before the window was read"
    kp, vp = oracle_pools(batch, full=sample is None)
    if sample is None:
        ref = oracle.decode_window(batch.q, kp, vp, batch.block_tables, batch.context_lens,
                                   batch.scale, batch.dtype, window)
        return assert_close(out, ref, batch.dtype, f"{batch.name} window {window}",
                            ulp_branch=batch.name == "long_skew")
    ref = oracle.decode_window(batch.q[sample], kp, vp, batch.block_tables[sample],
                               batch.context_lens[sample], batch.scale, batch.dtype, window)
    return assert_close(out[sample], ref, batch.dtype, f"{batch.name} window {window}",
                        ulp_branch=batch.name == "long_skew")


SHAPES = [
    # (Hq, Hkv, D, dtype, bs, lens)
    (4, 4, 64, "f16", 16, [0, 1, 15, 16, 17, 63, 64, 65, 200]),       # SIMT kernel (one q head per kv head)
    (32, 8, 128, "bf16", 16, [1, 31, 32, 33, 129, 511, 512, 513, 700]),
    (16, 8, 128, "f16", 8, [2, 9, 100, 257, 640]),
    (16, 4, 64, "bf16", 32, [5, 64, 65, 300]),
    (32, 4, 128, "bf16", 256, [1, 255, 256, 257, 900]),
    (8, 4, 128, "f16", 12, [3, 12, 13, 100, 250]),                     # block size not a power of two
]
WINDOWS = [1, 15, 16, 17, 64, 100, 256, 4096]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"h{s[0]}-{s[1]}d{s[2]}{s[3]}bs{s[4]}")
@pytest.mark.parametrize("mode", ["pt0", "pt64", "fused"])
def test_window_shapes(shape, mode):
    hq, hkv, d, dt, bs, lens = shape
    width = -(-max(lens) // bs) + 1
    nb = len(lens) * width + 3
    batch = synth.small_random(41 + bs, len(lens), lens, hq, hkv, d, bs, nb, dt, width=width)
    fused = mode == "fused"  # with a window: the write kernel, then the decode
    pt = 64 if mode == "pt64" else 0
    for w in WINDOWS:
        _window_case(batch, w, partition_tokens=pt, fused=fused)


def test_window_covering_everything_is_plain_decode():
    """A window at least as long as every context changes nothing: within
    tolerance of the plain oracle decode, and the same bits for any such window."""
    batch = synth.small_random(47, 4, [7, 100, 513, 64], 32, 8, 128, 16, 200, "bf16")
    outs = []
    for w in (513, 10_000):
        g = GpuBatch(batch, window=w)
        outs.append(g.run().clone())
        assert g.step.launches() == 1 + abi.pa_decode_window_launches(
            4, 32, 8, 128, 16, 200, batch.max_context_len, w)
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    kp, vp = oracle_pools(batch)
    ref = oracle.decode(batch.q, kp, vp, batch.block_tables, batch.context_lens, batch.scale,
                        batch.dtype)
    assert_close(widen_out(outs[0]), ref, batch.dtype, "window covering everything")


def test_window_rejects_nonpositive():
    batch = synth.small_random(48, 2, [5, 9], 8, 4, 64, 16, 8, "f16")
    g = GpuBatch(batch)
    with pytest.raises(abi.PAError):
        abi.pa_decode_window(g.step.out, g.step.q, g.k_cache, g.v_cache, g.step.block_tables,
                             g.step.context_lens, g.step.max_context_len, g.step.scale, 0,
                             g.step.workspace)


@pytest.mark.parametrize("window", [1000, 4096])
def test_window_llama8b_full(window):
    """The Llama-3.1-8B-shaped batch with a window, fused write, every output of a
    sample of 16 sequences against the oracle."""
    batch = synth.llama8b()
    sample = np.random.default_rng(3).choice(batch.num_seqs, size=16, replace=False)
    s = _window_case(batch, window, fused=True, sample=sample)
    print(f"\nllama8b window {window}: {s}")


def test_window_long_skew_full():
    batch = synth.long_skew()
    s = _window_case(batch, 4096, sample=np.arange(batch.num_seqs))
    print(f"\nlong_skew window 4096: {s}")


@pytest.mark.parametrize("fused", [False, True])
def test_window_bad_inputs_are_reported_not_accessed(fused):
    """Bad block ids and lengths under a window (the remap route of the even-split
    kernel and its fused write): reported in the device error word, never used to
    address memory, and the context stays usable."""
    batch = synth.small_random(49, 3, [40, 70, 9], 8, 2, 128, 16, 20, "bf16")
    g = GpuBatch(batch, window=32, fused=fused)
    g.run()
    assert abi.pa_device_status() == 0
    bad = batch.block_tables.copy()
    bad[1, 3] = batch.num_blocks + 1000      # inside sequence 1's window (positions 38..69)
    g.step.block_tables.copy_(torch.from_numpy(bad).cuda())
    g.run()
    assert abi.pa_device_status() & abi.PA_DEVERR_BLOCK_ID
    g.step.block_tables.copy_(torch.from_numpy(batch.block_tables).cuda())
    g.step.context_lens[2] = 10_000          # beyond the table and max_context_len
    g.run()
    assert abi.pa_device_status() & abi.PA_DEVERR_CONTEXT_LEN
    g.step.context_lens.copy_(torch.from_numpy(batch.context_lens).cuda())
    out = widen_out(g.run())
    assert abi.pa_device_status() == 0
    kp, vp = oracle_pools(batch)
    ref = oracle.decode_window(batch.q, kp, vp, batch.block_tables, batch.context_lens,
                               batch.scale, batch.dtype, 32)
    assert_close(out, ref, batch.dtype, "window after bad inputs")


def test_window_overlapped_launch_gives_the_same_bits():
    """pa_decode_append_window_overlapped (the windowed kernel may start during the
    preceding kernel's tail) returns the bits of pa_decode_append_window, also when
    its launches follow each other back to back and inside a CUDA graph; the
    entries and rows before each window are still never read."""
    batch = synth.llama8b()
    window = 1024
    ref = GpuBatch(batch, fused=True, window=window, step_tables=_forget(batch, window))
    _poison_before_window(ref, batch, window)
    want = ref.run().clone()
    assert abi.pa_device_status() == 0
    del ref
    g = GpuBatch(batch, fused=True, window=window, step_tables=_forget(batch, window))
    _poison_before_window(g, batch, window)
    g.step.overlapped = True
    for _ in range(3):  # each launch follows the previous one on the stream
        g.step.append()
    torch.cuda.synchronize()
    assert abi.pa_device_status() == 0
    assert torch.equal(g.step.out.view(torch.int16), want.view(torch.int16))
    graph = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            g.step.append()
            g.step.append()
    torch.cuda.current_stream().wait_stream(s)
    g.step.out.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert abi.pa_device_status() == 0
    assert torch.equal(g.step.out.view(torch.int16), want.view(torch.int16))
