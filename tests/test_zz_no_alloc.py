"""pa_decode_static_workspace: paged decode for callers that cannot allocate.

Some callers of this library cannot call cudaMalloc: a host framework that owns
all device memory through its own pooled allocator, or a plug-in that may only
touch the buffers it is handed. For them pa_decode_static_workspace keeps the
split-context scratch in a fixed device array inside the library instead of a
caller-provided workspace. These checks call it through the C ABI, twice in a
row (the array keeps the previous call's contents), and require each output to
be bit-identical to pa_decode's on the same inputs (same kernels, same
schedule) and within the parity tolerance of the fp64 oracle; on the even-split
tensor-core kernel and on the partition kernel with its merge kernel. A call
after one whose waits ran out (the array's counters may then be left non-zero)
must still be exact, and a call that needs more scratch than the array holds
must be refused.

This file is named to be collected last, and also passes on its own in a fresh
process (the first call looks up the array's address).
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from gpu_harness import GpuBatch, oracle_decode, oracle_pools, to_bits, widen_out
from paged_kv_cache_370_b200 import abi
from tolerance import assert_close

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)


def _static_call(step, out, partition_tokens):
    """The entry point, called through the C ABI with raw pointers."""
    q, kc = step.q, step.k_cache
    B, hq, d = q.shape
    nb, hkv, bs, _ = kc.shape
    code = abi.PA_BF16 if q.dtype == torch.bfloat16 else abi.PA_F16
    return abi.lib().pa_decode_static_workspace(
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(q.data_ptr()),
        ctypes.c_void_p(kc.data_ptr()), ctypes.c_void_p(step.v_cache.data_ptr()),
        ctypes.c_void_p(step.block_tables.data_ptr()), int(step.block_tables.shape[1]),
        ctypes.c_void_p(step.context_lens.data_ptr()), int(step.max_context_len), B, hq, hkv, d,
        bs, nb, float(step.scale), code, int(partition_tokens),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _check_twice(batch, partition_tokens, stream_kernel):
    g = GpuBatch(batch, partition_tokens=partition_tokens)
    ref = g.run().clone()  # pa_decode with a caller-provided workspace (after the KV write)
    nb, hkv, bs, d = g.k_cache.shape
    ctas = abi.pa_decode_grid_ctas(batch.num_seqs, batch.num_q_heads, hkv, d, bs, nb,
                                   batch.max_context_len, partition_tokens)
    assert (ctas > 0) == stream_kernel, f"expected the {'even-split' if stream_kernel else 'partition'} kernel"
    exact = oracle_decode(batch, *oracle_pools(batch, full=False))
    for call in range(2):
        out = torch.full_like(g.step.out, float("nan"))
        assert _static_call(g.step, out, partition_tokens) == abi.PA_OK
        torch.cuda.synchronize()
        assert np.array_equal(to_bits(out), to_bits(ref)), f"call {call + 1}: bits differ from pa_decode"
        assert_close(widen_out(out), exact, batch.dtype, f"static workspace, call {call + 1}")
    assert abi.pa_device_status() == 0
    return g, ref


@pytest.mark.parametrize("partition_tokens", [0, 1024])
def test_static_workspace_even_split_kernel(partition_tokens):
    # 64 sequences up to 2048 tokens, GQA 4, 16-token blocks: sequences split between CTAs
    _check_twice(synth.llama8b(), partition_tokens, stream_kernel=True)


def test_static_workspace_partition_kernel():
    # one q head per kv head and 256-token blocks: the partition kernel, several
    # partitions per sequence, merged by the second kernel
    lens = [1, 300, 2048, 1500, 777, 4000, 64, 2600]
    batch = synth.small_random(77, len(lens), lens, 16, 16, 128, 256, len(lens) * 16 + 3, "f16", 16)
    _check_twice(batch, 512, stream_kernel=False)


def test_static_workspace_after_a_timeout():
    """A call whose waits ran out (the library's test mode) may leave the even-split
    kernel's counters non-zero in the shared array; the next call must still be exact."""
    batch = synth.llama8b()
    g, ref = _check_twice(batch, 0, stream_kernel=True)
    abi.pa_debug_wait_test(True, 20_000)
    try:
        junk = torch.empty_like(g.step.out)
        assert _static_call(g.step, junk, 0) == abi.PA_OK
        torch.cuda.synchronize()
    finally:
        abi.pa_debug_wait_test(False)
    assert abi.pa_device_status() & abi.PA_DEVERR_TIMEOUT
    for call in range(2):
        out = torch.full_like(g.step.out, float("nan"))
        assert _static_call(g.step, out, 0) == abi.PA_OK
        torch.cuda.synchronize()
        assert np.array_equal(to_bits(out), to_bits(ref)), f"call {call + 1} after the timeout"
    assert abi.pa_device_status() == 0


def test_static_workspace_refuses_oversized_calls():
    # a valid call whose 64-token pieces need more scratch than the array holds
    batch = synth.llama8b()
    g = GpuBatch(batch, partition_tokens=64)
    need = abi.pa_decode_workspace_size(batch.num_seqs, batch.num_q_heads, batch.num_kv_heads,
                                        batch.head_dim, batch.max_context_len, 64)
    assert need > abi.PA_STATIC_WORKSPACE_BYTES
    out = torch.zeros_like(g.step.out)
    assert _static_call(g.step, out, 64) == abi.PA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0, "a refused call must launch nothing"
