"""pa_decode_static_workspace: paged decode for callers that cannot allocate.

Some callers of this library cannot call cudaMalloc: a host framework that owns
all device memory through its own pooled allocator, or a plug-in that may only
touch the buffers it is handed. For them pa_decode_static_workspace keeps the
split-context scratch in a fixed device array inside the library instead of a
caller-provided workspace. These checks call it through the C ABI, twice in a
row (the array keeps the previous call's contents), and compare each output
with pa_decode's on the same inputs within the tolerance the parity tests use;
a call that needs more scratch than the array holds must be refused.

This file is named to be collected last, and also passes on its own in a fresh
process (the first call looks up the array's address).
"""
import ctypes

import pytest
import torch

import synth
from gpu_harness import GpuBatch, widen_out
from paged_kv_cache_370_b200 import abi
from tolerance import assert_close

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)


def _static_call(step, out, partition_tokens):
    """The new entry point, called through the C ABI with raw pointers."""
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


@pytest.mark.parametrize("partition_tokens", [0, 1024])
def test_static_workspace_matches_pa_decode(partition_tokens):
    batch = synth.llama8b()  # 64 sequences up to 2048 tokens: several partitions each
    g = GpuBatch(batch, partition_tokens=partition_tokens)
    ref = widen_out(g.run())  # pa_decode with a caller-provided workspace
    need = abi.pa_decode_workspace_size(batch.num_seqs, batch.num_q_heads, batch.num_kv_heads,
                                        batch.head_dim, batch.max_context_len, partition_tokens)
    assert 0 < need <= abi.PA_STATIC_WORKSPACE_BYTES
    for call in range(2):
        out = torch.full_like(g.step.out, float("nan"))
        assert _static_call(g.step, out, partition_tokens) == abi.PA_OK
        torch.cuda.synchronize()
        assert_close(widen_out(out), ref, batch.dtype, f"static workspace, call {call + 1}")
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
