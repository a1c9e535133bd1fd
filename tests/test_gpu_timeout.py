"""The decode kernels' bounded waits, made to run out on purpose, on a B200.

Every wait of a decode kernel on its pipeline barriers is bounded; when one
runs out the kernel reports PA_DEVERR_TIMEOUT, finishes without waiting for
data again and returns, so the host sees an error status and the context
stays usable. The library's test mode (pa_debug_wait_test) makes this happen
without faulting or hanging anything: the producer warps issue no copy and
arrive on no data barrier, and the consumers give up each data wait after a
few microseconds. Nothing is in flight when the CTAs exit. These checks run
that mode on both decode kernels, then a normal call on the same buffers,
which must match the oracle again.
"""
import time

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

WAIT_NS = 20_000  # the consumers' data waits give up after 20 us

CASES = {
    # the even-split tensor-core kernel (GQA 4, power-of-two blocks); long
    # sequences are split between CTAs, so the piece merge runs too
    "even_split": ((32, 8, 128, "bf16", 16), [1, 700, 2049, 64, 3000, 333]),
    # the partition kernel (one q head per kv head) with its merge kernel
    "partition": ((8, 8, 128, "f16", 16), [1, 700, 2049, 64, 3000, 333]),
}


def _batch(case):
    (hq, hkv, d, dt, bs), lens = CASES[case]
    width = -(-max(lens) // bs)
    return synth.small_random(90 + len(case), len(lens), lens, hq, hkv, d, bs,
                              len(lens) * width + 5, dt, width)


def _starved(fn):
    """Run fn() in the test mode of the bounded waits; return the seconds it took
    on the device and the device error word."""
    torch.cuda.synchronize()
    abi.pa_debug_wait_test(True, WAIT_NS)
    try:
        t0 = time.perf_counter()
        fn()
        torch.cuda.synchronize()
        dt = time.perf_counter() - t0
    finally:
        abi.pa_debug_wait_test(False)
    return dt, abi.pa_device_status()


@pytest.mark.parametrize("case", sorted(CASES))
def test_wait_runs_out_and_context_recovers(case):
    batch = _batch(case)
    g = GpuBatch(batch, partition_tokens=512)
    ref = oracle_decode(batch, *oracle_pools(batch))
    assert_close(widen_out(g.run()), ref, batch.dtype, f"{case} before")
    assert abi.pa_device_status() == 0
    k0, v0 = to_bits(g.k_cache), to_bits(g.v_cache)

    dt, code = _starved(g.step.attend)
    assert code & abi.PA_DEVERR_TIMEOUT, f"no timeout reported ({code:#x})"
    assert code == abi.PA_DEVERR_TIMEOUT, f"unexpected error bits {code:#x}"
    assert dt < 1.0, f"the short limit was not used ({dt:.3f} s)"
    # the pools are untouched by the call that gave up
    assert np.array_equal(to_bits(g.k_cache), k0) and np.array_equal(to_bits(g.v_cache), v0)

    # as pa.h asks after a timeout: zero-fill the workspace, then call again
    if g.step.workspace is not None:
        g.step.workspace.zero_()
    out = widen_out(g.run())
    assert abi.pa_device_status() == 0
    assert_close(out, ref, batch.dtype, f"{case} after the timeout")


def test_fused_write_is_skipped_after_a_give_up():
    """pa_decode_append in the test mode: the new rows never land, so the kernel
    must not store them; the pools keep their bits. Then the normal fused call
    writes them and matches the oracle."""
    batch = _batch("even_split")
    g = GpuBatch(batch, partition_tokens=512, fused=True)
    kp, vp = oracle_pools(batch)
    new = batch.new_token_rows()
    slots = abi.pa_slot_mapping(batch.block_tables, batch.context_lens, batch.block_size)[new]
    # wipe the new tokens' rows so that a write would show
    bs = batch.block_size
    s = torch.from_numpy(slots).cuda()
    g.k_cache[s // bs, :, s % bs, :] = 0
    g.v_cache[s // bs, :, s % bs, :] = 0
    torch.cuda.synchronize()
    k0, v0 = to_bits(g.k_cache), to_bits(g.v_cache)
    dt, code = _starved(g.step.append)
    assert code == abi.PA_DEVERR_TIMEOUT, f"error word {code:#x}"
    assert np.array_equal(to_bits(g.k_cache), k0) and np.array_equal(to_bits(g.v_cache), v0)
    g.step.workspace.zero_()
    out = widen_out(g.run())
    assert abi.pa_device_status() == 0
    assert np.array_equal(to_bits(g.k_cache), kp) and np.array_equal(to_bits(g.v_cache), vp)
    assert_close(out, oracle_decode(batch, kp, vp), batch.dtype, "fused after the timeout")


def test_test_mode_is_off_again():
    """After the hook is switched off a decode needs no short limit: a batch large
    enough to keep every CTA busy for many tiles runs clean."""
    batch = synth.llama8b()
    g = GpuBatch(batch)
    g.run()
    assert abi.pa_device_status() == 0
