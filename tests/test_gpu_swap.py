"""Swap of KV blocks between the device pools and a pinned host swap space, on a
B200: bit-exact against the oracle's block assignment, and a swapped-out group
decodes to the same bits once it is back (in other blocks)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_harness import GpuBatch, oracle_decode, oracle_pools, to_bits, to_dev, widen_out
from paged_kv_cache_370_b200 import abi
from tolerance import assert_close

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU machines too; every test here needs the GPU
    pytest.skip("no CUDA device", allow_module_level=True)


def _status_clean():
    code = abi.pa_device_status()
    assert code == 0, f"device error word {code:#x}"


@pytest.mark.parametrize("shape,dtype", [((96, 8, 16, 128), "bf16"), ((40, 4, 32, 64), "f16")])
def test_swap_out_and_in_bit_exact(shape, dtype):
    rng = np.random.default_rng(31)
    nb = shape[0]
    nh = 50
    kb = rng.integers(0, 1 << 16, size=shape, dtype=np.uint64).astype(np.uint16)
    vb = rng.integers(0, 1 << 16, size=shape, dtype=np.uint64).astype(np.uint16)
    kc, vc = to_dev(kb, dtype), to_dev(vb, dtype)
    space = abi.SwapSpace(nh, *shape[1:], dtype)
    hshape = (nh,) + shape[1:]
    hk0 = rng.integers(0, 1 << 16, size=hshape, dtype=np.uint64).astype(np.uint16)
    hv0 = rng.integers(0, 1 << 16, size=hshape, dtype=np.uint64).astype(np.uint16)
    space.k_host[...] = hk0
    space.v_host[...] = hv0
    # out: 30 distinct device blocks to 30 distinct host blocks
    out_pairs = np.stack([rng.permutation(nb)[:30], rng.permutation(nh)[:30]], 1).astype(np.int64)
    abi.pa_swap_out(space, kc, vc, torch.from_numpy(out_pairs).cuda())
    torch.cuda.synchronize()
    ek, ev = hk0.copy(), hv0.copy()
    oracle.swap_blocks(ek, ev, kb, vb, out_pairs)
    assert np.array_equal(space.k_host, ek) and np.array_equal(space.v_host, ev)
    # in: those host blocks back into other device blocks
    in_pairs = np.stack([out_pairs[:, 1], rng.permutation(nb)[:30]], 1).astype(np.int64)
    abi.pa_swap_in(space, kc, vc, torch.from_numpy(in_pairs).cuda())
    torch.cuda.synchronize()
    oracle.swap_blocks(kb, vb, ek, ev, in_pairs)
    assert np.array_equal(to_bits(kc), kb) and np.array_equal(to_bits(vc), vb)
    _status_clean()
    # an id outside either pool is reported and that pair skipped
    bad = torch.tensor([[0, nh + 7]], dtype=torch.int64, device="cuda")
    abi.pa_swap_out(space, kc, vc, bad)
    assert abi.pa_device_status() & abi.PA_DEVERR_COPY_PAIR
    assert np.array_equal(space.k_host, ek)
    space.close()


def test_swapped_group_decodes_to_the_same_bits():
    """Decode a batch, swap every sequence out through the block manager (the
    device pool is then overwritten with NaN, as reuse by others would), swap
    back into fresh blocks and decode again: bit-identical outputs (the result
    depends on logical order only), within tolerance of the oracle."""
    batch = synth.small_random(32, 6, [1, 17, 64, 100, 333, 511], 32, 8, 128, 16, 400, "bf16")
    bs = batch.block_size
    mgr = abi.BlockManager(batch.num_blocks, bs)
    mgr.set_host_blocks(256)
    for b in range(batch.num_seqs):
        mgr.add_seq(b, int(batch.context_lens[b]))
    width = batch.block_tables.shape[1]
    tables, lens = mgr.fill_tables(list(range(batch.num_seqs)), width, pad=0)
    g = GpuBatch(batch, tables=tables)
    out1 = g.run().clone()
    _status_clean()
    pairs = mgr.swap_out(range(batch.num_seqs))
    assert mgr.num_free() == batch.num_blocks
    space = abi.SwapSpace(256, batch.num_kv_heads, bs, batch.head_dim, batch.dtype)
    abi.pa_swap_out(space, g.k_cache, g.v_cache, torch.from_numpy(pairs).cuda())
    torch.cuda.synchronize()
    g.k_cache.view(torch.int16).fill_(0x7FC0)
    g.v_cache.view(torch.int16).fill_(0x7FC0)
    # take some blocks first so the group comes back to other ids
    mgr.add_seq(1000, 5 * bs)
    back = mgr.swap_in(list(reversed(range(batch.num_seqs))))
    abi.pa_swap_in(space, g.k_cache, g.v_cache, torch.from_numpy(back).cuda())
    tables2, lens2 = mgr.fill_tables(list(range(batch.num_seqs)), width, pad=0)
    assert np.array_equal(lens2, lens) and not np.array_equal(tables2, tables)
    g.step.block_tables.copy_(torch.from_numpy(tables2).cuda())
    g.step.attend()
    out2 = g.step.out.clone()
    torch.cuda.synchronize()
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    kp, vp = oracle_pools(batch, tables=tables)
    assert_close(widen_out(out2), oracle_decode(batch, kp, vp, tables=tables), batch.dtype)
    _status_clean()
    space.close()
