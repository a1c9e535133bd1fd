"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, on a B200.

Writes and copies must match bit for bit; attention outputs must be within the
tolerance of ``tolerance.py``. Cases span several tiles and partitions with
ragged tails, every supported head_dim / group size, block sizes 1..256,
empty and length-1 contexts, and the five workloads at full size.
"""
import numpy as np
import pytest
import torch

import oracle
import pins
import synth
from gpu_harness import (GpuBatch, oracle_decode, oracle_pools, poisoned_pool, shared_prompt_gpu,
                         shared_prompt_oracle, to_bits, to_dev, widen_out)
from oracle.allocator_model import BlockManagerModel
from paged_kv_cache_370_b200 import abi
from tolerance import assert_close, compare

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU machines too; every test here needs the GPU
    pytest.skip("no CUDA device", allow_module_level=True)


def _status_clean():
    code = abi.pa_device_status()
    assert code == 0, f"device error word {code:#x}"


def _run_and_compare(batch, partition_tokens=0, full_pool=True, fused=False):
    g = GpuBatch(batch, partition_tokens=partition_tokens, fused=fused)
    out = widen_out(g.run())
    kp, vp = oracle_pools(batch, full=full_pool)
    if full_pool:
        assert np.array_equal(to_bits(g.k_cache), kp), "K pool differs from the oracle's"
        assert np.array_equal(to_bits(g.v_cache), vp), "V pool differs from the oracle's"
    ref = oracle_decode(batch, kp, vp)
    s = assert_close(out, ref, batch.dtype, batch.name)
    _status_clean()
    return g, out, ref, s


# ----------------------------------------------------------------------------- the tiny config
def test_tiny_config():
    batch = synth.tiny()
    g, out, ref, s = _run_and_compare(batch)
    # a context of one token returns that token's V exactly
    b1 = int(np.nonzero(batch.context_lens == 1)[0][0])
    v = pins.lib_f64(batch.v[batch.seq_start[b1]], batch.dtype)
    assert np.array_equal(out[b1], v)


# ----------------------------------------------------------------------- shapes and edge cases
SHAPES = [
    # (Hq, Hkv, D, dtype, bs, lens)
    (4, 4, 64, "f16", 16, [0, 1, 15, 16, 17, 63, 64, 65, 200]),
    (32, 8, 128, "bf16", 16, [1, 31, 32, 33, 129, 511, 512, 513, 700]),
    (16, 8, 128, "f16", 8, [2, 9, 100, 257, 640]),
    (64, 8, 128, "bf16", 32, [5, 96, 300, 1000]),
    (8, 1, 64, "bf16", 64, [1, 64, 65, 130, 900]),
    (16, 4, 64, "f16", 256, [3, 255, 256, 257, 800]),
    (8, 8, 128, "bf16", 1, [1, 2, 33, 70]),
    (12, 3, 128, "f16", 4, [4, 5, 47, 130]),
    (4, 2, 64, "bf16", 2048, [1, 1000, 2048]),
]


@pytest.mark.parametrize("mode", ["pt0", "pt64", "pt192", "fused", "fused_pt64"])
@pytest.mark.parametrize("shape", range(len(SHAPES)))
def test_shapes(shape, mode):
    hq, hkv, d, dt, bs, lens = SHAPES[shape]
    width = max(1, -(-max(lens) // bs))
    nb = len(lens) * width + 3
    batch = synth.small_random(100 + shape, len(lens), lens, hq, hkv, d, bs, nb, dt, width)
    pt = int(mode.split("pt")[1]) if "pt" in mode else 0
    _run_and_compare(batch, partition_tokens=pt, fused=mode.startswith("fused"))


def test_partitions_agree():
    batch = synth.small_random(7, 6, [700, 1500, 64, 1, 2049, 999], 32, 8, 128, 16, 6 * 129,
                               "bf16")
    kp, vp = oracle_pools(batch)
    ref = oracle_decode(batch, kp, vp)
    outs = {}
    for pt in (0, 64, 128, 512, 1024, 4096):
        outs[pt] = widen_out(GpuBatch(batch, partition_tokens=pt).run())
        assert_close(outs[pt], ref, batch.dtype, f"pt={pt}")
    for pt, o in outs.items():
        assert np.max(np.abs(o - outs[4096])) <= 2e-2
    _status_clean()


def test_relabelling_is_bit_identical():
    batch = synth.small_random(8, 5, [300, 17, 1, 640, 129], 32, 8, 128, 16, 5 * 40 + 9, "bf16")
    base = to_bits(GpuBatch(batch, partition_tokens=128).run())
    perm = np.random.default_rng(3).permutation(batch.num_blocks).astype(np.int32)
    tables = perm[batch.block_tables]
    again = to_bits(GpuBatch(batch, partition_tokens=128, tables=tables).run())
    assert np.array_equal(base, again)


def test_block_size_does_not_change_bits():
    lens = [1, 16, 100, 777, 4000, 2048, 513, 64]
    base = synth.small_random(9, len(lens), lens, 32, 8, 128, 16, len(lens) * 250 + 1, "bf16", 250)
    outs = []
    for bs in (8, 16, 32, 64, 256):
        width = -(-4096 // bs)
        nb = len(lens) * width
        ids = np.random.default_rng(bs).permutation(nb)[: len(lens) * width].astype(np.int32)
        b2 = synth.DecodeBatch(**{**base.__dict__, "block_size": bs, "num_blocks": nb,
                                  "max_blocks_per_seq": width,
                                  "block_tables": ids.reshape(len(lens), width)})
        outs.append(to_bits(GpuBatch(b2, partition_tokens=512).run()))
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


# ------------------------------------------------------------------------------- copy and write
def test_copy_blocks_bit_exact():
    rng = np.random.default_rng(4)
    shape = (64, 5, 16, 128)
    kb = rng.integers(0, 1 << 16, size=shape, dtype=np.uint64).astype(np.uint16)
    vb = rng.integers(0, 1 << 16, size=shape, dtype=np.uint64).astype(np.uint16)
    pairs = np.array([[3, 40], [0, 63], [7, 7], [12, 13], [50, 1]], dtype=np.int64)
    kc, vc = to_dev(kb, "f16"), to_dev(vb, "f16")
    abi.pa_copy_blocks(kc, vc, torch.from_numpy(pairs).cuda())
    oracle.copy_blocks(kb, vb, pairs)
    assert np.array_equal(to_bits(kc), kb) and np.array_equal(to_bits(vc), vb)
    _status_clean()


def test_reshape_and_cache_padding_and_canaries():
    rng = np.random.default_rng(5)
    nb, H, bs, D = 20, 8, 16, 128
    shape = (nb, H, bs, D)
    kb = rng.integers(0, 1 << 16, size=shape, dtype=np.uint64).astype(np.uint16)
    vb = rng.integers(0, 1 << 16, size=shape, dtype=np.uint64).astype(np.uint16)
    T = 37
    kn = rng.integers(0, 1 << 16, size=(T, H, D), dtype=np.uint64).astype(np.uint16)
    vn = rng.integers(0, 1 << 16, size=(T, H, D), dtype=np.uint64).astype(np.uint16)
    slots = rng.permutation(nb * bs)[:T].astype(np.int64)
    slots[[3, 10, 11]] = -1
    kc, vc = to_dev(kb, "bf16"), to_dev(vb, "bf16")
    abi.pa_reshape_and_cache(to_dev(kn, "bf16"), to_dev(vn, "bf16"), torch.from_numpy(slots).cuda(),
                             kc, vc)
    oracle.reshape_and_cache(kn, vn, slots, kb, vb)
    assert np.array_equal(to_bits(kc), kb) and np.array_equal(to_bits(vc), vb)
    _status_clean()


# ----------------------------------------------------------------------- device-side checking
def test_bad_ids_are_reported_not_accessed():
    batch = synth.small_random(6, 3, [40, 70, 9], 8, 2, 128, 16, 20, "bf16")
    g = GpuBatch(batch)
    g.run()
    _status_clean()
    bad = batch.block_tables.copy()
    bad[1, 2] = batch.num_blocks + 1000          # used by sequence 1 (70 tokens = 5 blocks)
    g.step.block_tables.copy_(torch.from_numpy(bad).cuda())
    g.run()
    assert abi.pa_device_status() & abi.PA_DEVERR_BLOCK_ID
    g.step.block_tables.copy_(torch.from_numpy(batch.block_tables).cuda())
    g.step.slot_mapping[0] = batch.num_blocks * batch.block_size + 5
    g.run()
    assert abi.pa_device_status() & abi.PA_DEVERR_SLOT
    g.step.slot_mapping[0] = -1
    g.step.context_lens[2] = 10_000              # beyond the table and max_context_len
    g.run()
    assert abi.pa_device_status() & abi.PA_DEVERR_CONTEXT_LEN
    pairs = torch.tensor([[0, batch.num_blocks + 3]], dtype=torch.int64, device="cuda")
    abi.pa_copy_blocks(g.k_cache, g.v_cache, pairs)
    assert abi.pa_device_status() & abi.PA_DEVERR_COPY_PAIR
    # the context is still usable
    g.step.context_lens.copy_(torch.from_numpy(batch.context_lens).cuda())
    g2 = GpuBatch(batch)
    out = widen_out(g2.run())
    kp, vp = oracle_pools(batch)
    assert_close(out, oracle_decode(batch, kp, vp), batch.dtype)
    _status_clean()


# ------------------------------------------------------------------ the five workloads, full size
def _sampled_pool_check(g, batch):
    slots = abi.pa_slot_mapping(batch.block_tables, batch.context_lens, batch.block_size)
    pick = np.random.default_rng(0).choice(len(slots), size=min(len(slots), 20000), replace=False)
    pick = np.union1d(pick, batch.new_token_rows())
    k_rows, v_rows = g.slot_rows(slots[pick])
    assert np.array_equal(k_rows, batch.k[pick]) and np.array_equal(v_rows, batch.v[pick])


def _full_size(batch, partition_tokens=0, fused=False):
    g = GpuBatch(batch, partition_tokens=partition_tokens, fused=fused)
    out = widen_out(g.run())
    _status_clean()
    _sampled_pool_check(g, batch)
    kp, vp = oracle_pools(batch, full=False)
    ref = oracle_decode(batch, kp, vp)
    # the long-context batch's keys scaled x8 collapse some softmaxes onto one V row:
    # outputs of magnitude >= 4, where bf16 itself is spaced 2^-5 apart
    s = assert_close(out, ref, batch.dtype, batch.name, ulp_branch=batch.name == "long_skew")
    print(f"\n{batch.name}: {s}")
    return g, out, s


def test_llama8b_full():
    _full_size(synth.llama8b())


@pytest.mark.parametrize("make", [synth.llama8b, synth.long_skew], ids=["llama8b", "long_skew"])
def test_fused_write_full(make):
    batch = make()
    g, out, s = _full_size(batch, fused=True)
    assert g.step.launches() == 1  # write and decode in one kernel
    # the fused write leaves exactly the pool the separate write kernel leaves
    ref = GpuBatch(batch)
    ref.run()
    assert torch.equal(ref.k_cache.view(torch.int16), g.k_cache.view(torch.int16))
    assert torch.equal(ref.v_cache.view(torch.int16), g.v_cache.view(torch.int16))


def test_overlapped_launch_gives_the_same_bits():
    """pa_decode_append_overlapped (the kernel may start during the preceding
    kernel's tail) returns the bits of pa_decode_append, also when its launches
    follow each other back to back and inside a CUDA graph."""
    batch = synth.llama8b()
    ref = GpuBatch(batch, fused=True)
    want = ref.run().clone()
    del ref
    g = GpuBatch(batch, fused=True)
    g.step.overlapped = True
    for _ in range(3):  # each launch follows the previous one on the stream
        g.step.append()
    torch.cuda.synchronize()
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
    assert torch.equal(g.step.out.view(torch.int16), want.view(torch.int16))
    _status_clean()


def test_fused_write_reports_bad_slots():
    batch = synth.small_random(16, 3, [40, 70, 9], 8, 2, 128, 16, 20, "bf16")
    g = GpuBatch(batch, fused=True)
    g.run()
    _status_clean()
    g.step.slot_mapping[1] = batch.num_blocks * batch.block_size + 7
    g.run()
    assert abi.pa_device_status() & abi.PA_DEVERR_SLOT


def test_long_skew_full():
    g, out, s = _full_size(synth.long_skew())
    assert g.step.workspace is not None  # sequences are split between CTAs and merged


def test_mixed_sweep_full():
    base = synth.mixed_sweep(16)
    outs = []
    for bs in (8, 16, 32, 64, 256):
        batch = base if bs == 16 else synth.mixed_sweep(bs, base=base)
        g, out, s = _full_size(batch)
        outs.append(to_bits(g.step.out))
        del g
        torch.cuda.empty_cache()
    for o in outs[1:]:
        assert np.array_equal(o, outs[0]), "block size changed the output bits"


@pytest.mark.parametrize("fused", [False, True])
def test_shared_prompt_copy_on_write(fused):
    script = synth.shared_prompt()
    mgr, step, tables, lens, pairs = shared_prompt_gpu(script, fused=fused)
    assert len(pairs) == script.num_prompts  # one copy-on-write per prompt
    out = widen_out(step.run())
    torch.cuda.synchronize()
    _status_clean()
    model, kp, vp, mtables, mlens, mpairs, ref = shared_prompt_oracle(script)
    assert np.array_equal(lens, mlens) and len(mpairs) == len(pairs)
    assert_close(out, ref, script.dtype, "shared_prompt")
    # every sequence's logical K/V, read through each side's own tables, is identical
    bs = script.block_size
    for r in range(len(lens)):
        n = int(lens[r])
        t = np.arange(n)
        gblk = torch.from_numpy(tables[r][t // bs]).cuda()
        goff = torch.from_numpy(t % bs).cuda()
        gk = to_bits(step.k_cache[gblk, :, goff, :])
        gv = to_bits(step.v_cache[gblk, :, goff, :])
        assert np.array_equal(gk, kp[mtables[r][t // bs], :, t % bs, :])
        assert np.array_equal(gv, vp[mtables[r][t // bs], :, t % bs, :])
    # reference counts agree up to relabelling: four sharers of every prompt block
    for i in range(script.num_prompts):
        for blk in mtables[4 * i][:script.prompt_len // bs - 1]:
            assert model.ref[blk] == 4
        for blk in tables[4 * i][:script.prompt_len // bs - 1]:
            assert mgr.ref_count(int(blk)) == 4
