"""Paged prefill attention (several query tokens per sequence) on a B200 against
the oracle's causal prefill. The pools start poisoned (NaN), so a read of any
slot that was not written shows in the output."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_harness import TORCH_DT, oracle_pools, poisoned_pool, to_dev, widen_out
from paged_kv_cache_370_b200 import abi
from tolerance import assert_close

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU machines too; every test here needs the GPU
    pytest.skip("no CUDA device", allow_module_level=True)


class GpuPrefill:
    """A prefill batch on the device: every position's K/V written with
    pa_reshape_and_cache at its slot, then pa_prefill."""

    def __init__(self, batch, device="cuda", tables=None):
        self.batch = batch
        bs, dt = batch.block_size, batch.dtype
        shape = (batch.num_blocks, batch.num_kv_heads, bs, batch.head_dim)
        self.k_cache = poisoned_pool(shape, dt, device)
        self.v_cache = poisoned_pool(shape, dt, device)
        tables = batch.block_tables if tables is None else tables
        slots = abi.pa_slot_mapping(batch.block_tables, batch.context_lens, bs)
        if len(slots):
            abi.pa_reshape_and_cache(to_dev(batch.k, dt, device), to_dev(batch.v, dt, device),
                                     torch.from_numpy(slots).to(device), self.k_cache,
                                     self.v_cache)
        self.q = to_dev(batch.q, dt, device)
        self.out = torch.empty_like(self.q)
        self.tables = torch.from_numpy(np.ascontiguousarray(tables)).to(device)
        self.lens = torch.from_numpy(batch.context_lens).to(device)
        self.q_start = torch.from_numpy(batch.meta["q_start"].astype(np.int32)).to(device)
        self.max_q_len = int(batch.meta["q_lens"].max()) if batch.num_seqs else 0

    def run(self, window=0):
        abi.pa_prefill(self.out, self.q, self.k_cache, self.v_cache, self.tables, self.lens,
                       self.q_start, self.max_q_len, max(self.batch.max_context_len, 1),
                       float(self.batch.scale), window)
        torch.cuda.synchronize()
        return self.out


def _status_clean():
    code = abi.pa_device_status()
    assert code == 0, f"device error word {code:#x}"


def _oracle(batch, window=0):
    kp, vp = oracle_pools(batch, full=True)
    # the oracle pools hold every position (history and query tokens alike)
    oracle.place_history(batch, kp, vp, include_new=True)
    return oracle.prefill(batch.q, kp, vp, batch.block_tables, batch.context_lens,
                          batch.meta["q_start"], batch.scale, batch.dtype, window)


SHAPES = [
    # (Hq, Hkv, D, dtype, bs, lens, q_lens)
    (32, 8, 128, "bf16", 16, [64, 200, 77, 513, 1], [64, 65, 1, 300, 1]),
    (8, 8, 128, "f16", 16, [130, 33, 64], [130, 20, 63]),
    (16, 4, 64, "bf16", 32, [100, 257, 40], [37, 257, 40]),
    (8, 2, 128, "f16", 8, [17, 300, 129], [9, 128, 129]),
    (32, 4, 128, "bf16", 256, [700, 256, 90], [400, 200, 90]),
    (4, 4, 64, "f16", 64, [0, 5, 140], [0, 5, 70]),
    # three q heads per kv head: items of 256 rows of one head, not head pairs
    (6, 2, 64, "bf16", 16, [300, 45, 129], [260, 45, 129]),
    # two q heads per kv head: each item is both heads of one kv head
    (8, 4, 128, "f16", 16, [200, 129, 16], [150, 129, 16]),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"h{s[0]}-{s[1]}d{s[2]}{s[3]}bs{s[4]}")
@pytest.mark.parametrize("window", [0, 1, 17, 100])
def test_prefill_shapes(shape, window):
    hq, hkv, d, dt, bs, lens, qlens = shape
    width = -(-max(max(lens), 1) // bs) + 1
    batch = synth.prefill_random(51 + bs + window, lens, qlens, hq, hkv, d, bs,
                                 len(lens) * width + 2, dt, width=width)
    g = GpuPrefill(batch)
    out = widen_out(g.run(window))
    _status_clean()
    assert_close(out, _oracle(batch, window), dt, f"prefill {shape[:5]} window {window}",
                 ulp_branch=True)


def test_prefill_single_tokens_match_decode():
    """One query token per sequence is decode: same result as the oracle's decode."""
    lens = [1, 40, 300, 1025]
    batch = synth.prefill_random(57, lens, [1] * 4, 32, 8, 128, 16, 4 * 66, "bf16", width=66)
    g = GpuPrefill(batch)
    out = widen_out(g.run())
    kp, vp = oracle_pools(batch, full=True)
    oracle.place_history(batch, kp, vp, include_new=True)
    ref = oracle.decode(batch.q, kp, vp, batch.block_tables, batch.context_lens, batch.scale,
                        batch.dtype)
    assert_close(out, ref, "bf16", "single-token prefill")
    _status_clean()


def test_prefill_many_sequences_in_index_order():
    """More (sequence, query tile) pairs than the kernel's item order holds (16,384):
    the items go in index order instead, with the same results. (Contexts of 48 to
    176 positions: with only a few keys, the weights' rounding to bf16 before the
    P V product can put an output in [2, 4) just past 1e-2 of the exact value, as in
    the 2-key case ([0.213, 0.787] over V = 0.691, -3.297) that a 1-to-40-key batch
    of this size contains; that property of the arithmetic is not what this test is
    about.)"""
    rng = np.random.default_rng(61)
    B = 16_500
    lens = rng.integers(48, 177, size=B)
    qlens = np.minimum(lens, rng.integers(1, 4, size=B))
    batch = synth.prefill_random(61, lens, qlens, 8, 2, 64, 16, B * 12, "bf16", width=12)
    g = GpuPrefill(batch)
    full = g.run().clone()
    _status_clean()
    # the first 8,000 sequences alone fit the order (longest first): same bits
    n = 8_000
    t = int(batch.meta["q_start"][n])
    part = torch.empty_like(g.q[:t])
    abi.pa_prefill(part, g.q[:t].contiguous(), g.k_cache, g.v_cache, g.tables[:n].contiguous(),
                   g.lens[:n].contiguous(), g.q_start[:n + 1].contiguous(),
                   int(batch.meta["q_lens"][:n].max()), int(batch.context_lens[:n].max()),
                   float(batch.scale), 0)
    torch.cuda.synchronize()
    _status_clean()
    assert torch.equal(part.view(torch.int16), full[:t].view(torch.int16))
    assert_close(widen_out(full), _oracle(batch), "bf16",
                 "prefill past the item order's capacity", ulp_branch=True)


def test_prefill_relabelling_is_bit_identical():
    batch = synth.prefill_random(58, [300, 70], [300, 33], 16, 8, 128, 16, 60, "bf16", width=20)
    a = GpuPrefill(batch).run().clone()
    perm = np.random.default_rng(9).permutation(batch.num_blocks)
    relabelled = synth.prefill_random(58, [300, 70], [300, 33], 16, 8, 128, 16, 60, "bf16",
                                      width=20)
    relabelled.block_tables = perm[batch.block_tables].astype(np.int32)
    b = GpuPrefill(relabelled).run().clone()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_prefill_bad_block_is_reported():
    batch = synth.prefill_random(59, [100, 50], [100, 50], 8, 4, 64, 16, 30, "f16", width=8)
    g = GpuPrefill(batch)
    bad = batch.block_tables.copy()
    bad[0, 3] = batch.num_blocks + 11
    g.tables.copy_(torch.from_numpy(bad).cuda())
    g.run()
    assert abi.pa_device_status() & abi.PA_DEVERR_BLOCK_ID


def test_prefill_llama8b_full():
    """Chunked prefill on the Llama-3.1-8B shapes: 16 sequences, 512 new tokens after
    a history of up to 1536; 2,000 sampled (token, head) outputs against the oracle."""
    batch = synth.llama8b_prefill()
    g = GpuPrefill(batch)
    out = widen_out(g.run())
    _status_clean()
    kp, vp = oracle_pools(batch, full=False)
    oracle.place_history(batch, kp, vp, include_new=True)
    rng = np.random.default_rng(4)
    qs = batch.meta["q_start"]
    T = int(qs[-1])
    toks = rng.choice(T, size=2000, replace=False)
    heads = rng.integers(0, batch.num_q_heads, size=2000)
    G = batch.num_q_heads // batch.num_kv_heads
    got, ref = [], []
    for tok, h in zip(toks, heads):
        b = int(np.searchsorted(qs, tok, side="right") - 1)
        n, m = int(batch.context_lens[b]), int(qs[b + 1] - qs[b])
        pos = n - m + int(tok - qs[b])
        ref.append(oracle.decode_one(batch.q[tok, h], kp, vp, batch.block_tables[b], pos + 1,
                                     int(h) // G, batch.scale, batch.dtype))
        got.append(out[tok, h])
    s = assert_close(np.array(got)[None], np.array(ref)[None], batch.dtype, "llama8b prefill",
                     ulp_branch=True)
    print(f"\nllama8b prefill sample: {s}")
