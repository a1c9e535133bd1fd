"""The C-ABI library on the CPU: exports, host block manager, slot helper and
host-side argument checks. No device work is launched here."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import pins
from conftest import ROOT, read_golden
from oracle.allocator_model import BlockManagerModel, OutOfBlocks as ModelOOM

from paged_kv_cache_370_b200 import abi
from paged_kv_cache_370_b200.abi import BlockManager, OutOfBlocks, PAError


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert len(names) >= 19
    missing = [n for n in names if not hasattr(abi.lib(), n)]
    assert not missing, f"declared in include/ but not exported: {missing}"


def test_status_strings():
    assert abi.status_string(0) == "PA_OK"
    assert abi.status_string(-2) == "PA_ERR_OUT_OF_BLOCKS"


# ------------------------------------------------------------------------- block manager pins
def test_worked_example_bs4():
    g = read_golden("worked_example_bs4.txt")
    bs = int(g["block_size"][0][0])
    n = int(g["num_tokens"][0][0])
    m = BlockManager(32, bs)
    m.add_seq(7, n)
    table = m.block_table(7)
    assert len(table) == int(g["blocks_needed"][0][0])
    nth, lb = (int(x) for x in g["nth_token_in_logical_block"][0])
    # the 11th and 12th tokens still land in logical block 2
    for pos in range(n, 12):
        slot, src, dst = m.append_slot(7)
        assert slot // bs == table[lb] and slot % bs == pos - lb * bs and src == dst == -1
    assert m.seq_len(7) == int(g["nth_token_needs_new_block"][0][0]) - 1
    m.append_slot(7)
    assert len(m.block_table(7)) == 4
    free_before = m.num_free()
    m.free_seq(7)
    assert m.num_free() - free_before in [int(x) for x in g["blocks_returned"][0]]
    assert m.num_free() == 32


def test_slots_follow_the_pages_tables():
    """Slots of the pages' printed tables through pa_slot_mapping: each position's
    slot decomposes into the printed physical block and its offset."""
    g4 = read_golden("worked_example_bs4.txt")
    g16 = read_golden("block_tables_bs16.txt")
    cases = [(int(g4["block_size"][0][0]), [int(x) for x in g4["physical"][0]], g4, 12)]
    for key in ("table_A", "table_section5"):
        cases.append((16, [int(x) for x in g16[key][0]], g16, 48))
    for bs, phys, g, npos in cases:
        ranges = [(int(v[0]), int(v[2]), int(v[3])) for v in g["logical_block"]]
        slots = abi.pa_slot_mapping(np.array([phys], np.int32), [npos], bs)
        for lb, lo, hi in ranges:
            for t in range(lo, hi + 1):
                assert slots[t] // bs == phys[lb] and slots[t] % bs == t - lo


def test_slot_mapping_matches_oracle():
    batch = pins.small_batches()[0]
    counts = batch.context_lens
    got = abi.pa_slot_mapping(batch.block_tables, counts, batch.block_size)
    want = np.concatenate([oracle.slots_for(batch.block_tables[b], range(int(counts[b])),
                                            batch.block_size) for b in range(batch.num_seqs)])
    assert np.array_equal(got, want)
    with pytest.raises(PAError):
        abi.pa_slot_mapping(batch.block_tables, counts + 10_000, batch.block_size)


def test_capacity_figures():
    g = read_golden("capacity_figures.txt")
    val = lambda k: int(g[k][0][0])  # noqa: E731
    m = BlockManager(4096, 16)
    m.add_seq(1, val("request_tokens"))
    assert len(m.block_table(1)) == val("request_blocks")
    free, used, wasted = m.stats()
    assert used == val("request_tokens") and 16 - wasted == val("request_last_block_fill")
    worst = 0
    for n in range(1, 400):
        mm = BlockManager(64, 16)
        mm.add_seq(0, n)
        worst = max(worst, mm.stats()[2])
    assert worst == val("max_waste_tokens_bs16")


def test_copy_on_write_reference_trace():
    m = BlockManager(16, 4)
    m.add_seq(0, 6)
    for c in (1, 2, 3):
        m.fork(0, c)
    shared = m.block_table(0)
    assert [m.ref_count(b) for b in shared] == [4, 4]
    slot, src, dst = m.append_slot(1)
    assert src == shared[1] and dst not in shared and slot == dst * 4 + 2
    assert m.ref_count(src) == 3 and m.ref_count(dst) == 1 and m.block_table(1)[1] == dst
    for c in (2, 3):
        assert m.append_slot(c)[1] == shared[1]
    slot0, s0, _ = m.append_slot(0)
    assert s0 == -1 and slot0 == shared[1] * 4 + 2
    for c in range(4):
        m.free_seq(c)
    assert m.num_free() == 16


def test_out_of_blocks_is_all_or_nothing():
    m = BlockManager(4, 16)
    m.add_seq(0, 40)  # 3 blocks
    with pytest.raises(OutOfBlocks):
        m.add_seq(1, 33)  # needs 3, 1 free
    assert m.num_free() == 1
    m.add_seq(1, 16)  # the last free block
    m.fork(0, 2)      # seq 2 shares seq 0's three blocks
    before, n_before = m.block_table(0), m.seq_len(0)
    with pytest.raises(OutOfBlocks):
        m.append_slot(0)  # writes into the shared, part-filled block 2: a copy needs a block
    assert m.block_table(0) == before and m.seq_len(0) == n_before
    assert m.ref_count(before[2]) == 2


def test_state_errors():
    m = BlockManager(8, 16)
    m.add_seq(0, 5)
    with pytest.raises(PAError):
        m.add_seq(0, 5)
    with pytest.raises(PAError):
        m.fork(5, 6)
    m.free_seq(0)
    with pytest.raises(PAError):
        m.free_seq(0)
    with pytest.raises(PAError):
        m.append_slot(0)


def _relabel_consistent(model, prod, seqs, host=False):
    """True if one bijection of block ids maps every model table onto the product's
    (device ids, or with ``host`` the host swap-space ids of swapped sequences)."""
    fwd, bwd = {}, {}
    mref = model.host_ref if host else model.ref
    for s in seqs:
        a, b = model.block_table(s), prod.block_table(s)
        if len(a) != len(b):
            return False
        for x, y in zip(a, b):
            if x == -1 or y == -1:  # released by a sliding window: on both sides
                if x != y:
                    return False
                continue
            if fwd.setdefault(x, y) != y or bwd.setdefault(y, x) != x:
                return False
            if not host and mref[x] != prod.ref_count(y):
                return False
    return True


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_random_trace_matches_model_up_to_relabelling(seed):
    rng = np.random.default_rng(seed)
    bs, nb, nh = 8, 96, 40
    model, prod = BlockManagerModel(nb, bs), BlockManager(nb, bs)
    model.set_host_blocks(nh)
    prod.set_host_blocks(nh)
    live, next_id = [], 0
    ops = ["add", "fork", "append", "append", "append", "free", "window", "swap_out", "swap_in",
           "cached", "cached"]
    # prompts for prefix caching: a few shared stems over a small vocabulary
    stems = [[int(t) for t in rng.integers(0, 3, size=48)] for _ in range(3)]
    for step in range(2000):
        op = rng.choice(ops)
        resident = [s for s in live if s not in model.swapped]
        swapped = [s for s in live if s in model.swapped]
        if step % 500 == 499:
            model.reset_prefix_cache()
            prod.reset_prefix_cache()
        if op == "cached":
            stem = stems[int(rng.integers(0, len(stems)))]
            toks = stem[:int(rng.integers(0, 49))] + \
                [int(t) for t in rng.integers(0, 3, size=int(rng.integers(0, 12)))]
            try:
                got = model.add_seq_cached(next_id, toks)
                ok = True
            except ModelOOM:
                ok = False
            if ok:
                assert prod.add_seq_cached(next_id, toks) == got
                live.append(next_id)
            else:
                with pytest.raises(OutOfBlocks):
                    prod.add_seq_cached(next_id, toks)
            next_id += 1
        elif op == "add" or not resident:
            n = int(rng.integers(0, 40))
            try:
                model.add_seq(next_id, n)
                ok = True
            except ModelOOM:
                ok = False
            if ok:
                prod.add_seq(next_id, n)
                live.append(next_id)
            else:
                with pytest.raises(OutOfBlocks):
                    prod.add_seq(next_id, n)
            next_id += 1
        elif op == "fork":
            p = int(rng.choice(resident))
            model.fork(p, next_id)
            prod.fork(p, next_id)
            live.append(next_id)
            next_id += 1
        elif op == "append":
            s = int(rng.choice(resident))
            try:
                ms, msrc, mdst = model.append_slot(s)
                ok = True
            except ModelOOM:
                ok = False
            if ok:
                ps, psrc, pdst = prod.append_slot(s)
                assert (msrc == -1) == (psrc == -1)
                assert ms % bs == ps % bs
            else:
                with pytest.raises(OutOfBlocks):
                    prod.append_slot(s)
        elif op == "window":
            s = int(rng.choice(resident))
            w = int(rng.integers(1, 30))
            assert model.slide_window(s, w) == prod.slide_window(s, w)
        elif op in ("swap_out", "swap_in"):
            pool = resident if op == "swap_out" else swapped
            if not pool:
                continue
            k = int(rng.integers(1, min(3, len(pool)) + 1))
            group = [int(x) for x in rng.choice(pool, size=k, replace=False)]
            try:
                mp = getattr(model, op)(group)
                ok = True
            except ModelOOM:
                ok = False
            if ok:
                pp = getattr(prod, op)(group)
                assert len(mp) == len(pp)
                for g in group:
                    assert prod.is_swapped(g) == (op == "swap_out")
            else:
                with pytest.raises(OutOfBlocks):
                    getattr(prod, op)(group)
        else:
            s = int(rng.choice(live))
            model.free_seq(s)
            prod.free_seq(s)
            live.remove(s)
        assert model.num_free() == prod.num_free()
        assert len(model.host_free) == prod.host_free()
        assert _relabel_consistent(model, prod, [s for s in live if s not in model.swapped])
        assert _relabel_consistent(model, prod, [s for s in live if s in model.swapped], host=True)
        assert model.stats() == prod.stats()
        assert model.cached_blocks() == prod.cached_blocks()


def test_prefix_cache_worked_example():
    """The hand-worked prefix-caching example on the product (block size 4, 8
    blocks, system prompt 1..10): shared blocks, the recomputed last block,
    release order and reuse of cached blocks, all-or-nothing."""
    m = BlockManager(8, 4)
    S = list(range(1, 11))
    assert m.add_seq_cached(0, S + [11, 12]) == 0
    a = m.block_table(0)
    assert m.add_seq_cached(1, S + [21]) == 8 and m.block_table(1)[:2] == a[:2]
    assert m.add_seq_cached(2, S + [11, 12, 13]) == 12 and m.block_table(2)[:3] == a
    assert m.add_seq_cached(3, S + [11, 12]) == 8 and m.block_table(3)[2] not in a
    assert [m.ref_count(b) for b in a] == [4, 4, 2] and m.cached_blocks() == (3, 0)
    for seq in range(4):
        m.free_seq(seq)
    assert m.num_free() == 8 and m.cached_blocks() == (3, 3)
    assert m.add_seq_cached(4, S + [11, 12]) == 8
    m.free_seq(4)
    m.add_seq(5, 24)
    assert a[2] in m.block_table(5) and m.cached_blocks() == (2, 2)
    m.add_seq(6, 4)
    assert m.block_table(6) == [a[1]]
    with pytest.raises(OutOfBlocks):
        m.add_seq_cached(7, S + [31])
    assert m.cached_blocks() == (1, 1) and m.num_free() == 1
    m.free_seq(5)
    assert m.add_seq_cached(7, S + [31]) == 4
    assert m.add_seq_cached(8, S + [11, 12, 13]) == 8
    assert m.cached_blocks() == (3, 0) and m.num_free() == 2
    for seq in (6, 7, 8):
        m.free_seq(seq)
    assert m.cached_blocks() == (3, 3)
    m.reset_prefix_cache()
    assert m.cached_blocks() == (0, 0) and m.num_free() == 8
    assert m.add_seq_cached(9, S + [11]) == 0


def test_prefix_cache_arguments():
    m = BlockManager(8, 4)
    assert m.add_seq_cached(0, []) == 0 and m.block_table(0) == []
    with pytest.raises(PAError):
        m.add_seq_cached(0, [1, 2, 3])           # the sequence exists
    assert m.add_seq_cached(1, [5]) == 0 and m.add_seq_cached(2, [5]) == 0


def test_swap_group_shares_blocks_once():
    m = BlockManager(16, 4)
    m.set_host_blocks(8)
    m.add_seq(0, 6)                  # 2 blocks
    m.fork(0, 1)                     # both shared (ref 2)
    m.add_seq(2, 3)                  # 1 private block
    t0 = m.block_table(0)
    free0 = m.num_free()
    pairs = m.swap_out([0, 1])       # the shared blocks move once
    assert sorted(pairs[:, 0].tolist()) == sorted(t0)
    assert m.num_free() == free0 + 2 and m.host_free() == 6
    assert m.block_table(0) == m.block_table(1) == pairs[:, 1].tolist()
    with pytest.raises(PAError):
        m.append_slot(0)             # swapped: no slots
    with pytest.raises(PAError):
        m.swap_out([0])              # already out
    back = m.swap_in([1, 0])
    assert back[:, 0].tolist() == pairs[:, 1].tolist()
    assert m.block_table(0) == m.block_table(1) == back[:, 1].tolist()
    assert [m.ref_count(b) for b in m.block_table(0)] == [2, 2] and m.host_free() == 8
    # a block also held outside the group is copied and stays for the other sequence
    m.fork(2, 3)
    p2 = m.swap_out([3])
    assert p2.shape == (1, 2) and m.ref_count(m.block_table(2)[0]) == 1
    m.free_seq(3)                    # a swapped sequence frees its host blocks
    assert m.host_free() == 8
    with pytest.raises(PAError):
        m.swap_in([2])               # not swapped


def test_fill_tables():
    m = BlockManager(64, 16)
    m.add_seq(3, 40)
    m.add_seq(9, 1)
    tables, lens = m.fill_tables([9, 3], 5, pad=-7)
    assert lens.tolist() == [1, 40]
    assert tables[0, 0] == m.block_table(9)[0] and (tables[0, 1:] == -7).all()
    assert tables[1, :3].tolist() == m.block_table(3) and (tables[1, 3:] == -7).all()


# ----------------------------------------------------------------- host-side argument checks
def test_decode_rejects_bad_arguments_before_launch():
    L = abi.lib()
    args = dict(out=None, q=None, k=None, v=None, bt=None, mbps=4, cl=None, maxlen=64, B=2, hq=6,
                hkv=4, d=128, bs=16, nb=8, scale=0.1, dt=abi.PA_BF16, ws=None, wsb=0, pt=0, st=None)

    def call(**kw):
        a = dict(args, **kw)
        return L.pa_decode(a["out"], a["q"], a["k"], a["v"], a["bt"], a["mbps"], a["cl"],
                           a["maxlen"], a["B"], a["hq"], a["hkv"], a["d"], a["bs"], a["nb"],
                           a["scale"], a["dt"], a["ws"], a["wsb"], a["pt"], a["st"])

    assert call() == abi.PA_ERR_INVALID            # 6 q heads over 4 kv heads
    assert call(hq=8, d=96) == abi.PA_ERR_UNSUPPORTED
    assert call(hq=8) == abi.PA_ERR_INVALID        # null pointers
    assert call(hq=8, pt=100) == abi.PA_ERR_INVALID  # not a multiple of 64
    assert call(hq=8, dt=7) == abi.PA_ERR_INVALID
    assert call(hq=8, B=0) == abi.PA_OK             # empty batch: nothing to do
    assert L.pa_reshape_and_cache(None, None, None, 0, None, None, 8, 4, 16, 128, 1, None) == 0
    assert L.pa_reshape_and_cache(None, None, None, 3, None, None, 8, 4, 16, 128, 1, None) == -1
    assert L.pa_copy_blocks(None, None, None, 0, 8, 4, 16, 128, 1, None) == 0
    assert L.pa_copy_blocks(None, None, None, 2, 8, 4, 16, 0, 1, None) == -1

    def call_window(w, **kw):
        a = dict(args, hq=8, B=0, **kw)
        return L.pa_decode_window(a["out"], a["q"], a["k"], a["v"], a["bt"], a["mbps"], a["cl"],
                                  a["maxlen"], a["B"], a["hq"], a["hkv"], a["d"], a["bs"], a["nb"],
                                  a["scale"], w, a["dt"], a["ws"], a["wsb"], a["pt"], a["st"])

    assert call_window(0) == abi.PA_ERR_INVALID     # a window holds at least one position
    assert call_window(-3) == abi.PA_ERR_INVALID
    assert call_window(5) == abi.PA_OK              # empty batch: nothing to do
    # swap: a null space or unaligned pools are refused before any launch
    assert L.pa_swap_out(None, None, None, 8, None, 0, None) == abi.PA_ERR_INVALID
    assert L.pa_swap_in(None, None, None, 8, None, 0, None) == abi.PA_ERR_INVALID
    # the read-rate probe: sizes, pointers and CTA counts are checked before any launch
    buf, sink = ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 12)
    assert L.pa_hbm_read(None, 16, sink, 4, None) == abi.PA_ERR_INVALID
    assert L.pa_hbm_read(buf, 16, None, 4, None) == abi.PA_ERR_INVALID
    assert L.pa_hbm_read(buf, 0, sink, 4, None) == abi.PA_ERR_INVALID
    assert L.pa_hbm_read(buf, 24, sink, 4, None) == abi.PA_ERR_INVALID      # not 16-byte units
    assert L.pa_hbm_read(ctypes.c_void_p((1 << 20) + 8), 16, sink, 4, None) == abi.PA_ERR_INVALID
    assert L.pa_hbm_read(buf, 16, sink, 0, None) == abi.PA_ERR_INVALID
    assert L.pa_hbm_read(buf, 16, sink, 5, None) == abi.PA_ERR_INVALID


def test_workspace_size():
    # a fixed 64 KiB counter region, then room for the larger of the two kernels' scratch
    region = 64 * 1024
    # fixed partitions (SIMT kernel): acc [D] + (max, sum) per (seq, q head, partition);
    # even split with 512 tokens per CTA: 2 pieces per CTA of G heads x (D + 4)
    simt = 4 * 8 * 3 * (128 + 2) * 4
    ctas = -(-(4 * 2 * -(-1100 // 64)) // (512 // 64))
    stream = 2 * ctas * 4 * (128 + 4) * 4
    assert abi.pa_decode_workspace_size(4, 8, 2, 128, 1100, 512) == region + max(simt, stream)
    assert abi.pa_decode_workspace_size(4, 8, 2, 128, 1100, 0) >= region
    assert abi.pa_decode_workspace_size(4, 6, 4, 128, 1100, 0) == 0  # 6 / 4 heads: invalid
    pt = abi.pa_decode_default_partition(64, 8, 2048)
    assert pt % 64 == 0 and 64 <= pt <= 8192



# ------------------------------------------------------------------------------ byte accounting
def test_kv_bytes_per_token_matches_the_pages():
    from paged_kv_cache_370_b200.accounting import kv_bytes_per_token
    g = read_golden("capacity_figures.txt")
    val = lambda k: int(g[k][0][0])  # noqa: E731
    per_tok = kv_bytes_per_token(val("llama31_8b_layers"), val("llama31_8b_kv_heads"),
                                 val("llama31_8b_head_dim"), 2)
    assert per_tok == val("llama31_8b_kv_bytes_per_token")
    assert 16 * per_tok == val("llama31_8b_block_bytes_bs16")
    assert round(50 * 2**30 / (16 * per_tok)) == val("llama31_8b_blocks_in_50GiB")
    assert abs(50 * 2**30 / per_tok - val("tokens_in_50GiB")) / val("tokens_in_50GiB") < 0.05
    opt = kv_bytes_per_token(val("opt13b_layers"), val("opt13b_hidden") // 128, 128, 2)
    approx = val("opt13b_kv_bytes_per_token_approx")
    assert abs(opt - approx) / approx < 0.05
    assert abs(opt * val("opt13b_tokens") - val("opt13b_bytes_for_2048_approx")) / 1.6e9 < 0.06


def test_decode_step_bytes():
    from paged_kv_cache_370_b200.accounting import decode_step_bytes
    b = decode_step_bytes([1, 17, 32], 32, 8, 128, 16)
    assert b["kv"] == 2 * 50 * 8 * 128 * 2
    assert b["block_tables"] == (1 + 2 + 2) * 4
    assert b["total"] == b["kv"] + 2 * 3 * 32 * 128 * 2 + 20 + 12


def test_tail_overread_bytes():
    from paged_kv_cache_370_b200.accounting import tail_overread_bytes
    # whole blocks read for lengths 1, 17, 32 at block size 16: 15 + 15 + 0 unfilled rows
    assert tail_overread_bytes([1, 17, 32], 8, 128, 16) == 2 * 30 * 8 * 128 * 2
    assert tail_overread_bytes([0, 16], 8, 128, 16) == 0


def _split_pieces_walk(lens, hkv, n, tile=64):
    """Pieces of split segments, found by walking every tile in order with CTA c
    owning tiles [floor(c W / n), floor((c + 1) W / n))."""
    tiles = [max(1, -(-int(l) // tile)) for l in lens for _ in range(hkv)]
    W = sum(tiles)
    starts = [c * W // n for c in range(n + 1)]
    c, x, pieces = 0, 0, 0
    for t in tiles:
        owners = set()
        for _ in range(t):
            while x >= starts[c + 1]:
                c += 1
            owners.add(c)
            x += 1
        pieces += len(owners) if len(owners) > 1 else 0
    return pieces


def test_split_scratch_bytes_counts_the_pieces():
    from paged_kv_cache_370_b200.accounting import stream_split_scratch_bytes
    per_piece = 2 * 4 * (128 + 2) * 4 + 8
    # one 10-tile segment over 2 CTAs: 5 tiles each, two pieces
    assert stream_split_scratch_bytes([640], 1, 4, 128, 2) == 2 * per_piece
    # two 1-tile segments over 2 CTAs: nothing is split
    assert stream_split_scratch_bytes([64, 64], 1, 4, 128, 2) == 0
    rng = np.random.default_rng(7)
    for _ in range(60):
        b = int(rng.integers(1, 40))
        lens = rng.integers(0, 3000, size=b)
        hkv, n = int(rng.choice([1, 2, 8])), int(rng.choice([1, 3, 16, 148, 296, 1000]))
        assert stream_split_scratch_bytes(lens, hkv, 4, 128, n) == \
            _split_pieces_walk(lens, hkv, n) * per_piece


def test_slide_window_releases_only_blocks_before_the_window():
    m = BlockManager(16, 4)
    m.add_seq(0, 10)                       # blocks for positions 0-3, 4-7, 8-9
    t0 = m.block_table(0)
    assert m.slide_window(0, 5) == 1       # window [5, 10): only block 0 is wholly before it
    assert m.block_table(0) == [-1] + t0[1:]
    assert m.slide_window(0, 5) == 0       # repeating it changes nothing
    with pytest.raises(PAError):
        m.seq_slots(0, 3, 2)               # position 3 was released
    assert m.seq_slots(0, 4, 6).tolist() == [t0[1] * 4 + i for i in range(4)] + [t0[2] * 4, t0[2] * 4 + 1]
    m.fork(0, 1)                            # a fork shares what is left
    assert m.block_table(1) == [-1] + t0[1:]
    assert m.slide_window(1, 2) == 0       # block 1 is still held by sequence 0
    assert m.ref_count(t0[1]) == 1
    assert m.slide_window(0, 2) == 1       # now nobody holds it
    m.free_seq(0)
    m.free_seq(1)
    assert m.stats()[0] == 16
    with pytest.raises(PAError):
        m.slide_window(7, 3)
    m.add_seq(2, 3)
    with pytest.raises(PAError):
        m.slide_window(2, 0)
