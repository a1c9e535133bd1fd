"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with
a fact fixed by the pages or by mathematics:

* the pages' printed examples (``tests/golden``): block tables, the
  block-size-4 worked example, capacity figures;
* special cases that reduce to a library routine: numpy's binary16 and
  torch's bfloat16 conversions; dense, unpaged attention written with
  numpy matmul on the logical (position-ordered) rows;
* closed forms: a context of one token returns that token's V exactly;
  identical keys give the mean of V; split-context partial results merge
  to the unsplit result (log-sum-exp identity);
* brute force on tiny inputs with ``math.fsum``;
* invariances: relabelling physical blocks, poison in slots never read.

``test_oracle_pins.py`` runs every pin against the oracle;
``test_oracle_mutants.py`` compiles copies of the oracle with a planted
mistake and checks that some pin fails for each.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import synth
from conftest import read_golden
from oracle.allocator_model import BlockManagerModel, OutOfBlocks

NAN_BITS = {"f16": 0x7E00, "bf16": 0x7FC0}


# --------------------------------------------------------------------------- library decoders
def lib_f64(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Widen 16-bit patterns with library routines (numpy / torch), not the oracle."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    if dtype == "f16":
        return bits.view(np.float16).astype(np.float64)
    t = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)
    return t.to(torch.float64).numpy()


def _same(a, b):
    return np.array_equal(np.isnan(a), np.isnan(b)) and np.array_equal(a[~np.isnan(a)],
                                                                       b[~np.isnan(b)])


def pin_f16_decoder():
    allbits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    assert _same(oracle.widen(allbits, "f16"), lib_f64(allbits, "f16")), "binary16 decode"


def pin_bf16_decoder():
    allbits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    assert _same(oracle.widen(allbits, "bf16"), lib_f64(allbits, "bf16")), "bfloat16 decode"


# --------------------------------------------------------------------------- slots (pages)
def _check_table_fixture(bs, ranges, physical, n_positions):
    row = np.array(physical, dtype=np.int32)
    for (lb, lo, hi) in ranges:
        for t in range(lo, min(hi, n_positions - 1) + 1):
            s = oracle.slot(row, t, bs)
            assert s // bs == physical[lb], f"token {t}: block {s // bs} != {physical[lb]}"
            assert s % bs == t - lo, f"token {t}: offset {s % bs} != {t - lo}"


def pin_worked_example_slots():
    g = read_golden("worked_example_bs4.txt")
    bs = int(g["block_size"][0][0])
    physical = [int(x) for x in g["physical"][0]]
    ranges = [(int(v[0]), int(v[2]), int(v[3])) for v in g["logical_block"]]
    _check_table_fixture(bs, ranges, physical, n_positions=12)
    # the 11th token (index 10) still lands in logical block 2
    nth, lb = (int(x) for x in g["nth_token_in_logical_block"][0])
    assert oracle.slot(np.array(physical, np.int32), nth - 1, bs) // bs == physical[lb]


def pin_bs16_tables():
    g = read_golden("block_tables_bs16.txt")
    bs = int(g["block_size"][0][0])
    ranges = [(int(v[0]), int(v[2]), int(v[3])) for v in g["logical_block"]]
    for key in ("table_A", "table_section5"):
        physical = [int(x) for x in g[key][0]]
        _check_table_fixture(bs, ranges, physical, n_positions=48)


# --------------------------------------------------------------------------- placement
def place_numpy(batch, include_new=True, poison=True):
    """Independent placement of a batch's logical rows into fresh pools by numpy
    indexing: position t of sequence b goes to block table[b][t // bs], offset
    t % bs. Unwritten entries hold NaN patterns when ``poison`` is set."""
    shape = (batch.num_blocks, batch.num_kv_heads, batch.block_size, batch.head_dim)
    fill = NAN_BITS[batch.dtype] if poison else 0
    kp = np.full(shape, fill, dtype=np.uint16)
    vp = np.full(shape, fill, dtype=np.uint16)
    bs = batch.block_size
    for b in range(batch.num_seqs):
        n = int(batch.context_lens[b]) - (0 if include_new else 1)
        if n <= 0:
            continue
        t = np.arange(n)
        blocks = batch.block_tables[b][t // bs]
        rows = batch.rows(b)
        kp[blocks, :, t % bs, :] = batch.k[rows][:n]
        vp[blocks, :, t % bs, :] = batch.v[rows][:n]
    return kp, vp


def dense_reference(batch):
    """Unpaged attention on the logical rows with numpy fp64 matmuls; query head h
    uses KV head h // (Hq / Hkv) (np.repeat = contiguous groups)."""
    G = batch.num_q_heads // batch.num_kv_heads
    out = np.zeros((batch.num_seqs, batch.num_q_heads, batch.head_dim))
    q = lib_f64(batch.q, batch.dtype)
    for b in range(batch.num_seqs):
        n = int(batch.context_lens[b])
        if n == 0:
            continue
        K = np.repeat(lib_f64(batch.k[batch.rows(b)], batch.dtype), G, axis=1)
        V = np.repeat(lib_f64(batch.v[batch.rows(b)], batch.dtype), G, axis=1)
        for h in range(batch.num_q_heads):
            s = (K[:, h, :] @ q[b, h]) * float(batch.scale)
            w = np.exp(s - s.max())
            out[b, h] = (w @ V[:, h, :]) / w.sum()
    return out


def oracle_out(batch, kp=None, vp=None):
    if kp is None:
        kp, vp = place_numpy(batch)
    return oracle.decode(batch.q, kp, vp, batch.block_tables, batch.context_lens, batch.scale,
                         batch.dtype)


def small_batches():
    """Small paged batches over the shapes that matter: GQA and MHA, both
    dtypes, block sizes 4..32, lengths 1, block-aligned and ragged."""
    return [
        synth.small_random(11, 5, [1, 4, 5, 17, 40], 4, 2, 16, 4, 80, "f16"),
        synth.small_random(12, 4, [3, 16, 31, 33], 8, 2, 32, 16, 16, "bf16"),
        synth.small_random(13, 3, [64, 9, 1], 6, 6, 8, 32, 12, "f16"),
        synth.small_random(14, 2, [100, 7], 4, 1, 24, 8, 40, "bf16"),
        synth.tiny(),
    ]


def pin_dense(batches=None, tol=1e-12):
    for batch in batches or small_batches():
        got = oracle_out(batch)
        ref = dense_reference(batch)
        err = np.max(np.abs(got - ref)) if got.size else 0.0
        assert err <= tol, f"{batch.name}: paged oracle vs dense numpy differ by {err}"


def pin_len1_returns_v():
    batch = synth.small_random(21, 6, [1] * 6, 8, 4, 16, 4, 64, "bf16")
    got = oracle_out(batch)
    G = batch.num_q_heads // batch.num_kv_heads
    for b in range(batch.num_seqs):
        v = lib_f64(batch.v[batch.seq_start[b]], batch.dtype)  # [Hkv, D]
        for h in range(batch.num_q_heads):
            assert np.array_equal(got[b, h], v[h // G]), "length-1 context must return V"


def pin_identical_keys_mean_v():
    batch = synth.small_random(22, 3, [5, 19, 37], 4, 4, 16, 8, 20, "f16")
    for b in range(batch.num_seqs):
        r = batch.rows(b)
        batch.k[r] = batch.k[r][0:1]  # every key row of the sequence equal to its first
    got = oracle_out(batch)
    for b in range(batch.num_seqs):
        V = lib_f64(batch.v[batch.rows(b)], batch.dtype)  # [n, H, D]
        for h in range(batch.num_q_heads):
            for d in range(batch.head_dim):
                mean = math.fsum(V[:, h, d]) / V.shape[0]
                assert abs(got[b, h, d] - mean) <= 1e-14, "identical keys must average V"


def pin_bruteforce_fsum():
    batch = synth.small_random(23, 3, [2, 6, 11], 4, 2, 8, 4, 12, "bf16")
    got = oracle_out(batch)
    G = batch.num_q_heads // batch.num_kv_heads
    q = lib_f64(batch.q, batch.dtype).tolist()
    for b in range(batch.num_seqs):
        K = lib_f64(batch.k[batch.rows(b)], batch.dtype).tolist()
        V = lib_f64(batch.v[batch.rows(b)], batch.dtype).tolist()
        n = len(K)
        for h in range(batch.num_q_heads):
            g = h // G
            s = [float(batch.scale) * math.fsum(q[b][h][d] * K[t][g][d]
                                                for d in range(batch.head_dim)) for t in range(n)]
            m = max(s)
            w = [math.exp(x - m) for x in s]
            den = math.fsum(w)
            for d in range(batch.head_dim):
                ref = math.fsum(w[t] * V[t][g][d] for t in range(n)) / den
                assert abs(got[b, h, d] - ref) <= 1e-13, "brute force disagrees"


def pin_decode_one_bruteforce():
    """The single-(sequence, q head) entry point used to check sampled outputs of
    large batches, against the same pure-Python brute force: every head of every
    sequence, each through its own table row, length and kv head."""
    batch = synth.small_random(24, 3, [3, 9, 14], 4, 2, 8, 4, 12, "f16")
    kp, vp = place_numpy(batch)
    G = batch.num_q_heads // batch.num_kv_heads
    q = lib_f64(batch.q, batch.dtype).tolist()
    for b in range(batch.num_seqs):
        K = lib_f64(batch.k[batch.rows(b)], batch.dtype).tolist()
        V = lib_f64(batch.v[batch.rows(b)], batch.dtype).tolist()
        n = len(K)
        for h in range(batch.num_q_heads):
            g = h // G
            got = oracle.decode_one(batch.q[b, h], kp, vp, batch.block_tables[b],
                                    int(batch.context_lens[b]), g, batch.scale, batch.dtype)
            s = [float(batch.scale) * math.fsum(q[b][h][d] * K[t][g][d]
                                                for d in range(batch.head_dim)) for t in range(n)]
            m = max(s)
            w = [math.exp(x - m) for x in s]
            den = math.fsum(w)
            for d in range(batch.head_dim):
                ref = math.fsum(w[t] * V[t][g][d] for t in range(n)) / den
                assert abs(got[d] - ref) <= 1e-13, "decode_one disagrees with brute force"


def pin_relabel():
    batch = synth.small_random(24, 4, [13, 30, 2, 47], 4, 2, 16, 8, 40, "f16")
    kp, vp = place_numpy(batch)
    base = oracle_out(batch, kp, vp)
    perm = np.random.default_rng(5).permutation(batch.num_blocks)
    kp2, vp2 = np.empty_like(kp), np.empty_like(vp)
    kp2[perm] = kp
    vp2[perm] = vp
    tables = perm[batch.block_tables].astype(np.int32)
    got = oracle.decode(batch.q, kp2, vp2, tables, batch.context_lens, batch.scale, batch.dtype)
    assert np.array_equal(got, base), "relabelling physical blocks changed the output"


def pin_poison():
    batch = synth.small_random(25, 4, [3, 17, 16, 9], 8, 2, 16, 8, 24, "bf16")
    clean = oracle_out(batch, *place_numpy(batch, poison=False))
    dirty = oracle_out(batch, *place_numpy(batch, poison=True))
    assert np.all(np.isfinite(dirty)), "poison in unread slots reached the output"
    assert np.array_equal(clean, dirty), "unread slots changed the output"


def pin_partition_merge():
    for batch in small_batches()[:4]:
        kp, vp = place_numpy(batch)
        full = oracle_out(batch, kp, vp)
        ref_scores = _dense_scores(batch)
        for pt in (1, 3, 16, 64, 512):
            out, pm, pl, _ = oracle.decode_partitioned(batch.q, kp, vp, batch.block_tables,
                                                       batch.context_lens, batch.scale,
                                                       batch.dtype, pt, return_partials=True)
            err = np.max(np.abs(out - full))
            assert err <= 1e-12, f"partition {pt}: merged result off by {err}"
            for b in range(batch.num_seqs):
                n = int(batch.context_lens[b])
                for h in range(batch.num_q_heads):
                    for p in range(-(-n // pt)):
                        s = ref_scores[b][h][p * pt:(p + 1) * pt]
                        assert abs(pm[b, h, p] - s.max()) <= 1e-12, "partition max"
                        assert abs(pl[b, h, p] - np.exp(s - s.max()).sum()) <= 1e-11, "partition sum"


def _dense_scores(batch):
    G = batch.num_q_heads // batch.num_kv_heads
    q = lib_f64(batch.q, batch.dtype)
    res = []
    for b in range(batch.num_seqs):
        K = lib_f64(batch.k[batch.rows(b)], batch.dtype)
        res.append([(K[:, h // G, :] @ q[b, h]) * float(batch.scale)
                    for h in range(batch.num_q_heads)])
    return res


# --------------------------------------------------------------------------- sliding window
WINDOWS = (1, 2, 3, 4, 15, 16, 17, 33, 1000)


def _window_lo(n, window):
    return n - window if 0 < window < n else 0


def dense_window_reference(batch, window):
    """Unpaged attention over the logical rows [n - window, n) of each sequence,
    numpy fp64 (the window's definition applied to the dense arrays)."""
    G = batch.num_q_heads // batch.num_kv_heads
    out = np.zeros((batch.num_seqs, batch.num_q_heads, batch.head_dim))
    q = lib_f64(batch.q, batch.dtype)
    for b in range(batch.num_seqs):
        n = int(batch.context_lens[b])
        if n == 0:
            continue
        rows = np.arange(batch.rows(b).start, batch.rows(b).stop)[_window_lo(n, window):n]
        K = lib_f64(batch.k[rows], batch.dtype)
        V = lib_f64(batch.v[rows], batch.dtype)
        for h in range(batch.num_q_heads):
            s = (K[:, h // G, :] @ q[b, h]) * float(batch.scale)
            w = np.exp(s - s.max())
            out[b, h] = (w @ V[:, h // G, :]) / w.sum()
    return out


def forget_before_window(batch, kp, vp, window):
    """What a moved window leaves behind: pool rows before each sequence's window
    poisoned, and the table entries of blocks wholly before it set to -1."""
    bs = batch.block_size
    tables = np.array(batch.block_tables, dtype=np.int32, copy=True)
    kp, vp = kp.copy(), vp.copy()
    for b in range(batch.num_seqs):
        lo = _window_lo(int(batch.context_lens[b]), window)
        for t in range(lo):
            kp[tables[b, t // bs], :, t % bs, :] = NAN_BITS[batch.dtype]
            vp[tables[b, t // bs], :, t % bs, :] = NAN_BITS[batch.dtype]
        tables[b, :lo // bs] = -1
    return kp, vp, tables


def pin_window_dense():
    for batch in small_batches():
        kp, vp = place_numpy(batch)
        for w in WINDOWS:
            got = oracle.decode_window(batch.q, kp, vp, batch.block_tables, batch.context_lens,
                                       batch.scale, batch.dtype, w)
            ref = dense_window_reference(batch, w)
            err = np.max(np.abs(got - ref)) if got.size else 0.0
            assert err <= 1e-12, f"{batch.name} window {w}: off by {err}"


def pin_window_one_returns_last_v():
    batch = synth.small_random(26, 4, [1, 9, 16, 40], 8, 2, 16, 8, 24, "f16")
    kp, vp = place_numpy(batch)
    got = oracle.decode_window(batch.q, kp, vp, batch.block_tables, batch.context_lens,
                               batch.scale, batch.dtype, 1)
    G = batch.num_q_heads // batch.num_kv_heads
    for b in range(batch.num_seqs):
        v = lib_f64(batch.v[batch.rows(b).stop - 1], batch.dtype)
        for h in range(batch.num_q_heads):
            assert np.array_equal(got[b, h], v[h // G]), "window 1 must return the last V"


def pin_window_ignores_what_it_left():
    batch = synth.small_random(27, 5, [2, 16, 31, 47, 64], 4, 2, 16, 4, 90, "bf16")
    kp, vp = place_numpy(batch)
    for w in (3, 8, 17):
        base = oracle.decode_window(batch.q, kp, vp, batch.block_tables, batch.context_lens,
                                    batch.scale, batch.dtype, w)
        kf, vf, tf = forget_before_window(batch, kp, vp, w)
        got = oracle.decode_window(batch.q, kf, vf, tf, batch.context_lens, batch.scale,
                                   batch.dtype, w)
        assert np.all(np.isfinite(got)), "rows before the window reached the output"
        assert np.array_equal(got, base), "rows or ids before the window changed the output"


def pin_window_bruteforce_fsum():
    batch = synth.small_random(28, 3, [5, 9, 14], 4, 2, 8, 4, 12, "f16")
    kp, vp = place_numpy(batch)
    window = 6
    got = oracle.decode_window(batch.q, kp, vp, batch.block_tables, batch.context_lens,
                               batch.scale, batch.dtype, window)
    G = batch.num_q_heads // batch.num_kv_heads
    q = lib_f64(batch.q, batch.dtype).tolist()
    for b in range(batch.num_seqs):
        rows = np.arange(batch.rows(b).start, batch.rows(b).stop)[-window:]
        K = lib_f64(batch.k[rows], batch.dtype).tolist()
        V = lib_f64(batch.v[rows], batch.dtype).tolist()
        for h in range(batch.num_q_heads):
            g = h // G
            s = [float(batch.scale) * math.fsum(q[b][h][d] * K[t][g][d]
                                                for d in range(batch.head_dim))
                 for t in range(len(K))]
            m = max(s)
            wts = [math.exp(x - m) for x in s]
            den = math.fsum(wts)
            for d in range(batch.head_dim):
                ref = math.fsum(wts[t] * V[t][g][d] for t in range(len(K))) / den
                assert abs(got[b, h, d] - ref) <= 1e-13, "window brute force disagrees"


# --------------------------------------------------------------------------- prefill
def prefill_batches():
    """Small prefill batches: GQA and MHA, both dtypes, chunks with and without
    history, a whole prompt, single-token chunks, ragged block tails."""
    return [
        synth.prefill_random(61, [5, 20, 33, 7], [3, 20, 16, 1], 4, 2, 16, 4, 60, "f16", width=10),
        synth.prefill_random(62, [64, 17, 40], [64, 9, 40], 8, 2, 32, 16, 30, "bf16", width=6),
        synth.prefill_random(63, [1, 12, 30], [1, 12, 5], 6, 6, 8, 8, 40, "f16", width=6),
    ]


def dense_prefill_reference(batch, window=0):
    """Causal attention of each sequence's query rows over its logical rows,
    numpy fp64: query i of sequence b sits at position n - m + i and its
    scores against later positions (or, with a window, positions before
    p + 1 - window) are masked out before the softmax."""
    G = batch.num_q_heads // batch.num_kv_heads
    qs = batch.meta["q_start"]
    q = lib_f64(batch.q, batch.dtype)
    out = np.zeros(q.shape)
    for b in range(batch.num_seqs):
        n, m = int(batch.context_lens[b]), int(qs[b + 1] - qs[b])
        if m == 0:
            continue
        K = lib_f64(batch.k[batch.rows(b)], batch.dtype)
        V = lib_f64(batch.v[batch.rows(b)], batch.dtype)
        pos = n - m + np.arange(m)
        keys = np.arange(n)
        mask = keys[None, :] > pos[:, None]
        if window > 0:
            mask |= keys[None, :] < (pos[:, None] + 1 - window)
        for h in range(batch.num_q_heads):
            S = (q[qs[b]:qs[b + 1], h, :] @ K[:, h // G, :].T) * float(batch.scale)
            S[mask] = -np.inf
            W = np.exp(S - S.max(axis=1, keepdims=True))
            out[qs[b]:qs[b + 1], h, :] = (W @ V[:, h // G, :]) / W.sum(axis=1, keepdims=True)
    return out


def _oracle_prefill(batch, kp=None, vp=None, window=0, tables=None):
    if kp is None:
        kp, vp = place_numpy(batch)
    return oracle.prefill(batch.q, kp, vp, batch.block_tables if tables is None else tables,
                          batch.context_lens, batch.meta["q_start"], batch.scale, batch.dtype,
                          window)


def pin_prefill_dense():
    for batch in prefill_batches():
        kp, vp = place_numpy(batch)
        for w in (0, 1, 3, 17):
            got = _oracle_prefill(batch, kp, vp, w)
            err = np.max(np.abs(got - dense_prefill_reference(batch, w)))
            assert err <= 1e-12, f"{batch.name} window {w}: prefill off by {err}"


def pin_prefill_first_token_of_a_prompt():
    """A whole prompt as the chunk: its first token sees only itself, so its
    output is its own V row exactly."""
    batch = synth.prefill_random(64, [9, 30], [9, 30], 8, 4, 16, 4, 30, "bf16", width=9)
    got = _oracle_prefill(batch)
    G = batch.num_q_heads // batch.num_kv_heads
    qs = batch.meta["q_start"]
    for b in range(batch.num_seqs):
        v0 = lib_f64(batch.v[batch.rows(b).start], batch.dtype)
        for h in range(batch.num_q_heads):
            assert np.array_equal(got[qs[b], h], v0[h // G]), "first prompt token must return its V"


def pin_prefill_bruteforce_fsum():
    batch = synth.prefill_random(65, [6, 4], [4, 2], 4, 2, 8, 4, 12, "f16", width=3)
    got = _oracle_prefill(batch)
    G = batch.num_q_heads // batch.num_kv_heads
    qs = batch.meta["q_start"]
    q = lib_f64(batch.q, batch.dtype).tolist()
    for b in range(batch.num_seqs):
        K = lib_f64(batch.k[batch.rows(b)], batch.dtype).tolist()
        V = lib_f64(batch.v[batch.rows(b)], batch.dtype).tolist()
        n, m = len(K), int(qs[b + 1] - qs[b])
        for i in range(m):
            p = n - m + i
            for h in range(batch.num_q_heads):
                g = h // G
                s = [float(batch.scale) * math.fsum(q[qs[b] + i][h][d] * K[t][g][d]
                                                    for d in range(batch.head_dim))
                     for t in range(p + 1)]
                mx = max(s)
                w = [math.exp(x - mx) for x in s]
                den = math.fsum(w)
                for d in range(batch.head_dim):
                    ref = math.fsum(w[t] * V[t][g][d] for t in range(p + 1)) / den
                    assert abs(got[qs[b] + i, h, d] - ref) <= 1e-13, "prefill brute force"


def pin_prefill_relabel():
    batch = prefill_batches()[1]
    kp, vp = place_numpy(batch)
    base = _oracle_prefill(batch, kp, vp)
    perm = np.random.default_rng(6).permutation(batch.num_blocks)
    kp2, vp2 = np.empty_like(kp), np.empty_like(vp)
    kp2[perm] = kp
    vp2[perm] = vp
    got = _oracle_prefill(batch, kp2, vp2, tables=perm[batch.block_tables].astype(np.int32))
    assert np.array_equal(got, base), "relabelling physical blocks changed the prefill output"


# --------------------------------------------------------------------------- write / copy
def pin_reshape_layout():
    """Write the worked example's 10 tokens (block size 4, blocks 8, 3, 15) at the
    oracle's slots; each row must sit at pool[physical, head, offset, :]."""
    g = read_golden("worked_example_bs4.txt")
    bs = int(g["block_size"][0][0])
    physical = [int(x) for x in g["physical"][0]]
    ranges = [(int(v[0]), int(v[2]), int(v[3])) for v in g["logical_block"]]
    n, H, D = int(g["num_tokens"][0][0]), 2, 4
    rng = np.random.default_rng(0)
    k_new = rng.integers(0, 1 << 16, size=(n + 1, H, D), dtype=np.uint64).astype(np.uint16)
    v_new = rng.integers(0, 1 << 16, size=(n + 1, H, D), dtype=np.uint64).astype(np.uint16)
    # the example's 10 tokens, then a padding token (slot -1), then a token at slot 0
    slots = np.append(oracle.slots_for(np.array(physical, np.int32), range(n), bs), [-1, 0])
    k_new = np.concatenate([k_new, k_new[:1]])
    v_new = np.concatenate([v_new, v_new[:1]])
    kc = oracle.empty_pool(16, H, bs, D)
    vc = oracle.empty_pool(16, H, bs, D)
    oracle.reshape_and_cache(k_new, v_new, slots, kc, vc)
    written = np.zeros(kc.shape[:3], dtype=bool)
    assert np.array_equal(kc[0, :, 0, :], k_new[-1]) and np.array_equal(vc[0, :, 0, :], v_new[-1])
    written[0, :, 0] = True
    for (lb, lo, hi) in ranges:
        for t in range(lo, min(hi, n - 1) + 1):
            assert np.array_equal(kc[physical[lb], :, t - lo, :], k_new[t]), f"K token {t}"
            assert np.array_equal(vc[physical[lb], :, t - lo, :], v_new[t]), f"V token {t}"
            written[physical[lb], :, t - lo] = True
    assert not kc[~written].any() and not vc[~written].any(), "write touched other slots"


def pin_copy_blocks():
    rng = np.random.default_rng(1)
    shape = (12, 3, 8, 16)
    kc = rng.integers(0, 1 << 16, size=shape, dtype=np.uint64).astype(np.uint16)
    vc = rng.integers(0, 1 << 16, size=shape, dtype=np.uint64).astype(np.uint16)
    k0, v0 = kc.copy(), vc.copy()
    pairs = np.array([[3, 7], [0, 11], [5, 5]], dtype=np.int64)
    oracle.copy_blocks(kc, vc, pairs)
    exp_k, exp_v = k0.copy(), v0.copy()
    for s, d in pairs:
        exp_k[d] = k0[s]
        exp_v[d] = v0[s]
    assert np.array_equal(kc, exp_k) and np.array_equal(vc, exp_v), "copy_blocks"


def pin_swap_blocks():
    """Swap out then in: the host pool gets exactly the named device blocks
    (numpy indexing as the reference), untouched host blocks keep their bits,
    and bringing the blocks back into other device blocks restores every row."""
    rng = np.random.default_rng(2)
    dev_shape, host_shape = (10, 2, 4, 8), (6, 2, 4, 8)
    dk = rng.integers(0, 1 << 16, size=dev_shape, dtype=np.uint64).astype(np.uint16)
    dv = rng.integers(0, 1 << 16, size=dev_shape, dtype=np.uint64).astype(np.uint16)
    hk = rng.integers(0, 1 << 16, size=host_shape, dtype=np.uint64).astype(np.uint16)
    hv = rng.integers(0, 1 << 16, size=host_shape, dtype=np.uint64).astype(np.uint16)
    hk0, hv0 = hk.copy(), hv.copy()
    out_pairs = np.array([[7, 0], [2, 5], [9, 3]], dtype=np.int64)
    oracle.swap_blocks(hk, hv, dk, dv, out_pairs)
    exp_k, exp_v = hk0.copy(), hv0.copy()
    exp_k[out_pairs[:, 1]] = dk[out_pairs[:, 0]]
    exp_v[out_pairs[:, 1]] = dv[out_pairs[:, 0]]
    assert np.array_equal(hk, exp_k) and np.array_equal(hv, exp_v), "swap out"
    in_pairs = np.array([[0, 1], [5, 4], [3, 8]], dtype=np.int64)  # host -> other device blocks
    dk2, dv2 = dk.copy(), dv.copy()
    oracle.swap_blocks(dk2, dv2, hk, hv, in_pairs)
    for (d_src, _), (_, d_dst) in zip(out_pairs, in_pairs):
        assert np.array_equal(dk2[d_dst], dk[d_src]) and np.array_equal(dv2[d_dst], dv[d_src])
    untouched = [b for b in range(dev_shape[0]) if b not in in_pairs[:, 1]]
    assert np.array_equal(dk2[untouched], dk[untouched]), "swap in wrote outside its pairs"


# --------------------------------------------------------------------------- placement helpers
def pin_place_history():
    """The oracle's placement helper (the pools every GPU parity test compares
    against) equals the independent numpy placement bit for bit, with and
    without each sequence's last position: block sizes 4..32, lengths 0, 1,
    block-aligned and ragged, both dtypes, GQA and MHA."""
    extra = synth.small_random(26, 4, [0, 1, 4, 9], 4, 2, 16, 4, 16, "f16")
    for batch in small_batches() + [extra]:
        for include_new in (True, False):
            want_k, want_v = place_numpy(batch, include_new=include_new, poison=True)
            kp = np.full_like(want_k, NAN_BITS[batch.dtype])
            vp = np.full_like(want_v, NAN_BITS[batch.dtype])
            oracle.place_history(batch, kp, vp, include_new=include_new)
            assert np.array_equal(kp, want_k), f"{batch.name}: K placement (new={include_new})"
            assert np.array_equal(vp, want_v), f"{batch.name}: V placement (new={include_new})"


def pin_new_token_slots():
    """The slot where each sequence's step token is written, on the worked example
    of page "大语言模型推理内存管理算法 paged attention", section 8 (block size 4,
    logical blocks 0, 1, 2 in physical blocks 8, 3, 15) with the slot formula of
    page "08. PagedAttention：把 KV Cache 分页管理", section "为什么叫
    PagedAttention". A sequence of length n writes position n - 1: with 11 tokens
    that is the 11th token, still in logical block 2, i.e. 15 * 4 + 2 = 62; with 12
    tokens 15 * 4 + 3 = 63. Every length 0..12 is checked against the fixture's
    block ranges; length 0 has no token (-1)."""
    import types
    g = read_golden("worked_example_bs4.txt")
    bs = int(g["block_size"][0][0])
    physical = [int(x) for x in g["physical"][0]]
    ranges = [(int(v[0]), int(v[2]), int(v[3])) for v in g["logical_block"]]
    lens = np.arange(0, 13, dtype=np.int32)
    batch = types.SimpleNamespace(num_seqs=len(lens), block_size=bs, context_lens=lens,
                                  block_tables=np.tile(np.array(physical, np.int32),
                                                       (len(lens), 1)))
    got = oracle.new_token_slots(batch)
    assert got.dtype == np.int64 and got.shape == (len(lens),)
    for n, s in zip(lens.tolist(), got.tolist()):
        if n == 0:
            assert s == -1, "an empty sequence writes nothing"
            continue
        lb, lo, _ = next(r for r in ranges if r[1] <= n - 1 <= r[2])
        assert s == physical[lb] * bs + (n - 1 - lo), f"length {n}: slot {s}"
    assert got[11] == 62 and got[12] == 63


# --------------------------------------------------------------------------- block manager
def pin_allocator_worked_example():
    g = read_golden("worked_example_bs4.txt")
    bs = int(g["block_size"][0][0])
    n = int(g["num_tokens"][0][0])
    m = BlockManagerModel(32, bs)
    m.add_seq(0, n)
    assert len(m.block_table(0)) == int(g["blocks_needed"][0][0])
    nth, lb = (int(x) for x in g["nth_token_in_logical_block"][0])
    # tokens n+1 .. nth-ish: the 11th and 12th tokens still go into logical block 2
    for pos in range(n, 12):
        slot, src, dst = m.append_slot(0)
        assert slot // bs == m.block_table(0)[lb] and src == dst == -1
    assert len(m.block_table(0)) == 3
    new_at = int(g["nth_token_needs_new_block"][0][0])
    assert m.lens[0] == new_at - 1
    m.append_slot(0)
    assert len(m.block_table(0)) == 4, "the 13th token must take a new block"
    before = m.num_free()
    m.free_seq(0)
    returned = m.num_free() - before
    assert returned in [int(x) for x in g["blocks_returned"][0]] and m.num_free() == 32


def pin_allocator_capacity():
    g = read_golden("capacity_figures.txt")
    val = lambda k: int(g[k][0][0])  # noqa: E731
    m = BlockManagerModel(4096, 16)
    m.add_seq(1, val("request_tokens"))
    assert len(m.block_table(1)) == val("request_blocks")
    free, used, wasted = m.stats()
    assert used == val("request_tokens") and 16 - wasted == val("request_last_block_fill")
    assert wasted * val("llama31_8b_kv_bytes_per_token") == val("request_waste_bytes")
    worst = 0
    for n in range(1, 600):
        mm = BlockManagerModel(64, 16)
        mm.add_seq(0, n)
        worst = max(worst, mm.stats()[2])
    assert worst == val("max_waste_tokens_bs16")
    rng = np.random.default_rng(2)
    mm = BlockManagerModel(1 << 18, 16)
    lens = rng.integers(1, 2000, size=2000)
    for i, n in enumerate(lens):
        mm.add_seq(i, int(n))
    avg = mm.stats()[2] / len(lens)
    assert abs(avg - val("avg_waste_tokens_bs16")) <= 0.75, f"average waste {avg}"


def pin_allocator_cow():
    """Reference-count trace of sharing and copy-on-write."""
    m = BlockManagerModel(16, 4)
    m.add_seq(0, 6)                    # blocks: one full, one holding 2 of 4
    for c in (1, 2, 3):
        m.fork(0, c)
    shared = m.block_table(0)
    assert all(m.ref[b] == 4 for b in shared), "fork adds one reference per block"
    slot, src, dst = m.append_slot(1)  # writes into the shared, partly filled block
    assert src == shared[1] and dst not in shared
    assert m.ref[src] == 3 and m.ref[dst] == 1 and m.block_table(1)[1] == dst
    assert slot == dst * 4 + 2
    for c in (2, 3):
        _, s2, _ = m.append_slot(c)
        assert s2 == shared[1]
    assert m.ref[shared[1]] == 1
    slot0, s0, _ = m.append_slot(0)   # now the sole owner: writes in place
    assert s0 == -1 and slot0 == shared[1] * 4 + 2
    for c in (0, 1, 2, 3):
        m.free_seq(c)
    assert m.num_free() == 16 and all(r == 0 for r in m.ref)


def pin_allocator_sliding_window():
    """Sliding-window release worked by hand (second page, section 5.2: blocks
    leave as the window moves; growth is block by block): block size 16,
    window 32. A 40-token prompt takes 3 blocks; nothing precedes position
    40 - 32 = 8 by a whole block. After 24 more tokens (length 64, 4 blocks) the
    window starts at 32, so blocks 0 and 1 (positions 0-31) go back; the free
    count returns to 8 - 4 + 2 = 6 and the table reads [-1, -1, c, d]."""
    m = BlockManagerModel(8, 16)
    t = m.add_seq(0, 40)
    assert len(t) == 3 and m.num_free() == 5
    assert m.slide_window(0, 32) == 0 and m.block_table(0) == t
    for _ in range(24):
        m.append_slot(0)
    t4 = m.block_table(0)
    assert len(t4) == 4 and m.num_free() == 4
    assert m.slide_window(0, 32) == 2
    assert m.block_table(0) == [-1, -1, t4[2], t4[3]] and m.num_free() == 6
    # the released blocks are the next ones handed out (free list is a stack)
    assert sorted(m.free[-2:]) == sorted(t4[:2])
    m.free_seq(0)
    assert m.num_free() == 8


def pin_allocator_swap():
    """Swapping worked by hand (third page, section "分页还顺带解决了什么": a
    request's blocks go to CPU memory and come back; second page, section 3.1).
    Block size 4, 8 device blocks, 4 host blocks. A 6-token prompt (2 blocks)
    forked once is one group sharing 2 blocks: swapping it out moves 2 blocks
    (not 4), each host block then counted twice, and all 8 device blocks are
    free; swapping back takes 2 device blocks, counted twice each, and frees
    the host space again."""
    m = BlockManagerModel(8, 4)
    m.set_host_blocks(4)
    t = m.add_seq(0, 6)
    m.fork(0, 1)
    out = m.swap_out([0, 1])
    assert len(out) == 2 and sorted(d for d, _ in out) == sorted(t)
    assert m.num_free() == 8 and len(m.host_free) == 2
    assert [m.host_ref[h] for _, h in out] == [2, 2]
    assert m.block_table(0) == m.block_table(1) == [h for _, h in out]
    back = m.swap_in([0, 1])
    assert [h for h, _ in back] == [h for _, h in out]
    assert m.num_free() == 6 and len(m.host_free) == 4
    assert [m.ref[d] for _, d in back] == [2, 2]
    assert m.block_table(0) == [d for _, d in back]
    m.free_seq(0)
    m.free_seq(1)
    assert m.num_free() == 8


def pin_allocator_prefix_cache():
    """Prefix caching worked by hand (third page, section "分页还顺带解决了什么":
    requests that begin alike point their first blocks at the same physical
    blocks, and only completely filled blocks are shared; first page, section
    9: the common prefix's KV is cached). Block size 4, 8 blocks; S is a
    10-token system prompt 1..10."""
    m = BlockManagerModel(8, 4)
    S = list(range(1, 11))
    # A = S + [11, 12]: nothing cached yet; its 3 full blocks get cached
    assert m.add_seq_cached(0, S + [11, 12]) == 0
    assert m.cached_blocks() == (3, 0) and m.num_free() == 5
    a = m.block_table(0)
    # B = S + [21] (11 tokens): blocks [1..4] and [1..8] are A's
    assert m.add_seq_cached(1, S + [21]) == 8
    assert m.block_table(1)[:2] == a[:2] and m.block_table(1)[2] not in a
    assert [m.ref[b] for b in a] == [2, 2, 1] and m.num_free() == 4
    # C = S + [11, 12, 13]: all three of A's blocks precede its last token
    assert m.add_seq_cached(2, S + [11, 12, 13]) == 12
    assert m.block_table(2)[:3] == a and m.num_free() == 3
    # D = A's own prompt: its last token sits in block 3, which is computed again
    assert m.add_seq_cached(3, S + [11, 12]) == 8
    assert m.block_table(3)[2] not in a
    assert m.cached_blocks() == (3, 0)          # block 3's prefix stays on A's block
    assert [m.ref[b] for b in a] == [4, 4, 2] and m.num_free() == 2
    for seq in (0, 1, 2, 3):
        m.free_seq(seq)
    # everything is free; A's blocks keep their prefixes, freed in the order
    # a[2] (when C went), a[1] and a[0] (when D went)
    assert m.num_free() == 8 and m.cached_blocks() == (3, 3)
    assert m.add_seq_cached(4, S + [11, 12]) == 8          # served from the cache
    assert m.block_table(4)[:2] == a[:2] and m.cached_blocks() == (3, 1)
    m.free_seq(4)                                          # a[1], a[0] released again, after a[2]
    # a 24-token request without caching needs 6 blocks: the 5 plain free ones,
    # then the cached block released longest ago, a[2]
    m.add_seq(5, 24)
    assert a[2] in m.block_table(5) and m.cached_blocks() == (2, 2) and m.num_free() == 2
    m.add_seq(6, 4)                                        # then a[1]
    assert m.block_table(6) == [a[1]] and m.cached_blocks() == (1, 1)
    # S + [31] would share a[0] and need 2 more blocks; only a[0] is free
    try:
        m.add_seq_cached(7, S + [31])
        raise AssertionError("expected OutOfBlocks")
    except OutOfBlocks:
        pass
    assert m.cached_blocks() == (1, 1) and m.num_free() == 1 and 7 not in m.tables
    m.free_seq(5)
    assert m.add_seq_cached(7, S + [31]) == 4              # [1..8] left with a[1]
    h = m.block_table(7)
    assert h[0] == a[0] and m.cached_blocks() == (2, 0)    # ... and is cached again on h[1]
    assert m.add_seq_cached(8, S + [11, 12, 13]) == 8      # [1..12] left with a[2]
    assert m.block_table(8)[:2] == h[:2] and m.cached_blocks() == (3, 0)
    assert m.num_free() == 2
    # a shared block that is free stops being free when shared: 3 blocks, one
    # plain free and one cached [1..4] free; 1..4, 6..9, 10 shares that block and
    # needs 2 more, but only 1 is left
    m = BlockManagerModel(3, 4)
    assert m.add_seq_cached(0, [1, 2, 3, 4, 5]) == 0
    m.free_seq(0)
    m.add_seq(1, 4)
    assert m.num_free() == 2 and m.cached_blocks() == (1, 1)
    try:
        m.add_seq_cached(2, [1, 2, 3, 4, 6, 7, 8, 9, 10])
        raise AssertionError("expected OutOfBlocks")
    except OutOfBlocks:
        pass
    assert m.num_free() == 2 and m.cached_blocks() == (1, 1) and 2 not in m.tables


def pin_allocator_prefix_cache_reconnect():
    """A cached prefix whose shorter prefix lost its block is found again once a
    request caches the shorter one anew: the KV of a full block depends only on
    the tokens from position 0 to its end. Block size 4, 6 blocks."""
    m = BlockManagerModel(6, 4)
    assert m.add_seq_cached(0, list(range(1, 13))) == 0    # 3 blocks, 3 prefixes cached
    q = m.block_table(0)
    assert m.slide_window(0, 4) == 2                       # blocks [1..4], [1..8] released
    assert m.cached_blocks() == (3, 2) and m.num_free() == 5
    m.add_seq(1, 12)                                       # the 3 plain free blocks
    m.add_seq(2, 4)                                        # reuses q[0]: [1..4] forgotten
    assert m.block_table(2) == [q[0]] and m.cached_blocks() == (2, 1)
    m.free_seq(1)
    assert m.add_seq_cached(3, [1, 2, 3, 4, 99]) == 0      # [1..4] not cached: computed
    r = m.block_table(3)
    assert m.cached_blocks() == (3, 1)                     # and cached again on r[0]
    assert m.add_seq_cached(4, list(range(1, 9)) + [100]) == 8
    assert m.block_table(4)[:2] == [r[0], q[1]]            # [1..8] still on q[1]
    assert m.cached_blocks() == (3, 0) and m.num_free() == 0


def pin_allocator_prefix_cache_bruteforce():
    """With a pool that never runs short and nothing freed, every full block a
    prompt fills stays cached, so a new prompt of n tokens reuses exactly the
    longest whole-block common prefix it has with any earlier prompt, capped at
    the full blocks before its last token -- counted here by comparing the
    token lists directly -- and takes its other blocks fresh."""
    rng = np.random.default_rng(12)
    bs = 4
    m = BlockManagerModel(4096, bs)
    stems = [list(rng.integers(0, 5, size=24)) for _ in range(3)]
    prompts, fresh = [], 0
    for k in range(120):
        stem = stems[int(rng.integers(0, 3))]
        cut = int(rng.integers(0, 25))
        p = [int(t) for t in stem[:cut]] + [int(t) for t in rng.integers(0, 5, size=int(rng.integers(0, 9)))]
        best = 0
        for r in prompts:
            lcp = 0
            while lcp < min(len(r), len(p)) and r[lcp] == p[lcp]:
                lcp += 1
            best = max(best, lcp // bs)
        want = min(best, max(len(p) - 1, 0) // bs) * bs
        assert m.add_seq_cached(k, p) == want, (k, p)
        fresh += -(-len(p) // bs) - want // bs
        prompts.append(p)
    assert m.num_free() == 4096 - fresh


ALL_ORACLE_PINS = [
    pin_f16_decoder, pin_bf16_decoder, pin_worked_example_slots, pin_bs16_tables, pin_dense,
    pin_len1_returns_v, pin_identical_keys_mean_v, pin_bruteforce_fsum, pin_decode_one_bruteforce,
    pin_relabel, pin_poison,
    pin_partition_merge, pin_reshape_layout, pin_copy_blocks, pin_window_dense,
    pin_window_one_returns_last_v, pin_window_ignores_what_it_left, pin_window_bruteforce_fsum,
    pin_swap_blocks, pin_prefill_dense, pin_prefill_first_token_of_a_prompt,
    pin_prefill_bruteforce_fsum, pin_prefill_relabel, pin_place_history,
    pin_new_token_slots,
]
ALL_MODEL_PINS = [pin_allocator_worked_example, pin_allocator_capacity, pin_allocator_cow,
                  pin_allocator_sliding_window, pin_allocator_swap, pin_allocator_prefix_cache,
                  pin_allocator_prefix_cache_reconnect, pin_allocator_prefix_cache_bruteforce]
