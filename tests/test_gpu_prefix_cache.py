"""Prefix caching on a B200: requests that share a system prompt are added
through the block manager's prefix cache ("08. PagedAttention：把 KV Cache
分页管理", section "分页还顺带解决了什么": requests that begin alike point
their first, completely filled blocks at the same physical blocks;
"大语言模型推理内存管理算法 paged attention", section 9). Each request writes
the K/V of the positions it does not share, and one paged prefill over every
request's remaining positions matches the oracle's causal prefill over each
whole prompt. The pools start as NaN, so a shared block that was not written
would show in the output. A second step, after every request has ended, is
served from blocks that stayed cached."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_harness import poisoned_pool, to_dev, widen_out
from oracle.allocator_model import BlockManagerModel
from paged_kv_cache_370_b200 import abi
from tolerance import assert_close

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU machines too; every test here needs the GPU
    pytest.skip("no CUDA device", allow_module_level=True)

HQ, HKV, D, BS, NB, DT = 32, 8, 128, 16, 48, "bf16"


def _rows(tokens, heads):
    """[n, heads, D] bits: position p's row depends on tokens[0 .. p] only, as a
    model's K, V and q do, so equal prefixes give equal rows."""
    out = np.empty((len(tokens), heads, D), dtype=np.uint16)
    h = 0
    for p, t in enumerate(tokens):
        h = (h * 1000003 + int(t) + 1) % (1 << 61)
        out[p] = synth.round_bits(np.random.default_rng([h, heads]).standard_normal(
            (heads, D), dtype=np.float32), DT)
    return out


def _kv(tokens):
    k = _rows(tokens, HKV)
    v = _rows([t + 7919 for t in tokens], HKV)  # a different function of the same prefix
    return k, v


def _step(mgr, model, kc, vc, prompts, first_id):
    """Add the prompts through the prefix cache, write what is not cached, one
    prefill over the rest; returns (device out, oracle out, cached counts)."""
    scale = float(synth.scale_for(D))
    ids = list(range(first_id, first_id + len(prompts)))
    cached = []
    for sid, toks in zip(ids, prompts):
        c = mgr.add_seq_cached(sid, toks)
        assert model.add_seq_cached(sid, toks) == c
        cached.append(c)
        n = len(toks)
        if n > c:
            k, v = _kv(toks)
            slots = torch.from_numpy(mgr.seq_slots(sid, c, n - c)).cuda()
            abi.pa_reshape_and_cache(to_dev(k[c:], DT), to_dev(v[c:], DT), slots, kc, vc)
    lens = np.array([len(p) for p in prompts], dtype=np.int32)
    q_lens = lens - np.array(cached, dtype=np.int32)
    q_start = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    q = np.concatenate([_rows([t + 104729 for t in p], HQ)[c:] for p, c in zip(prompts, cached)])
    width = -(-int(lens.max()) // BS)
    tables, lens2 = mgr.fill_tables(ids, width, pad=0)
    assert np.array_equal(lens2, lens)
    qd = to_dev(q, DT)
    out = torch.empty_like(qd)
    abi.pa_prefill(out, qd, kc, vc, torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda(),
                   torch.from_numpy(q_start).cuda(), int(q_lens.max()), int(lens.max()), scale, 0)
    torch.cuda.synchronize()
    # oracle: every prompt whole, each in blocks of its own
    kp = np.zeros((len(prompts) * width, HKV, BS, D), dtype=np.uint16)
    vp = np.zeros_like(kp)
    otab = np.arange(len(prompts) * width, dtype=np.int32).reshape(len(prompts), width)
    for b, p in enumerate(prompts):
        k, v = _kv(p)
        pos = np.arange(len(p))
        oracle.reshape_and_cache(k, v, (otab[b][pos // BS] * BS + pos % BS).astype(np.int64), kp, vp)
    ref = oracle.prefill(q, kp, vp, otab, lens, q_start, scale, DT)
    return widen_out(out), ref, cached


def test_prefix_cached_prefill():
    rng = np.random.default_rng(370)
    tok = lambda n: [int(t) for t in rng.integers(0, 50_000, size=n)]  # noqa: E731
    system = tok(40)
    r0 = system + tok(30)
    mgr, model = abi.BlockManager(NB, BS), BlockManagerModel(NB, BS)
    kc = poisoned_pool((NB, HKV, BS, D), DT)
    vc = poisoned_pool((NB, HKV, BS, D), DT)
    prompts = [r0, system + tok(15), system[:32] + tok(20), tok(30), list(r0)]
    out, ref, cached = _step(mgr, model, kc, vc, prompts, 0)
    # r0 first: nothing cached; then 2 shared blocks of the system prompt; 2; none;
    # r0 again: its 4 full blocks (its last token's block is computed)
    assert cached == [0, 32, 32, 0, 64]
    assert abi.pa_device_status() == 0
    assert_close(out, ref, DT, "prefix-cached prefill", ulp_branch=True)
    for sid in range(len(prompts)):
        mgr.free_seq(sid)
        model.free_seq(sid)
    assert mgr.cached_blocks() == model.cached_blocks()
    # later requests reuse what stayed cached after everyone ended
    prompts2 = [system + tok(25), r0 + tok(10), tok(17)]
    out2, ref2, cached2 = _step(mgr, model, kc, vc, prompts2, 100)
    assert cached2 == [32, 64, 0]
    assert abi.pa_device_status() == 0
    assert_close(out2, ref2, DT, "prefill from blocks cached after the requests ended",
                 ulp_branch=True)
