"""Many decode steps driven by the block manager, on a B200, against the oracle
driven by the block-manager model.

Every step appends one token to every sequence: the manager hands out its slot
(a new block when the last one is full, a copy-on-write when the block is
shared), the step runs the copies (pa_copy_blocks), then writes the new K/V and
decodes in one kernel (pa_decode_append) over the tables the manager fills. The
oracle side replays the same steps with the model allocator and the oracle's
copy / write / decode. Forks mid-loop create shared blocks, frees return them,
so the pools are reused while the loop runs (paged allocation on demand:
"大语言模型推理内存管理算法 paged attention", sections 7-8; copy-on-write:
"PagedAttention 核心思想解析", section 2.3)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_harness import NAN_BITS, poisoned_pool, to_dev, widen_out
from oracle.allocator_model import BlockManagerModel
from paged_kv_cache_370_b200 import abi
from paged_kv_cache_370_b200.step import DecodeStep
from tolerance import assert_close

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU machines too; every test here needs the GPU
    pytest.skip("no CUDA device", allow_module_level=True)


@pytest.mark.parametrize("hq,hkv,dtype", [(32, 8, "bf16"), (8, 8, "f16")])
def test_decode_loop_with_forks_and_frees(hq, hkv, dtype):
    rng = np.random.default_rng(77)
    D, bs, nb, steps, width = 128, 16, 200, 48, 16
    mgr, model = abi.BlockManager(nb, bs), BlockManagerModel(nb, bs)
    shape = (nb, hkv, bs, D)
    kc, vc = poisoned_pool(shape, dtype), poisoned_pool(shape, dtype)
    kp = np.full(shape, NAN_BITS[dtype], dtype=np.uint16)
    vp = np.full(shape, NAN_BITS[dtype], dtype=np.uint16)
    scale = float(synth.scale_for(D))

    def rows(n):
        k = synth.round_bits(rng.standard_normal((n, hkv, D), dtype=np.float32), dtype)
        v = synth.round_bits(rng.standard_normal((n, hkv, D), dtype=np.float32), dtype)
        return k, v

    def add(seq, n):
        mgr.add_seq(seq, n)
        model.add_seq(seq, n)
        if n == 0:
            return
        k, v = rows(n)
        abi.pa_reshape_and_cache(to_dev(k, dtype), to_dev(v, dtype),
                                 torch.from_numpy(mgr.seq_slots(seq, 0, n)).cuda(), kc, vc)
        oracle.reshape_and_cache(k, v, np.asarray(model.seq_slots(seq, 0, n), dtype=np.int64),
                                 kp, vp)

    live = list(range(6))
    for s in live:
        add(s, int(rng.integers(1, 70)))
    next_id = 6
    checked = 0
    for step in range(steps):
        if step % 12 == 5:  # fork: the child shares every block of its parent
            parent = int(rng.choice(live))
            mgr.fork(parent, next_id)
            model.fork(parent, next_id)
            live.append(next_id)
            next_id += 1
        if step % 16 == 11 and len(live) > 3:  # a finished sequence returns its blocks
            gone = int(rng.choice(live))
            mgr.free_seq(gone)
            model.free_seq(gone)
            live.remove(gone)
        if step % 20 == 7:
            add(next_id, int(rng.integers(1, 40)))
            live.append(next_id)
            next_id += 1
        # this step's slots and copy-on-write pairs, on both sides
        slots, mslots, pairs, mpairs = [], [], [], []
        for s in live:
            sl, src, dst = mgr.append_slot(s)
            msl, msrc, mdst = model.append_slot(s)
            assert (src == -1) == (msrc == -1)
            slots.append(sl)
            mslots.append(msl)
            if src >= 0:
                pairs.append((src, dst))
                mpairs.append((msrc, mdst))
        B = len(live)
        q = synth.round_bits(rng.standard_normal((B, hq, D), dtype=np.float32), dtype)
        kn, vn = rows(B)
        tables, lens = mgr.fill_tables(live, width, pad=0)
        mtables = np.zeros((B, width), dtype=np.int32)
        for i, s in enumerate(live):
            t = model.block_table(s)
            mtables[i, :len(t)] = t
        assert np.array_equal(lens, [model.lens[s] for s in live])
        # device: copies, then write + decode in one kernel
        step_obj = DecodeStep(
            k_cache=kc, v_cache=vc, q=to_dev(q, dtype), k_new=to_dev(kn, dtype),
            v_new=to_dev(vn, dtype), slot_mapping=torch.tensor(slots, dtype=torch.int64).cuda(),
            block_tables=torch.from_numpy(tables).cuda(), context_lens=torch.from_numpy(lens).cuda(),
            max_context_len=int(lens.max()), scale=scale,
            copy_pairs=torch.tensor(pairs, dtype=torch.int64).reshape(-1, 2).cuda(), fused=True)
        out = widen_out(step_obj.run())
        # oracle
        oracle.copy_blocks(kp, vp, np.asarray(mpairs, dtype=np.int64).reshape(-1, 2))
        oracle.reshape_and_cache(kn, vn, np.asarray(mslots, dtype=np.int64), kp, vp)
        ref = oracle.decode(q, kp, vp, mtables, lens, scale, dtype)
        assert_close(out, ref, dtype, f"step {step}")
        checked += 1
    assert checked == steps
    code = abi.pa_device_status()
    assert code == 0, f"device error word {code:#x}"
    # the manager and the model agree on what is free at the end
    assert mgr.num_free() == model.num_free()
