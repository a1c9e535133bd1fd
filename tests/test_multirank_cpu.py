"""The N > 1 host logic on CPU with gloo, world size 2.

Decode shards by sequence with no exchange: each rank decodes its own
sequences and the results equal a single-process decode of the whole batch.
The benchmark's whole-job numbers take the slowest rank's time and the sum of
all ranks' bytes.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for p in (root, os.path.join(root, "tests")):
        if p not in sys.path:
            sys.path.insert(0, p)
    import datetime

    import torch
    import torch.distributed as dist

    import bench
    import oracle
    import pins
    import synth

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # whole-job aggregation: max of times, sum of bytes
        ms, nbytes = bench.rank_aggregate(10.0 + rank, 100.0 * (rank + 1), dist)
        # data-parallel decode: each rank takes every world-th sequence
        batch = synth.small_random(77, 6, [3, 40, 17, 1, 64, 29], 8, 2, 64, 16, 6 * 4 + 1, "bf16")
        kp, vp = pins.place_numpy(batch)
        mine = np.arange(rank, batch.num_seqs, world)
        out = oracle.decode(np.ascontiguousarray(batch.q[mine]), kp, vp,
                            np.ascontiguousarray(batch.block_tables[mine]),
                            np.ascontiguousarray(batch.context_lens[mine]), batch.scale,
                            batch.dtype, num_threads=1)
        gathered = [None] * world
        dist.all_gather_object(gathered, (mine.tolist(), out))
        if rank == 0:
            full = oracle.decode(batch.q, kp, vp, batch.block_tables, batch.context_lens,
                                 batch.scale, batch.dtype, num_threads=1)
            merged = np.zeros_like(full)
            for idx, o in gathered:
                merged[idx] = o
            q.put(("ok", ms, nbytes, bool(np.array_equal(merged, full))))
        dist.barrier()
    except Exception as e:  # noqa: BLE001
        q.put(("error", repr(e)))
        raise
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_by_sequence():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("rank did not finish")
    res = q.get(timeout=10)
    assert res[0] == "ok", res
    _, ms, nbytes, same = res
    assert ms == 11.0 and nbytes == 300.0
    assert same, "sharded decode differs from the single-process decode"
