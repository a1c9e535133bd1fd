"""The host-fed decode step (HostDecodeStep) on a B200: inputs packed in one
pinned host buffer, copied in, the step's kernels, the output copied back.
Serial run() and the three-stream enqueue() give the same bits as the
device-resident step, and those are within tolerance of the oracle (decode
over the paged cache: "大语言模型推理内存管理算法 paged attention", sections 7-8)."""
import numpy as np
import pytest
import torch

import synth
from gpu_harness import GpuBatch, oracle_decode, oracle_pools, widen_out
from paged_kv_cache_370_b200 import abi
from paged_kv_cache_370_b200.step import HostDecodeStep, HostStepPipeline
from tolerance import assert_close

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU machines too; every test here needs the GPU
    pytest.skip("no CUDA device", allow_module_level=True)


def _host_step(step, overlapped=False):
    return HostDecodeStep(k_cache=step.k_cache, v_cache=step.v_cache, q=step.q,
                          k_new=step.k_new, v_new=step.v_new, slot_mapping=step.slot_mapping,
                          block_tables=step.block_tables, context_lens=step.context_lens,
                          max_context_len=step.max_context_len, scale=step.scale,
                          partition_tokens=step.partition_tokens, copy_pairs=step.copy_pairs,
                          fused=step.fused, overlapped=overlapped)


@pytest.mark.parametrize("fused", [False, True])
def test_host_step_serial_and_pipelined(fused):
    batch = synth.small_random(61, 7, [1, 16, 17, 200, 513, 64, 1000], 32, 8, 128, 16, 600,
                               "bf16")
    g = GpuBatch(batch, fused=fused)
    dev = g.run().clone()
    h = _host_step(g.step)
    # inputs on the host, so a stale device copy cannot pass: clear the device side
    h.d_in.zero_()
    got = h.run()
    torch.cuda.synchronize()
    assert torch.equal(got.view(torch.int16), dev.cpu().view(torch.int16))
    # three instances pipelined over three streams, twice over (buffers reused)
    hs = [h] + [_host_step(g.step) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    cs = torch.cuda.current_stream()
    for _ in range(2):
        for x in hs:
            x.h_out.fill_(0)
            x.d_in.zero_()
        s_in.wait_stream(cs)
        s_out.wait_stream(cs)
        for x in hs:
            x.enqueue(s_in, cs, s_out)
        cs.wait_stream(s_in)
        cs.wait_stream(s_out)
        torch.cuda.synchronize()
        for x in hs:
            assert torch.equal(x.h_out.view(torch.int16), dev.cpu().view(torch.int16))
    code = abi.pa_device_status()
    assert code == 0, f"device error word {code:#x}"
    kp, vp = oracle_pools(batch)
    assert_close(widen_out(dev), oracle_decode(batch, kp, vp), batch.dtype, "host step")


def test_host_step_graph_round_matches():
    """A captured round of pipelined host steps replays to the same bits."""
    batch = synth.small_random(62, 5, [3, 100, 257, 640, 31], 32, 8, 128, 16, 300, "bf16")
    g = GpuBatch(batch, fused=True)
    dev = g.run().clone().cpu()
    hs = [_host_step(g.step) for _ in range(3)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def round_fn():
        cs = torch.cuda.current_stream()
        s_in.wait_stream(cs)
        s_out.wait_stream(cs)
        for x in hs:
            x.enqueue(s_in, cs, s_out)
        cs.wait_stream(s_in)
        cs.wait_stream(s_out)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        round_fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        round_fn()
    for _ in range(3):
        for x in hs:
            x.h_out.fill_(0)
        graph.replay()
        torch.cuda.synchronize()
        for x in hs:
            assert torch.equal(x.h_out.view(torch.int16), dev.view(torch.int16))
    assert abi.pa_device_status() == 0


@pytest.mark.parametrize("overlapped", [False, True])
def test_host_step_pipeline(overlapped):
    """Two rounds of host-fed steps over two batches (each with its own pools), run
    for several rounds with the copies under other rounds' kernels: every step's
    output has the bits of the device-resident step."""
    b1 = synth.small_random(63, 6, [1, 64, 300, 1000, 17, 513], 32, 8, 128, 16, 400, "bf16")
    b2 = synth.small_random(64, 6, [5, 129, 2, 700, 256, 90], 32, 8, 128, 16, 400, "bf16")
    g1 = GpuBatch(b1, fused=True)
    g2 = GpuBatch(b2, fused=True)
    ref = [g1.run().clone().cpu(), g2.run().clone().cpu()]
    gs = [g1, g2]
    rounds = [[_host_step(gs[i % 2].step, overlapped) for i in range(4)] for _ in range(2)]
    pipe = HostStepPipeline(rounds)
    pipe.capture()
    for n in (1, 2, 5):
        for r in rounds:
            for h in r:
                h.h_out.fill_(0)
        pipe.run(n)
        torch.cuda.synchronize()
        for k, r in enumerate(rounds[:min(n, 2)]):
            for i, h in enumerate(r):
                assert torch.equal(h.h_out.view(torch.int16), ref[i % 2].view(torch.int16)), \
                    f"round set {k} step {i} after {n} rounds"
    assert abi.pa_device_status() == 0
    kp, vp = oracle_pools(b2)
    assert_close(widen_out(ref[1]), oracle_decode(b2, kp, vp), b2.dtype, "pipeline")


@pytest.mark.parametrize("order", [[0, 1, 2], [0, 1, 0, 1, 2]])
def test_host_step_pipeline_as_one_graph(order):
    """Rounds of different sizes (1, 3 and 2 steps) captured as one graph with the
    three streams inside it, sets reused within the pass: every step's output has
    the bits of the device-resident step, after every replay."""
    b1 = synth.small_random(65, 5, [1, 64, 300, 1000, 17], 32, 8, 128, 16, 400, "bf16")
    b2 = synth.small_random(66, 5, [5, 129, 2, 700, 256], 32, 8, 128, 16, 400, "bf16")
    g1 = GpuBatch(b1, fused=True)
    g2 = GpuBatch(b2, fused=True)
    ref = [g1.run().clone().cpu(), g2.run().clone().cpu()]
    gs = [g1, g2]
    sizes = [1, 3, 2]
    rounds, k = [], 0
    for n in sizes:
        rounds.append([_host_step(gs[(k + i) % 2].step, True) for i in range(n)])
        k += n
    pipe = HostStepPipeline(rounds)
    pipe.capture()
    graph = pipe.graph(order)
    for _ in range(3):
        for r in rounds:
            for h in r:
                h.h_out.fill_(0)
        graph.replay()
        torch.cuda.synchronize()
        k = 0
        for r in rounds:
            for i, h in enumerate(r):
                assert torch.equal(h.h_out.view(torch.int16), ref[(k + i) % 2].view(torch.int16))
            k += len(r)
    assert abi.pa_device_status() == 0
