#!/usr/bin/env python
"""Benchmark: paged decode attention on B200 -- KV GB/s, % of HBM peak, query tokens/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload llama8b|long_skew|mixed|shared_prompt] [--block-size BS]

A step is one pass of the whole hot path over one batch: the slot-indexed
write of every sequence's new K/V (pa_reshape_and_cache), copy-on-write block
copies where the workload has them (pa_copy_blocks), and paged decode
attention with its split-context merge (pa_decode). The default workload is
the Llama-3.1-8B-shaped single-layer batch: 64 sequences, 32 q / 8 KV heads,
head_dim 128, bf16, 16-token blocks, lengths uniform in [128, 2048], a
65,536-block pool. Four such batches with disjoint blocks live in the pool and
steps rotate through them, so each step reads KV that is not in L2 (1.1 GB of
KV across the four versus a 126 MB L2).

Timing: the W warm-up steps and then exactly the K timed steps are each one
CUDA graph of consecutive steps (K above 512: rounds of 16 steps and one graph
of the rest), the batches in rotation; CUDA events on the launching stream
bracket the timed steps, with a barrier and a device synchronise on both
sides. The decode kernel's own duration comes from at least 50 replays of a
graph of decode launches. With N > 1 (torchrun, one process per GPU) every
rank runs its own batches -- the sequences shard across GPUs with no exchange
-- and the slowest rank's time is used. ``e2e`` repeats the K steps with each
step's inputs in pinned host memory, copied in, and its output copied out,
inside the timed region.

On one GPU the line also carries, under ``workloads``, the other decode
workloads (long-context skew, the mixed batch at every block size, the
shared-prompt batch with its unique and logical bytes, a sliding window) and
chunked prefill, each timed the same way over a short run (``--no-extras``
skips them).

``--impl reference`` times the fp64 CPU oracle on the same workload instead
(a bounded sample of sequences per step), on the host's cores.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402
from paged_kv_cache_370_b200.accounting import (decode_step_bytes, new_token_bytes,  # noqa: E402
                                                split_scratch_bytes, stream_split_scratch_bytes,
                                                tail_overread_bytes, unique_kv_bytes)

METRIC = "paged decode attention: KV GB/s and % of B200 HBM peak; query tokens/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0
MAX_GRAPH_STEPS = 512
# DRAM-traffic records written by bench_traffic.py from ncu captures
TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "pa_decode_llama8b_traffic.json")
PREFILL_TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "pa_prefill_llama8b_traffic.json")


# ------------------------------------------------------------------------------------- setup
def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama8b",
                    choices=["llama8b", "long_skew", "mixed", "shared_prompt", "swap", "prefill"])
    ap.add_argument("--block-size", type=int, default=16, help="block size of the mixed workload")
    ap.add_argument("--variants", type=int, default=4, help="batches rotated (llama8b)")
    ap.add_argument("--partition-tokens", type=int, default=0)
    ap.add_argument("--pool-blocks", type=int, default=65536,
                    help="llama8b pool size (smaller for profiler captures)")
    ap.add_argument("--window", type=int, default=0,
                    help="sliding window: attend to each sequence's last W positions (0: all)")
    ap.add_argument("--no-overlap", action="store_true",
                    help="no programmatic early start of each decode kernel")
    ap.add_argument("--no-fuse", action="store_true",
                    help="separate KV-write kernel instead of pa_decode_append")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--round-reps", type=int, default=4,
                    help="each captured round holds this many steps of every rotated batch "
                         "(device-resident and host-fed timing alike)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="only the headline workload (no per-workload sub-objects)")
    ap.add_argument("--kernel-seconds", type=float, default=0.5,
                    help="length of the kernel-duration loop (at least 50 graph replays)")
    ap.add_argument("--extra-steps", type=int, default=20,
                    help="timed steps of each extra workload")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def measured_peaks():
    """(HBM GB/s, kind) from MEASURED_PEAKS.json, else the fallback figure."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def measured_bf16_sustained():
    """(sustained dense bf16 TFLOP/s, kind) from MEASURED_PEAKS.json, else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return (float(json.load(f)["bf16_tflops_sustained"]),
                    "measured sustained bf16 (cuBLAS, seconds-long loop)")
    except (OSError, KeyError, ValueError):
        return FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback (sustained bf16 under the power cap)"


def read_stream_gbs(torch, device):
    """The read-only streaming rate of this GPU, for context beside the copy peak: the
    library's pa_hbm_read (16-byte evict-first loads, four in flight per thread, 4 CTAs
    of 512 threads per SM) over 4 GiB, best of 5 after 2 warm-up runs; torch's sum over
    the same buffer (a library reduction) beside it."""
    from paged_kv_cache_370_b200 import abi
    x = torch.ones(2 << 30, dtype=torch.bfloat16, device=device)
    sink = torch.zeros(1, dtype=torch.int32, device=device)

    def best_ms(fn):
        best = float("inf")
        for i in range(7):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            if i >= 2:
                best = min(best, a.elapsed_time(b))
        return best

    ours = best_ms(lambda: abi.pa_hbm_read(x, sink))
    lib = best_ms(lambda: torch.sum(x, dtype=torch.float32))
    nbytes = x.numel() * x.element_size()
    del x, sink
    torch.cuda.empty_cache()
    return {"value": round(nbytes / (ours * 1e-3) / 1e9, 1), "unit": "GB/s",
            "how": "pa_hbm_read over 4 GiB (16-byte evict-first loads), best of 5 after 2 "
                   "warm-up runs",
            "torch_sum_gbs": round(nbytes / (lib * 1e-3) / 1e9, 1)}


def recorded_traffic(algorithmic_now: float, record=TRAFFIC_RECORD):
    """DRAM bytes per launch of the kernel, from the ncu record written by
    bench_traffic.py, scaled from the captured case to this launch by algorithmic
    bytes (or FLOPs); None when there is no record or the kernel's source changed
    since the capture."""
    try:
        with open(record) as f:
            rec = json.load(f)
        src = os.path.join(ROOT, rec["source"])
        if hashlib.sha256(open(src, "rb").read()).hexdigest() != rec["source_sha256"]:
            return None
        return int(round(rec["traffic_bytes_per_launch"] * algorithmic_now /
                         rec["algorithmic_per_launch"]))
    except (OSError, KeyError, ValueError, ZeroDivisionError):
        return None


# ---------------------------------------------------------------------------------- clocks
def bus_id_of(torch, device) -> str | None:
    """The PCI bus id of a CUDA device as nvidia-smi and NVML print it."""
    props = torch.cuda.get_device_properties(device)
    bus = getattr(props, "pci_bus_id", None)
    if not isinstance(bus, int):
        return None
    return (f"{getattr(props, 'pci_domain_id', 0):08x}:{bus:02x}:"
            f"{getattr(props, 'pci_device_id', 0):02x}.0")


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons for one GPU (every 50 ms
    over the whole run), and NVML samples every ~0.2 ms while ``fast_start`` /
    ``fast_stop`` bracket a timed region shorter than that interval."""

    # NVML's clock-event reason bits, in the order of FIELDS' four reasons
    _NVML_REASONS = ("nvmlClocksEventReasonHwSlowdown", "nvmlClocksEventReasonHwThermalSlowdown",
                     "nvmlClocksEventReasonSwThermalSlowdown", "nvmlClocksEventReasonSwPowerCap")

    FIELDS = ("timestamp,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.bus_id = (bus_id or "").lower()
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            if self.bus_id and not parts[1].lower().endswith(self.bus_id[-12:]):
                continue
            try:
                self.samples.append((time.time(), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue

    def fast_start(self):
        """Poll NVML from a thread until fast_stop (needs the GPU's bus id)."""
        self._fast = None
        if not self.bus_id:
            return
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByPciBusId(self.bus_id)
            max_sm = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            bits = [getattr(pynvml, n) for n in self._NVML_REASONS]
        except Exception:
            return
        stop = threading.Event()

        def poll():
            while not stop.is_set():
                ts = time.time()
                try:
                    sm = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                    r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                except Exception:
                    return
                # (time, SM MHz, max MHz, reasons, start of the query): a query that
                # overlaps the timed region counts as taken in it
                self.samples.append((time.time(), sm, max_sm,
                                     ["Active" if r & b else "Not Active" for b in bits], ts))
                time.sleep(2e-4)

        self._fast = (threading.Thread(target=poll, daemon=True), stop)
        self._fast[0].start()

    def fast_stop(self):
        if getattr(self, "_fast", None):
            self._fast[1].set()
            self._fast[0].join(timeout=2)
            self._fast = None

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float, t_end: float | None = None) -> dict:
        """Clocks over the timed region [t0, t1]; when it is too short for a sample
        (50 ms apart), over it and the kernel-timing loop that follows, up to t_end."""
        inside = [s for s in self.samples
                  if (s[4] if len(s) > 4 else s[0]) <= t1 and s[0] >= t0]
        end = max(t1, t_end or t1)
        used = inside or [s for s in self.samples if t0 - 0.1 <= s[0] <= end + 0.1]
        if not used:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "samples_in_timed_region": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in used for i, v in enumerate(s[3]) if v == "Active"})
        return {"sm_mhz": float(np.median([s[1] for s in used])),
                "sm_max_mhz": float(max(s[2] for s in used)), "reasons": reasons,
                "samples": len(used), "samples_in_timed_region": len(inside),
                "window": ("the timed region (NVML queries that overlap it)" if inside else
                           f"the timed region ({1e3 * (t1 - t0):.1f} ms) and the kernel-timing "
                           f"loop after it ({1e3 * (end - t1):.0f} ms), sampled every 50 ms")}


# ------------------------------------------------------------------------------- workloads
def make_batches(args, rank):
    """Host-side batches of the workload for one rank (seeded per rank)."""
    seed_shift = 1_000_003 * rank
    if args.workload == "llama8b":
        return [synth.llama8b(seed=synth.SEED_BASE + 2 + seed_shift, variant=v,
                              num_variants=args.variants, num_blocks=args.pool_blocks)
                for v in range(args.variants)]
    if args.workload == "long_skew":
        return [synth.long_skew(seed=synth.SEED_BASE + 3 + seed_shift)]
    if args.workload == "mixed":
        return [synth.mixed_sweep(args.block_size, seed=synth.SEED_BASE + 5 + seed_shift)]
    return None  # shared_prompt is built through the block manager


def workload_config(args, batches, pt):
    cfg = _workload_config(args, batches, pt)
    if getattr(args, "window", 0) > 0:
        cfg["window"] = args.window
    return cfg


def _workload_config(args, batches, pt):
    if args.workload == "llama8b":
        b = batches[0]
        return {"workload": "Llama-3.1-8B-shaped single-layer paged decode",
                "num_seqs": b.num_seqs, "num_q_heads": b.num_q_heads,
                "num_kv_heads": b.num_kv_heads, "head_dim": b.head_dim,
                "block_size": b.block_size, "context_lens": "uniform [128, 2048]",
                "num_blocks": b.num_blocks, "partition_tokens": pt,
                "batches_rotated": len(batches),
                "l2": f"inputs larger than L2: {len(batches)} rotating batches, "
                      f"{sum(decode_step_bytes(x.context_lens, 32, 8, 128, 16)['kv'] for x in batches) / 1e9:.2f} GB of KV",
                "timing": (f"one CUDA graph of the {args.steps} timed steps (the batches in "
                           "rotation), after a graph of the warm-up steps; CUDA events on the "
                           "stream" if args.steps <= MAX_GRAPH_STEPS else
                           f"CUDA graphs of {len(batches) * max(1, args.round_reps)} steps "
                           "(the batches in rotation) replayed back to back, then one graph "
                           "of the rest; CUDA events on the stream") +
                          "; a 0.1 ms idle kernel queued ahead of the start event, so that "
                          "the host's submission of the graph is not inside the timed region",
                "launch": ("plain stream order" if args.no_overlap or args.no_fuse else
                           "programmatic early start: each decode kernel's start-up overlaps "
                           "the previous kernel's tail (pa_decode_append_overlapped)")}
    if args.workload == "long_skew":
        return {"workload": "long-context skew decode", "num_seqs": 8, "num_q_heads": 32,
                "num_kv_heads": 8, "head_dim": 128, "block_size": 16,
                "context_lens": "uniform [8192, 32768]", "partition_tokens": pt,
                "l2": "inputs larger than L2 (671 MB KV per step)"}
    if args.workload == "mixed":
        return {"workload": "mixed serving batch", "num_seqs": 256, "num_q_heads": 32,
                "num_kv_heads": 8, "head_dim": 128, "block_size": args.block_size,
                "context_lens": "log-uniform [16, 4096]", "partition_tokens": pt,
                "l2": "inputs larger than L2 (~770 MB KV per step)"}
    return {"workload": "OPT-13B-shaped shared-prompt decode with copy-on-write",
            "num_seqs": 64, "num_q_heads": 40, "num_kv_heads": 40, "head_dim": 128,
            "block_size": 16, "prompts": 16, "prompt_len": 512, "fork": 4,
            "partition_tokens": pt, "l2": "shared prompt blocks hit in L2 by design"}


def to_dev(bits, dtype, torch, device):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device)
    return t.view(torch.bfloat16 if dtype == "bf16" else torch.float16)


def device_steps(args, batches, torch, device):
    """Place the batches into one device pool and return (steps, byte counts, pool)."""
    from paged_kv_cache_370_b200 import abi
    from paged_kv_cache_370_b200.step import DecodeStep
    if batches is None:
        return shared_prompt_steps(args, torch, device)
    b0 = batches[0]
    shape = (b0.num_blocks, b0.num_kv_heads, b0.block_size, b0.head_dim)
    tdt = torch.bfloat16 if b0.dtype == "bf16" else torch.float16
    kc = torch.zeros(shape, dtype=tdt, device=device)
    vc = torch.zeros(shape, dtype=tdt, device=device)
    steps, infos = [], []
    for b in batches:
        slots = abi.pa_slot_mapping(b.block_tables, b.context_lens, b.block_size)
        hist, new = b.history_rows(), b.new_token_rows()
        k_all, v_all = to_dev(b.k, b.dtype, torch, device), to_dev(b.v, b.dtype, torch, device)
        hidx = torch.from_numpy(hist).to(device)
        abi.pa_reshape_and_cache(k_all[hidx].contiguous(), v_all[hidx].contiguous(),
                                 torch.from_numpy(slots[hist]).to(device), kc, vc)
        nidx = torch.from_numpy(new).to(device)
        step = DecodeStep(k_cache=kc, v_cache=vc, q=to_dev(b.q, b.dtype, torch, device),
                          k_new=k_all[nidx].contiguous(), v_new=v_all[nidx].contiguous(),
                          slot_mapping=torch.from_numpy(slots[new]).to(device),
                          block_tables=torch.from_numpy(b.block_tables).to(device),
                          context_lens=torch.from_numpy(b.context_lens).to(device),
                          max_context_len=b.max_context_len, scale=float(b.scale),
                          partition_tokens=args.partition_tokens, fused=not args.no_fuse,
                          window=args.window, overlapped=not args.no_overlap)
        del k_all, v_all
        steps.append(step)
        infos.append(_byte_info(b.context_lens, b.num_q_heads, b.num_kv_heads, b.head_dim,
                                b.block_size, step.partition, b.num_seqs, args.window,
                                _grid_ctas(step)))
    torch.cuda.synchronize()
    return steps, infos


def _byte_info(lens, hq, hkv, d, bs, pt, ntok, window=0, nctas=0):
    """Algorithmic bytes of one step and the bytes moved beyond them. ``nctas``: CTAs
    of the even-split kernel (0: the partition kernel runs), whose split-segment
    pieces are its scratch."""
    lens = np.asarray(lens, dtype=np.int64)
    seen = lens
    if window > 0:
        # the positions a window reads: the last `window` of each sequence; the
        # even-split kernel sees each from the block of its first attended position
        seen = np.minimum(lens, window)
        lo = np.maximum(lens - window, 0)
        kernel_lens = lens - (lo // bs) * bs
    else:
        kernel_lens = lens
    scratch = (stream_split_scratch_bytes(kernel_lens, hkv, hq // hkv, d, nctas) if nctas
               else split_scratch_bytes(seen, hq, d, pt))
    return {"decode": decode_step_bytes(seen, hq, hkv, d, bs), "scratch": scratch,
            "tail": tail_overread_bytes(seen, hkv, d, bs),
            "write": new_token_bytes(ntok, hkv, d), "lens": seen}


def shared_prompt_steps(args, torch, device):
    from paged_kv_cache_370_b200 import abi
    from paged_kv_cache_370_b200.step import DecodeStep
    s = synth.shared_prompt()
    mgr = abi.BlockManager(s.num_blocks, s.block_size)
    shape = (s.num_blocks, s.num_heads, s.block_size, s.head_dim)
    kc = torch.zeros(shape, dtype=torch.float16, device=device)
    vc = torch.zeros(shape, dtype=torch.float16, device=device)
    slots, rows_k, rows_v = [], [], []
    for i in range(s.num_prompts):
        p0, p1, p2, p3 = (4 * i + j for j in range(4))
        mgr.add_seq(p0, s.prompt_len)
        slots.extend(mgr.seq_slots(p0, 0, s.prompt_len).tolist())
        rows_k.append(s.prompt_k[i])
        rows_v.append(s.prompt_v[i])
        mgr.fork(p0, p1)
        mgr.fork(p0, p2)
        for _ in range(int(s.n_before_fork[i])):
            slots.append(mgr.append_slot(p1)[0])
        rows_k.append(s.gen_k[i][1])
        rows_v.append(s.gen_v[i][1])
        mgr.fork(p1, p3)
        for seq, j, n in ((p0, 0, s.n_after[i, 0]), (p2, 2, s.n_after[i, 1])):
            for _ in range(int(n)):
                slots.append(mgr.append_slot(seq)[0])
            rows_k.append(s.gen_k[i][j])
            rows_v.append(s.gen_v[i][j])
    abi.pa_reshape_and_cache(to_dev(np.concatenate(rows_k), "f16", torch, device),
                             to_dev(np.concatenate(rows_v), "f16", torch, device),
                             torch.tensor(slots, dtype=torch.int64, device=device), kc, vc)
    new_slots, pairs = [], []
    ids = [4 * i + j for i in range(s.num_prompts) for j in range(4)]
    for sid in ids:
        slot, src, dst = mgr.append_slot(sid)
        new_slots.append(slot)
        if src >= 0:
            pairs.append((src, dst))
    tables, lens = mgr.fill_tables(ids, 48, pad=0)
    step = DecodeStep(k_cache=kc, v_cache=vc, q=to_dev(s.q, "f16", torch, device),
                      k_new=to_dev(s.new_k, "f16", torch, device),
                      v_new=to_dev(s.new_v, "f16", torch, device),
                      slot_mapping=torch.tensor(new_slots, dtype=torch.int64, device=device),
                      block_tables=torch.from_numpy(tables).to(device),
                      context_lens=torch.from_numpy(lens).to(device),
                      max_context_len=int(lens.max()), scale=float(s.scale),
                      partition_tokens=args.partition_tokens,
                      copy_pairs=torch.tensor(pairs, dtype=torch.int64, device=device),
                      fused=not args.no_fuse)
    torch.cuda.synchronize()
    info = _byte_info(lens, 40, 40, 128, 16, step.partition, len(ids), 0, _grid_ctas(step))
    info["copy"] = 2 * 2 * len(pairs) * 40 * 16 * 128 * 2
    # each physical block once, however many branches read it (the forked prompt)
    info["unique_kv"] = unique_kv_bytes(tables, lens, 16, 40, 128)
    return [step], [info]


# ------------------------------------------------------------------------------ timing (GPU)
def rank_aggregate(ms: float, nbytes: float, dist, device=None):
    """Whole-job numbers: the slowest rank's time and the bytes all ranks moved."""
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    b = torch.tensor([nbytes], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(b, op=dist.ReduceOp.SUM)
    return float(t.item()), float(b.item())


def capture(fn, torch):
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # warm the launch path outside capture
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    return g


def _grid_ctas(step):
    from paged_kv_cache_370_b200 import abi
    B, hq, d = step.q.shape
    nb, hkv, bs, _ = step.k_cache.shape
    return abi.pa_decode_grid_ctas(B, hq, hkv, d, bs, nb, step.max_context_len,
                                   step.partition_tokens)


def _launches(step, fused):
    return step.append_launches if fused else step.decode_launches


def upload_graphs(plan, stream):
    """Upload each graph's executable to the device ahead of its first replay
    (cudaGraphUpload: no work runs), so that the timed region does not pay for
    the upload a first launch would otherwise do."""
    try:
        from cuda.bindings import runtime as rt
    except ImportError:  # older cuda-python layout
        from cuda import cudart as rt
    st = rt.cudaStream_t(init_value=int(stream.cuda_stream))
    for g, _ in plan:
        handle = g.raw_cuda_graph_exec()
        err = rt.cudaGraphUpload(rt.cudaGraphExec_t(init_value=int(handle)), st)[0]
        if int(err) != 0:
            raise RuntimeError(f"cudaGraphUpload failed: {err}")


def time_graphs(plan, stream, torch):
    """Device milliseconds of replaying [(graph, times), ...] once, CUDA events on
    ``stream`` (behind a 0.1 ms idle kernel, so the host's submission is not timed)."""
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        torch.cuda._sleep(int(0.1e-3 * 1.965e9))
    a.record(stream)
    for g, n in plan:
        for _ in range(n):
            g.replay()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b)


def step_plan(n, start, fn, steps, R, torch):
    """Graphs that run exactly n consecutive steps (batch (start + i) % V for step
    i): one graph of n steps, or above MAX_GRAPH_STEPS rounds of R and one graph of
    the rest (R a multiple of V, so the rotation carries on across rounds)."""
    V = len(steps)

    def graph(m):
        return capture(lambda: [fn(steps[(start + i) % V]) for i in range(m)], torch)

    if n <= 0:
        return []
    if n <= MAX_GRAPH_STEPS:
        return [(graph(n), 1)]
    rounds, rest = divmod(n, R)
    plan = [(graph(R), rounds)]
    if rest:
        plan.append((graph(rest), 1))
    return plan


def run_ours(args, rank, world, local, dist):
    import torch
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    batches = make_batches(args, rank)
    steps, infos = device_steps(args, batches, torch, device)
    pt = steps[0].partition
    fused = steps[0].fused
    V = len(steps)

    def pre(s):
        s.copy()
        if not s.fused:
            s.write()

    def has_pre(s):
        return (not s.fused) or (s.copy_pairs is not None and s.copy_pairs.numel() > 0)

    def one_step(s):
        pre(s) if has_pre(s) else None
        s.append() if s.fused else s.attend()

    def decode_only(s):
        s.append() if s.fused else s.attend()

    K, Wm = args.steps, args.warmup
    R = V * max(1, args.round_reps)
    off = Wm % V  # the timed steps carry the batch rotation on from the warm-up
    warm = step_plan(Wm, 0, one_step, steps, R, torch)
    timed = step_plan(K, off, one_step, steps, R, torch)
    g_dec = capture(lambda: [decode_only(steps[i % V]) for i in range(R)], torch)
    g_pre = [capture(lambda s=s: pre(s), torch) if has_pre(s) else None for s in steps]

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    stream = torch.cuda.current_stream()
    sampler = ClockSampler(bus_id_of(torch, device))
    sampler.start()
    time.sleep(0.3)
    # ---- warm-up: exactly W steps, untimed; the timed graphs uploaded to the device
    time_graphs(warm, stream, torch)
    upload_graphs(timed, stream)
    # ---- the timed region: exactly K steps
    start_ev, end_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    sampler.fast_start()
    t0 = time.time()
    # the device idles ~0.1 ms on a spin kernel (torch's) while the host queues the
    # start event and the graph behind it: the events then bracket the K steps'
    # execution, not the host's submission of the graph
    with torch.cuda.stream(stream):
        torch.cuda._sleep(int(0.1e-3 * 1.965e9))
    start_ev.record(stream)
    for g, n in timed:
        for _ in range(n):
            g.replay()
    end_ev.record(stream)
    barrier()
    t1 = time.time()
    sampler.fast_stop()
    total_ms = start_ev.elapsed_time(end_ev)
    # ---- the decode kernel's own duration: >= 50 replays of a graph of R decode
    # launches (about half a second), CUDA events on the same stream
    est = max(total_ms / max(K, 1), 1e-3)
    reps = max(50, int(math.ceil(1e3 * args.kernel_seconds / (est * R))))
    tk0 = time.time()
    dec_ms = time_graphs([(g_dec, reps)], stream, torch) / (reps * R)
    tk1 = time.time()
    pre_ms = 0.0
    if any(g is not None for g in g_pre):
        pre_ms = time_graphs([(g, 50) for g in g_pre if g is not None], stream, torch) / (50 * V)
    # ---- the spread: the timed steps replayed again, an event after each replay
    rep_ms = [time_graphs(timed, stream, torch) / K for _ in range(5)]
    time.sleep(0.2)
    sampler.stop()
    read_stream = read_stream_gbs(torch, device)
    step_bytes = [infos[(off + i) % V]["decode"]["total"] for i in range(K)]
    total_ms_max, all_bytes = rank_aggregate(total_ms, float(sum(step_bytes)), dist, device)
    ms_per_step = total_ms_max / K
    gbs = all_bytes / (total_ms_max * 1e-3) / 1e9
    q_tok = sum(len(infos[(off + i) % V]["lens"]) for i in range(K)) * world / \
        (total_ms_max * 1e-3)

    peak, peak_kind = measured_peaks()
    # the fused kernel also reads each new token's K/V and stores it at its slot
    dec_bytes = float(np.mean([infos[i % V]["decode"]["total"] +
                               (infos[i % V]["write"] if fused else 0) for i in range(R)]))
    achieved = dec_bytes / (dec_ms * 1e-3) / 1e9
    # recorded for the plain (no window) kernel on this workload only
    traffic = (recorded_traffic(dec_bytes) if args.workload == "llama8b" and args.window == 0
               else None)
    launches = sum(steps[(off + i) % V].launches() for i in range(K))
    nctas = _grid_ctas(steps[0])

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, steps, infos, torch, device, dist, world, dec_ms)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and batches is not None:
        cpu = cpu_baseline(batches[0], args.cpu_seconds)
    clocks = sampler.summary(t0, t1, tk1)
    res = {
        "metric": METRIC, "value": round(gbs, 2), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": Wm, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype":
            "bf16" if (batches and batches[0].dtype == "bf16") else "f16",
        "data": "synthetic (seeded N(0,1) K/V/q, random block tables)",
        "config": workload_config(args, batches, pt),
        "query_tokens_per_s": round(q_tok, 1),
        "pct_of_copy_peak": round(100 * gbs / world / peak, 2),
        "pct_of_hbm_nominal_8tbs": round(100 * gbs / world / NOMINAL_HBM_GBS, 2),
        "ms_per_step_over_replays": {"median": round(float(np.median(rep_ms)), 5),
                                     "min": round(float(np.min(rep_ms)), 5),
                                     "max": round(float(np.max(rep_ms)), 5),
                                     "replays": len(rep_ms),
                                     "how": "the K timed steps replayed again 5 times, "
                                            "CUDA events around each replay"},
        "hbm_read_stream": read_stream,
        "roofline": {"bound": "hbm",
                     "kernel": ("pa_decode_append (KV write + decode, one kernel)" if fused
                                else "pa_decode"),
                     "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                     "traffic": traffic, "algorithmic_bytes_per_launch": int(dec_bytes),
                     "avg_launch_ms": round(dec_ms, 5),
                     "how": f"{reps} replays of a graph of {R} decode launches (the batches "
                            "in rotation), CUDA events on the launching stream",
                     "frac_of_nominal_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
                     "frac_of_read_stream": (round(achieved / read_stream["value"], 4)
                                             if read_stream.get("value") else None)},
        "kernel_ms": {"before_decode": round(pre_ms, 5), "decode": round(dec_ms, 5)},
        "extra_bytes_per_step": {
            "split_scratch": int(np.mean([infos[i % V]["scratch"] for i in range(V)])),
            "split_scratch_kernel": ("even-split: pieces of split segments, "
                                     f"{nctas} CTAs" if nctas else
                                     "partition kernel: partial states of split sequences"),
            "kv_write": int(infos[0]["write"]),
            "copy_on_write": int(infos[0].get("copy", 0)),
            "tail_overread": int(np.mean([infos[i % V]["tail"] for i in range(V)]))},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    if e2e is not None:
        res["e2e"] = e2e
    if cpu is not None:
        res["cpu_baseline"] = cpu
    del steps, g_dec, g_pre, timed, warm
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def run_e2e(args, steps, infos, torch, device, dist, world, step_ms):
    """The same K steps fed from pinned host buffers through the library's
    HostStepPipeline: each round's uploads, kernels and downloads are graphs on
    three streams, the next round's uploads and the previous round's downloads
    running under a round's kernels. Up to 64 steps: rounds that grow from one
    step and shrink back to one (only the first upload and the last download are
    exposed); beyond: two sets of 16 steps taking turns, then the rest."""
    from paged_kv_cache_370_b200.step import HostDecodeStep, HostStepPipeline
    V = len(steps)
    K = args.steps
    off = args.warmup % V

    def host_step(s):
        return HostDecodeStep(k_cache=s.k_cache, v_cache=s.v_cache, q=s.q, k_new=s.k_new,
                              v_new=s.v_new, slot_mapping=s.slot_mapping,
                              block_tables=s.block_tables, context_lens=s.context_lens,
                              max_context_len=s.max_context_len, scale=s.scale,
                              partition_tokens=s.partition_tokens, copy_pairs=s.copy_pairs,
                              fused=s.fused, window=s.window, overlapped=s.overlapped)

    # this box's copy times for one step's inputs and output (pinned host memory),
    # to plan the rounds: a round's uploads must fit under the kernels before it
    probe = host_step(steps[0])
    probe.upload()
    probe.download()
    torch.cuda.synchronize()
    st = torch.cuda.Stream()

    def copy_us(fn, reps=20):
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(st):
            a0.record(st)
            for _ in range(reps):
                fn()
            a1.record(st)
        torch.cuda.synchronize()
        return 1e3 * a0.elapsed_time(a1) / reps

    up_us, down_us = copy_us(probe.upload), copy_us(probe.download)
    kern_us = 1e3 * step_ms
    del probe
    if K <= 64:
        sizes = HostStepPipeline.ramp_sizes(K, kernel_us=kern_us, upload_us=up_us,
                                            download_us=down_us)
        rounds, i = [], 0
        for n in sizes:
            rounds.append([host_step(steps[(off + i + j) % V]) for j in range(n)])
            i += n
        order = list(range(len(rounds)))
        shape = (f"rounds of {sizes} steps, planned from {up_us:.1f} us per upload, "
                 f"{down_us:.1f} us per download and {kern_us:.1f} us of kernels per step")
    else:
        R = V * max(1, args.round_reps)
        n_rounds, rest = divmod(K, R)
        rounds = [[host_step(steps[(off + j) % V]) for j in range(R)] for _ in range(2)]
        order = [r % 2 for r in range(n_rounds)]
        if rest:
            rounds.append([host_step(steps[(off + j) % V]) for j in range(rest)])
            order.append(2)
        shape = f"two sets of {R} steps taking turns, then {rest}"
    pipe = HostStepPipeline(rounds)
    pipe.capture()
    # the whole pass (every round's uploads, kernels and downloads on their three
    # streams) as one graph: one launch from the host
    g = pipe.graph(order)
    stream = torch.cuda.current_stream()
    for _ in range(max(1, -(-max(args.warmup, 3) // K))):  # >= W (and >= 3) warm-up steps
        g.replay()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    g.replay()
    b.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    my_bytes = sum(infos[(off + i) % V]["decode"]["total"] for i in range(K))
    ms, total = rank_aggregate(a.elapsed_time(b), float(my_bytes), dist, device)
    h_all = [h for x in order for h in rounds[x]]
    return {"value": round(total / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "ms_per_step": round(ms / K, 5),
            "h2d_bytes_per_step": int(np.mean([h.h2d_bytes for h in h_all])),
            "d2h_bytes_per_step": int(np.mean([h.d2h_bytes for h in h_all])),
            "how": "pinned host inputs copied in and output copied out every step through the "
                   f"library's HostStepPipeline ({shape}): each round's uploads, kernels and "
                   "downloads on three streams, the next round's uploads and the previous "
                   "round's downloads under a round's kernels, the whole pass one CUDA graph "
                   "(HostStepPipeline.graph)"}


# --------------------------------------------------------------------------- CPU (oracle)
def _oracle_setup(batch):
    import oracle
    shape = (batch.num_blocks, batch.num_kv_heads, batch.block_size, batch.head_dim)
    kp = np.zeros(shape, dtype=np.uint16)
    vp = np.zeros(shape, dtype=np.uint16)
    oracle.place_history(batch, kp, vp, include_new=True)
    return kp, vp


def _oracle_pass(batch, kp, vp, seqs, threads=0):
    import oracle
    return oracle.decode(np.ascontiguousarray(batch.q[seqs]), kp, vp,
                         np.ascontiguousarray(batch.block_tables[seqs]),
                         np.ascontiguousarray(batch.context_lens[seqs]), batch.scale,
                         batch.dtype, num_threads=threads)


def cpu_baseline(batch, target_s):
    """The oracle, as it stands, on whole sequences of the batch for about target_s seconds."""
    import oracle
    kp, vp = _oracle_setup(batch)
    cores = oracle.max_threads()
    order = np.arange(batch.num_seqs)
    done, nbytes, t_used, passes = 0, 0, 0.0, 0
    while t_used < target_s and passes < 64:
        seqs = order[done % batch.num_seqs: done % batch.num_seqs + 8]
        t = time.perf_counter()
        _oracle_pass(batch, kp, vp, seqs)
        t_used += time.perf_counter() - t
        nbytes += decode_step_bytes(batch.context_lens[seqs], batch.num_q_heads,
                                    batch.num_kv_heads, batch.head_dim,
                                    batch.block_size)["total"]
        done += len(seqs)
        passes += 1
    # one thread, on a smaller sample of the same sequences
    n1, b1, t1 = 0, 0, 0.0
    while t1 < max(1.0, target_s / 6) and n1 < batch.num_seqs:
        seqs = order[n1: n1 + 2]
        t = time.perf_counter()
        _oracle_pass(batch, kp, vp, seqs, threads=1)
        t1 += time.perf_counter() - t
        b1 += decode_step_bytes(batch.context_lens[seqs], batch.num_q_heads,
                                batch.num_kv_heads, batch.head_dim, batch.block_size)["total"]
        n1 += len(seqs)
    return {"value": round(nbytes / t_used / 1e9, 4), "unit": "GB/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{done} sequences of the batch (8 per call, {passes} calls, "
                      f"{t_used:.1f} s), fp64, OpenMP over (sequence, q head)",
            "query_tokens_per_s": round(done / t_used, 2),
            "single_thread": {"value": round(b1 / t1 / 1e9, 4), "unit": "GB/s",
                              "sample": f"{n1} sequences (2 per call, {t1:.1f} s), one thread"}}


def run_reference(args, rank, world):
    import oracle
    batches = make_batches(args, rank)
    if batches is None:
        return {"impl": "reference", "unavailable": "the oracle arm covers the random-table "
                "workloads only"}
    batch = batches[0]
    kp, vp = _oracle_setup(batch)
    cores = oracle.max_threads()
    # size the per-step sample so the whole run stays within about two minutes
    t = time.perf_counter()
    _oracle_pass(batch, kp, vp, np.arange(1))
    one = max(time.perf_counter() - t, 1e-4)
    per_step_budget = 120.0 / max(1, args.steps + args.warmup)
    nseq = int(max(1, min(batch.num_seqs, per_step_budget / one)))
    for i in range(args.warmup):
        _oracle_pass(batch, kp, vp, (np.arange(nseq) + i * nseq) % batch.num_seqs)
    total_t, total_b, total_q = 0.0, 0, 0
    for i in range(args.steps):
        seqs = (np.arange(nseq) + i * nseq) % batch.num_seqs
        t = time.perf_counter()
        _oracle_pass(batch, kp, vp, seqs)
        total_t += time.perf_counter() - t
        total_b += decode_step_bytes(batch.context_lens[seqs], batch.num_q_heads,
                                     batch.num_kv_heads, batch.head_dim,
                                     batch.block_size)["total"]
        total_q += nseq
    gbs = total_b / total_t / 1e9
    cfg = workload_config(args, batches, 0)
    return {"metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "impl": "reference",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * total_t / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": cfg,
            "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": cores,
                             "kind": "oracle",
                             "sample": f"{nseq} of {batch.num_seqs} sequences per step"},
            "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "query_tokens_per_s": round(total_q / total_t, 2)}


# ------------------------------------------------------------------------------------- swap
def run_swap(args):
    """Block swap between the device pool and the pinned host swap space
    (pa_swap_out / pa_swap_in): Llama-3.1-8B-shaped blocks (8 kv heads x 16
    slots x 128 bf16, K and V = 64 KiB per block), 2048 random blocks per call
    (128 MiB each way), CUDA events on the stream, one call per direction per step."""
    import torch
    from paged_kv_cache_370_b200 import abi
    dev = torch.device("cuda", 0)
    nb, nh, hkv, bs, d, n = 65536, 4096, 8, 16, 128, 2048
    kc = torch.zeros((nb, hkv, bs, d), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    space = abi.SwapSpace(nh, hkv, bs, d, "bf16")
    rng = np.random.default_rng(9)
    out_pairs = torch.from_numpy(np.stack([rng.permutation(nb)[:n], rng.permutation(nh)[:n]], 1)
                                 .astype(np.int64)).to(dev)
    in_pairs = torch.from_numpy(np.stack([out_pairs[:, 1].cpu().numpy(), rng.permutation(nb)[:n]], 1)
                                .astype(np.int64)).to(dev)
    nbytes = n * 2 * hkv * bs * d * 2
    res = {}
    for name, fn, pairs in (("out", abi.pa_swap_out, out_pairs), ("in", abi.pa_swap_in, in_pairs)):
        for _ in range(args.warmup):
            fn(space, kc, vc, pairs)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            fn(space, kc, vc, pairs)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / args.steps
        res[name] = {"ms": round(ms, 4), "GB/s": round(nbytes / ms / 1e6, 2)}
    code = abi.pa_device_status()
    space.close()
    return {"metric": "KV block swap GB/s (device pool <-> pinned host swap space)",
            "value": round((res["out"]["GB/s"] + res["in"]["GB/s"]) / 2, 2), "unit": "GB/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "swap 2048 random 64 KiB blocks each way", "bytes_per_call": nbytes},
            "out": res["out"], "in": res["in"], "device_error_word": code,
            "gpu_launches": 2 * args.steps}


# ---------------------------------------------------------------------------------- prefill
def prefill_flops(batch, window=0) -> float:
    """Algorithmic FLOPs of causal paged prefill attention: for every (query
    token, q head), 2*D for its scores and 2*D for its weighted V per key it
    attends to (positions [lo, p])."""
    qs = batch.meta["q_start"]
    keys = 0
    for b in range(batch.num_seqs):
        n, m = int(batch.context_lens[b]), int(qs[b + 1] - qs[b])
        p = np.arange(n - m, n, dtype=np.int64)
        lo = np.maximum(p + 1 - window, 0) if window > 0 else np.zeros_like(p)
        keys += int((p + 1 - lo).sum())
    return 4.0 * batch.head_dim * batch.num_q_heads * keys


def prefill_measure(pool_blocks, window, n_timed, n_warm):
    """Chunked prefill on the Llama-3.1-8B shapes (16 sequences x 512 new tokens
    after up to 1,536 history tokens): one step = the chunk's K/V write
    (pa_reshape_and_cache) + pa_prefill, over 4 rotating batches. n_warm steps,
    then exactly n_timed steps, each a graph of consecutive steps; the prefill
    kernel's own duration from >= 50 replays of a graph of its launches."""
    import torch
    from paged_kv_cache_370_b200 import abi
    dev = torch.device("cuda", torch.cuda.current_device())
    # 4 batches, each drawing distinct ids from its own quarter of the pool
    nv, per = 4, max(2048, pool_blocks // 4)
    batches = [synth.llama8b_prefill(seed=synth.SEED_BASE + 7 + 10 * v, num_blocks=per)
               for v in range(nv)]
    b0 = batches[0]
    shape = (nv * per, b0.num_kv_heads, b0.block_size, b0.head_dim)
    kc = torch.zeros(shape, dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    steps = []
    for v, b in enumerate(batches):
        tables = (b.block_tables + v * per).astype(np.int32)
        b.block_tables = tables
        slots = abi.pa_slot_mapping(tables, b.context_lens, b.block_size)
        qs = b.meta["q_start"]
        new_rows = np.concatenate([np.arange(b.seq_start[i + 1] - (qs[i + 1] - qs[i]),
                                             b.seq_start[i + 1]) for i in range(b.num_seqs)])
        hist = np.setdiff1d(np.arange(b.total_tokens), new_rows)
        k_all, v_all = to_dev(b.k, "bf16", torch, dev), to_dev(b.v, "bf16", torch, dev)
        abi.pa_reshape_and_cache(k_all[torch.from_numpy(hist).to(dev)].contiguous(),
                                 v_all[torch.from_numpy(hist).to(dev)].contiguous(),
                                 torch.from_numpy(slots[hist]).to(dev), kc, vc)
        nidx = torch.from_numpy(new_rows).to(dev)
        st = {"k_new": k_all[nidx].contiguous(), "v_new": v_all[nidx].contiguous(),
              "slots": torch.from_numpy(slots[new_rows]).to(dev),
              "q": to_dev(b.q, "bf16", torch, dev), "tables": torch.from_numpy(tables).to(dev),
              "lens": torch.from_numpy(b.context_lens).to(dev),
              "q_start": torch.from_numpy(qs.astype(np.int32)).to(dev),
              "max_q": int(b.meta["q_lens"].max()), "max_len": b.max_context_len,
              "scale": float(b.scale), "flops": prefill_flops(b, window)}
        st["out"] = torch.empty_like(st["q"])
        steps.append(st)
        del k_all, v_all

    def write(st):
        abi.pa_reshape_and_cache(st["k_new"], st["v_new"], st["slots"], kc, vc)

    def attend(st):
        abi.pa_prefill(st["out"], st["q"], kc, vc, st["tables"], st["lens"], st["q_start"],
                       st["max_q"], st["max_len"], st["scale"], window)

    def one_step(st):
        write(st)
        attend(st)

    V = len(steps)
    stream = torch.cuda.current_stream()
    warm = step_plan(n_warm, 0, one_step, steps, 4 * V, torch)
    timed = step_plan(n_timed, n_warm % V, one_step, steps, 4 * V, torch)
    g_att = capture(lambda: [attend(st) for st in steps], torch)
    clocks = ClockSampler(bus_id_of(torch, dev))
    clocks.start()
    time.sleep(0.3)
    time_graphs(warm, stream, torch)
    upload_graphs(timed, stream)
    torch.cuda.synchronize()
    clocks.fast_start()
    t0 = time.time()
    step_ms = time_graphs(timed, stream, torch) / n_timed
    t1 = time.time()
    clocks.fast_stop()
    reps = 50
    att_ms = time_graphs([(g_att, reps)], stream, torch) / (reps * V)
    t2 = time.time()
    clocks.stop()
    flops = float(np.mean([st["flops"] for st in steps]))
    step_flops = float(np.mean([steps[(n_warm + i) % V]["flops"] for i in range(n_timed)]))
    peak, kind = measured_bf16_sustained()
    tflops = flops / (att_ms * 1e-3) / 1e12
    tokens = float(np.mean([int(st["q"].shape[0]) for st in steps]))
    code = abi.pa_device_status()
    del steps, kc, vc, g_att, warm, timed
    torch.cuda.empty_cache()
    return {"value": round(step_flops / (step_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(step_ms, 5), "steps": n_timed, "warmup": n_warm,
            "query_tokens_per_s": round(tokens / (step_ms * 1e-3), 1),
            "config": {"workload": "Llama-3.1-8B-shaped chunked prefill", "num_seqs": 16,
                       "chunk_tokens": 512, "history": "uniform [0, 1536]",
                       "num_q_heads": 32, "num_kv_heads": 8, "head_dim": 128,
                       "block_size": 16, "window": window, "batches_rotated": V,
                       "step": "the chunk's KV write + pa_prefill"},
            "roofline": {"bound": "tensor", "kernel": "pa_prefill", "achieved": round(tflops, 2),
                         "peak": peak, "unit": "TFLOP/s", "frac": round(tflops / peak, 4),
                         "peak_kind": kind, "flops_per_launch": flops,
                         "avg_launch_ms": round(att_ms, 5),
                         "how": f"{reps} replays of a graph of {V} prefill launches",
                         "traffic": (recorded_traffic(flops, PREFILL_TRAFFIC_RECORD)
                                     if window == 0 else None)},
            "gpu_launches": 2 * n_timed, "clocks": clocks.summary(t0, t1, t2),
            "device_error_word": code}


def run_prefill(args):
    r = prefill_measure(args.pool_blocks, args.window, args.steps, max(3, args.warmup))
    r.update({"metric": "paged prefill attention TFLOP/s (causal, bf16 in, fp32 accumulate)",
              "n_gpus": 1, "higher_is_better": True, "dtype": "bf16", "data": "synthetic"})
    return r


# ---------------------------------------------------------------------- the other workloads
def _decode_measure(args, batches, torch, device, n_timed, n_warm, extra=None):
    """One decode workload on its own: the step graphs and CUDA events as for the
    headline, over n_timed steps after n_warm."""
    steps, infos = device_steps(args, batches, torch, device)
    fused = steps[0].fused
    V = len(steps)

    def one_step(s):
        s.copy()
        if not s.fused:
            s.write()
        s.append() if s.fused else s.attend()

    stream = torch.cuda.current_stream()
    warm = step_plan(n_warm, 0, one_step, steps, 4 * V, torch)
    timed = step_plan(n_timed, n_warm % V, one_step, steps, 4 * V, torch)
    g_dec = capture(lambda: [(s.append() if s.fused else s.attend()) for s in steps], torch)
    time_graphs(warm, stream, torch)
    upload_graphs(timed, stream)
    torch.cuda.synchronize()
    ms = time_graphs(timed, stream, torch) / n_timed
    reps = 50
    dec_ms = time_graphs([(g_dec, reps)], stream, torch) / (reps * V)
    peak, kind = measured_peaks()
    nbytes = float(np.mean([infos[(n_warm + i) % V]["decode"]["total"] for i in range(n_timed)]))
    kbytes = float(np.mean([i["decode"]["total"] + (i["write"] if fused else 0) for i in infos]))
    gbs = nbytes / (ms * 1e-3) / 1e9
    kgbs = kbytes / (dec_ms * 1e-3) / 1e9
    from paged_kv_cache_370_b200 import abi
    res = {"value": round(gbs, 2), "unit": "GB/s", "ms_per_step": round(ms, 5),
           "steps": n_timed, "warmup": n_warm,
           "pct_of_copy_peak": round(100 * gbs / peak, 2),
           "pct_of_hbm_nominal_8tbs": round(100 * gbs / NOMINAL_HBM_GBS, 2),
           "bytes_per_step": int(nbytes),
           "query_tokens_per_s": round(float(np.mean([len(i["lens"]) for i in infos])) /
                                       (ms * 1e-3), 1),
           "kernel": {"avg_launch_ms": round(dec_ms, 5), "achieved_gbs": round(kgbs, 2),
                      "frac": round(kgbs / peak, 4), "peak": peak, "peak_kind": kind,
                      "algorithmic_bytes_per_launch": int(kbytes)},
           "extra_bytes_per_step": {"split_scratch": int(np.mean([i["scratch"] for i in infos])),
                                    "tail_overread": int(np.mean([i["tail"] for i in infos])),
                                    "kv_write": int(infos[0]["write"]),
                                    "copy_on_write": int(infos[0].get("copy", 0))},
           "gpu_launches": int(sum(steps[(n_warm + i) % V].launches() for i in range(n_timed))),
           "device_error_word": abi.pa_device_status()}
    if "unique_kv" in infos[0]:
        u = infos[0]["unique_kv"] + (infos[0]["decode"]["total"] - infos[0]["decode"]["kv"])
        res["unique_bytes_per_step"] = int(u)
        res["logical_bytes_per_step"] = int(nbytes)
        res["unique_gbs"] = round(u / (ms * 1e-3) / 1e9, 2)
        res["pct_of_copy_peak_unique"] = round(100 * u / (ms * 1e-3) / 1e9 / peak, 2)
        res["note"] = ("logical bytes count every branch's read of the shared prompt blocks; "
                       "unique bytes count each physical block once (the prompt blocks are "
                       "read by four branches and hit in L2 after the first)")
    if extra:
        res.update(extra)
    del steps, g_dec, warm, timed
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def run_extras(args, torch, device):
    """The other workloads of the line, each measured on its own over a short run."""
    n, w = max(1, args.extra_steps), 5
    base = argparse.Namespace(**vars(args))
    base.window, base.partition_tokens = 0, 0
    out = {}

    def ns(**kw):
        a = argparse.Namespace(**vars(base))
        for k, v in kw.items():
            setattr(a, k, v)
        return a

    def guarded(name, fn):
        try:
            out[name] = fn()
        except Exception as e:  # noqa: BLE001 -- reported in the line, the headline stands
            out[name] = {"error": f"{type(e).__name__}: {e}"}
        torch.cuda.synchronize()
        torch.cuda.empty_cache()

    guarded("long_skew", lambda: _decode_measure(
        ns(workload="long_skew"), [synth.long_skew()], torch, device, n, w,
        {"config": {"workload": "long-context skew decode", "num_seqs": 8,
                    "context_lens": "uniform [8192, 32768]", "num_q_heads": 32,
                    "num_kv_heads": 8, "head_dim": 128, "block_size": 16,
                    "l2": "inputs larger than L2 (671 MB of KV per step)"}}))

    def mixed():
        rows = {}
        mb = synth.mixed_sweep(16)
        for bs in (8, 16, 32, 64, 256):
            batch = mb if bs == 16 else synth.mixed_sweep(bs, base=mb)
            r = _decode_measure(ns(workload="mixed", block_size=bs), [batch], torch, device, n, w)
            rows[str(bs)] = {k: r[k] for k in ("value", "ms_per_step", "pct_of_copy_peak",
                                                "pct_of_hbm_nominal_8tbs", "kernel",
                                                "gpu_launches", "device_error_word")}
            del batch
        return {"unit": "GB/s", "by_block_size": rows,
                "config": {"workload": "mixed serving batch", "num_seqs": 256,
                           "context_lens": "log-uniform [16, 4096]", "num_q_heads": 32,
                           "num_kv_heads": 8, "head_dim": 128,
                           "pool": "2^20 / block_size blocks (the same token capacity)",
                           "l2": "inputs larger than L2 (~770 MB of KV per step)"}}

    guarded("mixed", mixed)
    guarded("shared_prompt", lambda: _decode_measure(
        ns(workload="shared_prompt"), None, torch, device, n, w,
        {"config": {"workload": "OPT-13B-shaped shared-prompt decode with copy-on-write",
                    "num_seqs": 64, "num_q_heads": 40, "num_kv_heads": 40, "head_dim": 128,
                    "block_size": 16, "prompts": 16, "prompt_len": 512, "fork": 4}}))
    guarded("window_1024", lambda: _decode_measure(
        ns(workload="llama8b", window=1024), make_batches(ns(workload="llama8b"), 0),
        torch, device, n, w,
        {"config": {"workload": "Llama-3.1-8B-shaped decode, sliding window of 1,024 "
                                "positions (bytes: the window's positions)",
                    "batches_rotated": args.variants}}))
    guarded("prefill", lambda: prefill_measure(args.pool_blocks, 0, n, w))
    return out


# ------------------------------------------------------------------------------------- main
def main():
    args = parse_args()
    rank, world, local = dist_env()
    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, rank, world)), flush=True)
        return 0
    if args.workload in ("swap", "prefill"):
        if rank == 0:
            fn = run_swap if args.workload == "swap" else run_prefill
            print(json.dumps(fn(args)), flush=True)
        return 0
    dist = None
    if world > 1:
        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(local)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                 device_id=torch.device("cuda", local))
        dist = tdist
    try:
        res = run_ours(args, rank, world, local, dist)
        if world == 1 and not args.no_extras and args.window == 0 and \
                args.workload == "llama8b":
            import torch
            res["workloads"] = run_extras(args, torch, torch.device("cuda", local))
    finally:
        if dist is not None:
            dist.barrier()
    if rank == 0:
        print(json.dumps(res), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
