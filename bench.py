#!/usr/bin/env python
"""Benchmark: bit-exact GPU decode of entropy-coded bf16 weights.

One step = decoding every code-table scope of the workload (for the default
Llama-3-8B-shaped model: embedding, 32 transformer blocks, lm_head; 34
launches of the decode kernel, one per block, into one reused scratch
buffer).  Inputs are resident in HBM when the timed region starts.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c5]
  torchrun --nproc-per-node N bench.py --gpus N ...   (one replica per rank)
  python bench.py --impl reference ...                (the CPU oracle, timed)

Prints one JSON line on rank 0.  Multi-GPU runs are weak scaling: every rank
decodes its own resident copy of the model; there is no data-path
collective; time is the max over ranks.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import ctypes
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "decoded bf16 weights/sec & effective GB/s as % of HBM roofline; compression ratio"
FALLBACK_HBM_GBS = 6650.0
# the sources that define each decode kernel (a change to any of them makes a
# committed traffic figure stale)
_CSRC = "lossless_entropy_coded_canonical_b200/csrc/"
KERNEL_SOURCES = {
    "decode_lanes": [_CSRC + "dfw_lanes.cuh", _CSRC + "dfw_device.cuh", _CSRC + "dfw_internal.h"],
    "decode_lanes_multi": [_CSRC + "dfw_lanes.cuh", _CSRC + "dfw_device.cuh", _CSRC + "dfw_internal.h"],
    "decode_tiles": [_CSRC + "dfw_decode.cu", _CSRC + "dfw_device.cuh", _CSRC + "dfw_internal.h"],
}


# ------------------------------------------------------------------ helpers

CAP = 32  # code length cap of every encoding this run makes (--cap)


def reseed(blocks, offset: int):
    """The same workload with every tensor's recipe seed moved by offset
    (offset 0 leaves the workload's own seeds)."""
    if not offset:
        return blocks
    return [workloads.BlockSpec(b.name, [workloads.TensorSpec(t.name, t.numel, t.kind, t.seed + offset, t.std,
                                                              t.zero_frac) for t in b.tensors]) for b in blocks]


def workload_blocks(name: str):
    if name == "c5":
        return workloads.c5(), "llama3-8b-shaped model: embed + 32 blocks + lm_head, 34 code tables, N(0,0.02)"
    if name == "c4":  # the three edge-case tensors as one sequence (their own table each)
        return ([workloads.c4("a"), workloads.c4("b"), workloads.c4("c")],
                "c4: tensors 4a, 4b, 4c (3 x 67108864 weights), one code table each")
    table = {"c1": workloads.c1(), "c2": workloads.c2(), "c3": workloads.c3(), "c4a": workloads.c4("a"),
             "c4b": workloads.c4("b"), "c4bp": workloads.c4("bp"), "c4c": workloads.c4("c")}
    return [table[name]], f"{name} ({table[name].numel} weights)"


def _code_only(src: str) -> str:
    """Source text without comments and with whitespace collapsed, so that
    editing a comment does not mark a committed measurement stale (none of
    these files has // or /* inside a string literal)."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def kernel_source_hash(kernel: str = "decode_lanes") -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, p), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def closed_form(table) -> bool:
    """Whether a code table is one of the two closed forms the decoder reads in
    place (two exponents with 1-bit codes; all 256 with 8-bit codes)."""
    lens = [int(table.len[s]) for s in range(256) if table.len[s]]
    return (len(lens) == 2 and set(lens) == {1}) or (len(lens) == 256 and set(lens) == {8})


def scope_kernel(d) -> str:
    """The kernel dfw_decode_lanes runs for one scope."""
    if int(d.table.total_bits) == 0:
        return "fill_single"
    return "decode_closed" if closed_form(d.table) else "decode_lanes"


def measured_peak_hbm():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def committed_traffic(kernel: str):
    """Per-weight DRAM traffic of the decode kernel from a committed ncu
    summary, used only if it was taken on the current kernel source."""
    p = os.path.join(ROOT, "profiles", f"{kernel}_traffic.txt")
    if not os.path.exists(p):
        return None
    kv = {}
    for line in open(p):
        if ":" in line and not line.startswith("#"):
            k, v = line.split(":", 1)
            kv[k.strip()] = v.strip()
    if kv.get("kernel_source_sha256_16") != kernel_source_hash(kernel):
        return None
    try:
        return float(kv["dram_bytes_per_weight"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        self.path = None
        try:
            p = torch.cuda.get_device_properties(device)
            self.gpu_id = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
        except Exception:
            self.gpu_id = str(device)

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu_id}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        self.proc.wait(timeout=10)
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def max_over_ranks(value: float, group=None) -> float:
    """Max of a per-rank float over all ranks (identity without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    dev = "cuda" if dist.get_backend(group) == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ------------------------------------------------------------------ setup

def prepare(blocks, device, window, tile, threads, variant="window"):
    """Generates each block on the GPU and encodes it; returns the
    device-resident blocks and host copies (pinned) for the end-to-end leg.
    The known-start plan comes from the GPU encoder (the same bytes as the host
    encoder, which the tests check), so preparing the 8B-shaped model takes
    seconds and needs no host cores; the windowed plan is made on the host."""
    import lossless_entropy_coded_canonical_b200 as dfw
    if variant == "lanes":
        return prepare_on_device(blocks, device)
    host_threads = max(1, (os.cpu_count() or 8))
    enc_threads = threads or max(1, host_threads // 2)
    pool = cf.ThreadPoolExecutor(max_workers=min(8, host_threads))

    def host_side(i, tensors):
        enc = dfw.encode_multi(tensors, CAP, n_threads=enc_threads, pin=True)
        pl = dfw.plan_lanes(enc, pin=True) if variant == "lanes" else dfw.plan(enc, window, tile, pin=True)
        return i, enc, pl

    futs = []
    for i, b in enumerate(blocks):
        ts = [t.cpu() for t in workloads.generate_block(b, device)]
        futs.append(pool.submit(host_side, i, ts))
        while sum(not f.done() for f in futs) >= 8:
            time.sleep(0.01)
    res = [None] * len(blocks)
    for f in futs:
        i, enc, pl = f.result()
        res[i] = (enc, pl)
    pool.shutdown()
    up = dfw.DeviceLanes.upload if variant == "lanes" else dfw.DeviceCompressed.upload
    devs = [up(enc, pl, device) for enc, pl in res]
    torch.cuda.synchronize(device)
    torch.cuda.empty_cache()  # drop the generator's temporaries before timing
    return devs, res


def prepare_on_device(blocks, device):
    import lossless_entropy_coded_canonical_b200 as dfw
    scratch = torch.empty(dfw.encode_device_scratch_bytes(), dtype=torch.uint8, device=device)
    devs, res = [], []
    for b in blocks:
        ts = workloads.generate_block(b, device)
        sizes = [t.numel() for t in ts]
        x = torch.cat([t.reshape(-1) for t in ts]) if len(ts) > 1 else ts[0].reshape(-1)
        del ts
        dl = dfw.encode_device(x, CAP, scratch=scratch)
        del x
        offs = np.concatenate([[0], np.cumsum(sizes)]).astype(np.uint64)
        dl.tensor_offsets = offs
        pin = lambda t: torch.empty(t.shape, dtype=t.dtype, pin_memory=True).copy_(t)  # noqa: E731
        enc = dfw.Encoded(pin(dl.stream), pin(dl.mant), dl.table, offs)
        pl = dfw.LanesPlan(pin(dl.chunk_bits), pin(dl.group_start), pin(dl.lut), dl.info)
        devs.append(dl)
        res.append((enc, pl))
    torch.cuda.synchronize(device)
    torch.cuda.empty_cache()  # drop the generator's temporaries before timing
    return devs, res


def decode_one(d, scratch, stream=None):
    """One decode launch of a block into the scratch buffer (either plan)."""
    import lossless_entropy_coded_canonical_b200 as dfw
    if isinstance(d, dfw.DeviceLanes):
        dfw.decode_lanes(d, scratch, stream=stream)
    else:
        dfw.decode_block(d, scratch, stream=stream)


def verify(blocks, devs, scratch, device):
    """Decodes each block once more, with the kernel the step uses (the
    sequence kernel for the known-start plan, one scope per call), and
    compares with the regenerated input; for the known-start plan the whole
    sequence is then decoded once more and the buffer must end as the last
    scope's input."""
    import lossless_entropy_coded_canonical_b200 as dfw
    lanes = isinstance(devs[0], dfw.DeviceLanes)

    def same(b):
        off = 0
        for t in workloads.generate_block(b, device):
            if not torch.equal(scratch[off: off + t.numel()].view(torch.int16), t.view(torch.int16)):
                return False
            off += t.numel()
        return True

    for b, d in zip(blocks, devs):
        if lanes:
            dfw.decode_lanes_seq([d], scratch)
        else:
            decode_one(d, scratch)
        dfw.check()
        if not same(b):
            return False
    if lanes:
        scratch.view(torch.int16).fill_(0x5A5A)
        dfw.decode_lanes_seq(devs, scratch)
        dfw.check()
        return same(blocks[-1])
    return True


# ------------------------------------------------------------------ L2 policy

class L2Guard:
    """Whether a step's traffic is large enough that no step finds the
    previous one's data in L2.  Below 8x the L2 size, every timed step is
    preceded by a write of a buffer 4x the L2 size (outside the timed
    interval: each step is bracketed by its own CUDA events)."""
    FACTOR = 8

    def __init__(self, device, bytes_per_step: int):
        try:
            l2 = int(torch.cuda.get_device_properties(device).L2_cache_size)
        except Exception:
            l2 = 126 << 20
        self.l2 = l2
        self.bytes_per_step = int(bytes_per_step)
        self.buf = None
        if self.bytes_per_step < self.FACTOR * l2:
            self.buf = torch.empty(4 * l2, dtype=torch.uint8, device=device)

    @property
    def flushing(self) -> bool:
        return self.buf is not None

    def flush(self, stream=None):
        if self.buf is not None:
            with torch.cuda.stream(stream or torch.cuda.current_stream()):
                self.buf.zero_()

    def label(self, what: str) -> str:
        mb = self.bytes_per_step / 1e6
        if self.buf is None:
            return (f"inputs larger than L2: each step moves {mb:.0f} MB ({what}), "
                    f"over {self.FACTOR}x the {self.l2 >> 20} MB L2; no reuse between steps")
        return (f"L2 flushed before every timed step (a {self.buf.numel() >> 20} MB write, outside the step's own "
                f"CUDA events): a step moves only {mb:.0f} MB ({what}) against the {self.l2 >> 20} MB L2")


def timed_steps(fn, steps: int, stream, guard: L2Guard | None = None, per_step: list | None = None) -> float:
    """Device time of ``steps`` calls of fn on ``stream`` (ms, total): CUDA
    events between consecutive calls (the total spans all of them), or, when
    the guard flushes L2, a pair around each call with the flush in between.
    ``per_step``, if a list, receives each call's own time (ms)."""
    barrier()
    torch.cuda.synchronize()
    if guard is None or not guard.flushing:
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        ev[0].record(stream)
        for i in range(steps):
            fn()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
        barrier()
        if per_step is not None:
            per_step.extend(ev[i].elapsed_time(ev[i + 1]) for i in range(steps))
        return ev[0].elapsed_time(ev[-1])
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in ev:
        guard.flush(stream)
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    barrier()
    if per_step is not None:
        per_step.extend(a.elapsed_time(b) for a, b in ev)
    return sum(a.elapsed_time(b) for a, b in ev)


def step_stats(per_step: list) -> dict | None:
    """Median, best and worst of the timed steps (ms, this rank's own)."""
    if not per_step:
        return None
    a = np.array(per_step, dtype=np.float64)
    return {"median": float(np.median(a)), "best": float(a.min()), "worst": float(a.max()), "steps": int(a.size)}


# ------------------------------------------------------------------ timed arms

def run_device(devs, scratch, steps, warmup, stream, guard: L2Guard | None = None):
    """Every scope launched on its own with CUDA events around each launch
    (the kernel's roofline figure); with an L2 guard that flushes, L2 is
    flushed before every launch, outside its events."""
    import lossless_entropy_coded_canonical_b200 as dfw
    for _ in range(warmup):
        for d in devs:
            decode_one(d, scratch, stream)
    dfw.check(stream)
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in devs]
          for _ in range(steps)]
    barrier()
    torch.cuda.synchronize()
    for s in range(steps):
        for j, d in enumerate(devs):
            if guard is not None:
                guard.flush(stream)
            ev[s][j][0].record(stream)
            decode_one(d, scratch, stream)
            ev[s][j][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    per_launch = [[a.elapsed_time(b) for a, b in row] for row in ev]
    total_ms = float(np.sum(per_launch))
    status = dfw.check_status(stream)
    return total_ms, per_launch, status


def run_device_seq(devs, scratch, steps, warmup, stream, graph=False, guard: L2Guard | None = None,
                   per_step: list | None = None):
    """The step as one dfw_decode_lanes_seq call over every scope: the same
    launches in the same order into the same scratch buffer, each one a
    programmatic dependent of the one before (it may start while the previous
    drains and stores only after it completes).  With ``graph`` the call is
    captured once into a CUDA graph and each step replays it."""
    import lossless_entropy_coded_canonical_b200 as dfw
    for _ in range(warmup):
        dfw.decode_lanes_seq(devs, scratch, stream=stream)
    dfw.check(stream)
    g = None
    if graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            dfw.decode_lanes_seq(devs, scratch)
        for _ in range(warmup):
            g.replay()
        torch.cuda.synchronize()

    def step():
        if g is not None:
            g.replay()
        else:
            dfw.decode_lanes_seq(devs, scratch, stream=stream)

    total = timed_steps(step, steps, stream, guard, per_step)
    del g
    return total, dfw.check_status(stream)


def run_e2e(results, devs, device, steps, stream):
    """Same metric through the public API from pinned host buffers: per block
    H2D of its compressed form, decode, D2H of the decoded weights; copies run
    on their own streams, double-buffered so they overlap the decode."""
    import lossless_entropy_coded_canonical_b200 as dfw
    nmax = max(d.n for d in devs)
    lanes = isinstance(results[0][1], dfw.LanesPlan)
    aux_names = ("chunk_bits", "group_start", "lut") if lanes else ("gap", "out_start", "lut")
    h2d_s, d2h_s = torch.cuda.Stream(device), torch.cuda.Stream(device)
    slots = []
    for _ in range(2):
        sl = {"stream": torch.empty(max(int(e.table.stream_bytes) for e, _ in results), dtype=torch.uint8, device=device),
              "mant": torch.empty(max(e.mant.numel() for e, _ in results), dtype=torch.uint8, device=device),
              "scratch": torch.empty(nmax, dtype=torch.bfloat16, device=device),
              "host_out": torch.empty(nmax, dtype=torch.bfloat16, pin_memory=True),
              "loaded": torch.cuda.Event(), "decoded": torch.cuda.Event(), "drained": torch.cuda.Event()}
        for a in aux_names:
            t0 = getattr(results[0][1], a)
            sl[a] = torch.empty(max(getattr(p, a).numel() for _, p in results), dtype=t0.dtype, device=device)
        slots.append(sl)
    h2d = sum(int(e.table.stream_bytes) + e.mant.numel() + sum(getattr(p, a).numel() * getattr(p, a).element_size()
                                                                for a in aux_names) for e, p in results)
    d2h = sum(2 * e.n for e, _ in results)

    def one_step():
        # slot i % 2 is reused by block i + 2: its H2D waits until block i's
        # decode has read the inputs, and its decode waits until block i's
        # D2H has read the scratch buffer
        for i, (enc, pl) in enumerate(results):
            sl = slots[i % 2]
            h2d_s.wait_event(sl["decoded"])
            with torch.cuda.stream(h2d_s):
                sl["stream"][: enc.stream.numel()].copy_(enc.stream, non_blocking=True)
                sl["mant"][: enc.mant.numel()].copy_(enc.mant, non_blocking=True)
                for a in aux_names:
                    src = getattr(pl, a)
                    sl[a][: src.numel()].copy_(src, non_blocking=True)
                sl["loaded"].record(h2d_s)
            stream.wait_event(sl["loaded"])
            stream.wait_event(sl["drained"])
            if lanes:
                dc = dfw.DeviceLanes(sl["stream"], sl["mant"], sl["lut"], sl["chunk_bits"], sl["group_start"],
                                     enc.table, pl.info, enc.tensor_offsets)
            else:
                dc = dfw.DeviceCompressed(sl["stream"], sl["mant"], sl["lut"], sl["gap"], sl["out_start"], enc.table,
                                          pl.info, enc.tensor_offsets)
            decode_one(dc, sl["scratch"], stream)
            sl["decoded"].record(stream)
            d2h_s.wait_event(sl["decoded"])
            with torch.cuda.stream(d2h_s):
                sl["host_out"][: enc.n].copy_(sl["scratch"][: enc.n], non_blocking=True)
                sl["drained"].record(d2h_s)

    one_step()  # warm-up (allocator, first copies)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    t0.record(stream)
    for _ in range(steps):
        one_step()
    stream.wait_stream(d2h_s)
    stream.wait_stream(h2d_s)
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    st = dfw.check_status(stream)
    return t0.elapsed_time(t1) / steps, h2d, d2h, st


def host_cpu() -> dict:
    """The host's CPU model and the cores this process may run on."""
    model = ""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        usable = len(os.sched_getaffinity(0))
    except AttributeError:
        usable = os.cpu_count() or 1
    return {"model": model or "unknown", "nproc": usable, "logical_cpus": os.cpu_count()}


def _sample_scope(blocks):
    """The scope the single-core sample is drawn from: the first transformer
    block of the 34-scope model, else the workload's only scope."""
    return blocks[1] if len(blocks) > 1 else blocks[0]


def cpu_sample(block, sample_weights: int) -> np.ndarray:
    """The first ``sample_weights`` weights of a scope (its tensors in order),
    drawn on the host with each tensor's own recipe and seed.  Tensors whose
    exponent counts depend on their size (the geometric and Fibonacci bit
    patterns) are drawn whole and cut; the others are drawn at the size taken."""
    parts, got = [], 0
    for t in block.tensors:
        take = min(t.numel, sample_weights - got)
        if take <= 0:
            break
        whole = t.kind in ("geometric", "fibonacci")
        spec = workloads.TensorSpec(t.name, t.numel if whole else take, t.kind, t.seed, t.std, t.zero_frac)
        parts.append(workloads.as_u16_numpy(workloads.generate(spec, "cpu"))[:take])
        got += take
    return np.concatenate(parts)


def cpu_baseline_sample(blocks, sample_weights: int, reps: int):
    """The oracle's bit-serial decoder, as it stands, on one host thread, on
    a prefix of the workload (the oracle encodes it, untimed).  Returns
    (weights, median seconds, the oracle's encoding, the input)."""
    import oracle
    oracle.build()
    u = cpu_sample(_sample_scope(blocks), sample_weights)
    enc = oracle.encode(u)
    times = []
    for _ in range(reps):
        t0 = time.perf_counter()
        out = oracle.decode(enc)
        times.append(time.perf_counter() - t0)
    assert np.array_equal(out, u)
    return u.size, statistics.median(times), enc, u


def cpu_baseline_all_cores(blocks, per_scope: int, reps: int):
    """The same oracle decoder on every host core, over independent streams:
    one sample of ``per_scope`` weights from each code-table scope of the
    workload (the 34 scopes of the 8B-shaped model), each encoded on its own
    and decoded concurrently by a thread pool of one thread per core (the
    oracle is C called through ctypes, which releases the interpreter lock).
    Returns (weights, median wall seconds, threads, scopes)."""
    import oracle
    oracle.build()
    threads = host_cpu()["nproc"]
    us = [cpu_sample(b, per_scope) for b in blocks]
    encs = [oracle.encode(u) for u in us]
    with cf.ThreadPoolExecutor(threads) as ex:
        list(ex.map(oracle.decode, encs))  # warm the pool
        times = []
        for _ in range(reps):
            t0 = time.perf_counter()
            outs = list(ex.map(oracle.decode, encs))
            times.append(time.perf_counter() - t0)
    assert all(np.array_equal(o, u) for o, u in zip(outs, us))
    return sum(u.size for u in us), statistics.median(times), threads, len(us)


# ------------------------------------------------------------------ encode mode

def run_encode_mode(args, rank, world, blocks, wdesc, device):
    """Times the GPU encoder over every scope of the workload, from bf16
    already resident on the device, into preallocated outputs: one
    dfw_encode_device_multi call for all scopes (the host builds scope i's
    code while the GPU runs scope i + 1's histogram pass), then
    dfw_pack_device per scope; ``--encode-api single`` times
    dfw_encode_device + dfw_pack_device scope by scope instead.  The time
    includes the host synchronisations and the host-side code construction."""
    import ctypes
    import lossless_entropy_coded_canonical_b200 as dfw
    lib = dfw.lib()
    stream = torch.cuda.current_stream(device)
    sh = ctypes.c_void_p(stream.cuda_stream)
    scopes = []
    for b in blocks:
        x = torch.cat([t.reshape(-1) for t in workloads.generate_block(b, device)])
        n = x.numel()
        groups = -(-(-(-n // 64)) // 32)
        scopes.append({"x": x, "n": n, "mant": torch.empty(dfw.mant_bytes(n), dtype=torch.uint8, device=device),
                       "cb": torch.empty(32 * groups, dtype=torch.int16, device=device),
                       "gs": torch.empty(groups + 1, dtype=torch.int64, device=device),
                       "table": dfw.Table(), "info": dfw.LanesInfo(), "stream": None})
    scratch = torch.empty(int(lib.dfw_encode_device_scratch_bytes(0)), dtype=torch.uint8, device=device)
    torch.cuda.synchronize(device)
    torch.cuda.empty_cache()

    def encode_scope(sc):
        dfw._check(lib.dfw_encode_device(sc["x"].data_ptr(), sc["n"], CAP, sc["mant"].data_ptr(), sc["cb"].data_ptr(),
                                         sc["gs"].data_ptr(), scratch.data_ptr(), scratch.numel(),
                                         ctypes.byref(sc["table"]), ctypes.byref(sc["info"]), sh), "dfw_encode_device")
        if sc["stream"] is None:  # sized by the first (warm-up) encode; the data do not change
            sc["stream"] = torch.empty(int(sc["table"].stream_bytes), dtype=torch.uint8, device=device)
        dfw._check(lib.dfw_pack_device(sc["x"].data_ptr(), ctypes.byref(sc["table"]), ctypes.byref(sc["info"]),
                                       sc["gs"].data_ptr(), sc["stream"].data_ptr(), sc["stream"].numel(), sh),
                   "dfw_pack_device")

    k = len(scopes)
    mscratch = torch.empty(k * int(lib.dfw_encode_device_scratch_bytes(0)), dtype=torch.uint8, device=device)
    staging = torch.empty(int(lib.dfw_encode_device_multi_staging_bytes(k)), dtype=torch.uint8, pin_memory=True)
    arr = (dfw.EncodeScope * k)()
    for i, sc in enumerate(scopes):
        arr[i] = dfw.EncodeScope(sc["x"].data_ptr(), sc["n"], sc["mant"].data_ptr(), sc["cb"].data_ptr(),
                                 sc["gs"].data_ptr())
    tables, infos = (dfw.Table * k)(), (dfw.LanesInfo * k)()

    def encode_step():
        if args.encode_api == "single":
            for sc in scopes:
                encode_scope(sc)
            return
        dfw._check(lib.dfw_encode_device_multi(k, arr, CAP, mscratch.data_ptr(), mscratch.numel(), staging.data_ptr(),
                                               staging.numel(), tables, infos, sh), "dfw_encode_device_multi")
        for i, sc in enumerate(scopes):
            sc["table"], sc["info"] = tables[i], infos[i]
            if sc["stream"] is None:
                sc["stream"] = torch.empty(int(sc["table"].stream_bytes), dtype=torch.uint8, device=device)
            dfw._check(lib.dfw_pack_device(sc["x"].data_ptr(), ctypes.byref(sc["table"]), ctypes.byref(sc["info"]),
                                           sc["gs"].data_ptr(), sc["stream"].data_ptr(), sc["stream"].numel(), sh),
                       "dfw_pack_device")

    for _ in range(args.warmup):
        encode_step()
    torch.cuda.synchronize(device)
    alg = sum(2 * sc["n"] + sc["mant"].numel() + int(sc["table"].stream_bytes) + 2 * sc["cb"].numel()
              + 8 * sc["gs"].numel() for sc in scopes)
    guard = L2Guard(device, alg)
    sampler = ClockSampler(int(device.index or 0))
    sampler.start()
    ms_step = max_over_ranks(timed_steps(encode_step, args.steps, stream, guard) / args.steps)
    clocks = sampler.stop()

    # round trip on the device: every scope decodes back to its input
    ok = True
    out = torch.empty(max(sc["n"] for sc in scopes), dtype=torch.bfloat16, device=device)
    for sc in scopes:
        lut = torch.empty(int(sc["info"].lut_words), dtype=torch.int32)
        dfw._check(lib.dfw_lanes_lut(ctypes.byref(sc["table"]), ctypes.byref(sc["info"]), lut.data_ptr()),
                   "dfw_lanes_lut")
        dl = dfw.DeviceLanes(sc["stream"], sc["mant"], lut.to(device), sc["cb"], sc["gs"], sc["table"], sc["info"])
        dfw.decode_lanes(dl, out)
        ok = ok and dfw.check_status() == dfw.OK and torch.equal(out[: sc["n"]].view(torch.int16),
                                                                   sc["x"].view(torch.int16))
    n_total = sum(sc["n"] for sc in scopes)
    peak, peak_kind = measured_peak_hbm()
    achieved = alg / (ms_step * 1e-3) / 1e9
    line = {
        "metric": "encoded bf16 weights/sec (GPU encoder, bit-exact with the host encoder and the oracle)",
        "value": world * n_total / (ms_step * 1e-3), "unit": "weights/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u8", "data": "synthetic",
        "config": {"workload": wdesc, "weights": n_total, "code_tables": len(scopes), "mode": "encode",
                   "l2": guard.label("every scope's bf16 read three times, raw bytes and stream written"),
                   "encode_api": args.encode_api,
                   "parallelism": f"replica{world}" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": None, "peak_source": peak_kind, "kernel": "encoder (6 kernels per scope, host code construction)",
                     "algorithmic_bytes_per_step": alg, "mean_scope_ms": ms_step / k},
        "clocks": clocks, "gpu_launches": args.steps * k * 6, "verified_roundtrip": bool(ok),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0 if ok else 1


# ------------------------------------------------------------------ gemv mode

def run_gemv_mode(args, rank, world, blocks, wdesc, device):
    """Times decode fused with y = W x (``dfw_decode_gemv_lanes``) over every
    scope of the workload (each tensor read as a row-major [out, in] matrix,
    the embedding as a tied 128256 x 4096 output matrix), against decode into
    the scratch buffer followed by cuBLAS's bf16 matrix-vector product on the
    same inputs, timed in the same run."""
    import lossless_entropy_coded_canonical_b200 as dfw
    devs, _ = prepare(blocks, device, args.window, args.tile, args.threads, "lanes")
    gen = torch.Generator(device=device).manual_seed(77)
    work = []
    for b, d in zip(blocks, devs):
        cols = [workloads.matrix_cols(t) for t in b.tensors]
        xs = [torch.randn(c, generator=gen, device=device).to(torch.bfloat16) for c in cols]
        offs = [int(v) for v in d.tensor_offsets]
        ys = [torch.empty((offs[i + 1] - offs[i]) // cols[i], dtype=torch.float32, device=device)
              for i in range(len(cols))]
        work.append((d, cols, xs, ys, offs))
    nmax = max(d.n for d in devs)
    partial = torch.empty(nmax // 64 + 1, dtype=torch.float32, device=device)
    scratch = torch.empty(nmax, dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(device)

    def fused():
        for d, cols, xs, ys, _ in work:
            dfw.decode_gemv_lanes(d, xs, cols, ys=ys, partial=partial, stream=stream)

    def unfused():
        for d, cols, xs, ys, offs in work:
            dfw.decode_lanes(d, scratch, stream=stream)
            for i, c in enumerate(cols):
                w = scratch[offs[i]: offs[i + 1]].view(-1, c)
                torch.mv(w, xs[i])

    n_total = sum(d.n for d in devs)
    alg = sum(int(d.table.stream_bytes) + d.n + 2 * d.chunk_bits.numel() + 8 * d.group_start.numel()
              + 4 * d.lut.numel() + 8 * (d.n // 64) + sum(2 * c for c in cols) + 4 * sum(y.numel() for y in ys)
              for d, cols, _, ys, _ in work)
    guard = L2Guard(device, alg)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(device)
        return max_over_ranks(timed_steps(fn, args.steps, stream, guard) / args.steps)

    sampler = ClockSampler(int(device.index or 0))
    sampler.start()
    ms_fused = timed(fused)
    clocks = sampler.stop()
    ms_unfused = timed(unfused)
    ok = dfw.check_status(stream) == dfw.OK
    # every y against fp64 of the decoded weights (decode_lanes is bit-exact
    # by its own tests) within the fp32 summation bound
    fused()
    for d, cols, xs, ys, offs in work:
        dfw.decode_lanes(d, scratch, stream=stream)
        for i, c in enumerate(cols):
            w = scratch[offs[i]: offs[i + 1]].view(-1, c).double()
            x = xs[i].double()
            want, scale = w @ x, w.abs() @ x.abs()
            gamma = c * 2.0 ** -24 / (1 - c * 2.0 ** -24)
            ok = ok and bool(((ys[i].double() - want).abs() <= gamma * scale + 1e-30).all())
    peak, peak_kind = measured_peak_hbm()
    achieved = alg / (ms_fused * 1e-3) / 1e9
    line = {
        "metric": "weights/s through decode fused with y = W x (bf16 x, fp32 y; weights never written)",
        "value": world * n_total / (ms_fused * 1e-3), "unit": "weights/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_fused, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u8+bf16->fp32", "data": "synthetic",
        "config": {"workload": wdesc, "weights": n_total, "code_tables": len(devs), "mode": "gemv",
                   "l2": guard.label("every scope's compressed form and x read, partials and y written"),
                   "parallelism": f"replica{world}" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": None, "peak_source": peak_kind, "kernel": "decode_lanes<DotEpi> + gemv_rows",
                     "algorithmic_bytes_per_step": alg},
        "unfused": {"ms_per_step": ms_unfused, "what": "decode_lanes into scratch, then torch.mv (cuBLAS, bf16)",
                    "speedup_of_fused": ms_unfused / ms_fused},
        "clocks": clocks, "gpu_launches": args.steps * 2 * len(devs), "verified_within_fp32_bound": bool(ok),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0 if ok else 1


# ------------------------------------------------------------------ rans mode

def run_rans_mode(args, rank, world, blocks, wdesc, device):
    """The rANS variant against the Huffman known-start plan on the same
    weights, in the same run: compressed size (with and without aux) and
    decode time of every scope into the scratch buffer."""
    import lossless_entropy_coded_canonical_b200 as dfw
    devs_h, _ = prepare(blocks, device, args.window, args.tile, args.threads, "lanes")
    devs_r = []
    for b in blocks:
        ts = [t.cpu() for t in workloads.generate_block(b, device)]
        devs_r.append(dfw.DeviceRans.upload(dfw.rans_encode(ts), device))
    torch.cuda.synchronize(device)
    torch.cuda.empty_cache()
    nmax = max(d.n for d in devs_h)
    scratch = torch.empty(nmax, dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(device)

    guard = L2Guard(device, sum(d.algorithmic_bytes() for d in devs_r))

    def timed(step):
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize(device)
        return max_over_ranks(timed_steps(step, args.steps, stream, guard) / args.steps)

    sampler = ClockSampler(int(device.index or 0))
    sampler.start()
    ms_r = timed(lambda: [dfw.rans_decode(d, scratch, stream=stream) for d in devs_r])
    clocks = sampler.stop()
    ms_h = timed(lambda: [dfw.decode_lanes(d, scratch, stream=stream) for d in devs_h])
    ok = dfw.check_status(stream) == dfw.OK
    for b, d in zip(blocks, devs_r):  # every scope decodes back to its input
        dfw.rans_decode(d, scratch, stream=stream)
        ref = torch.cat([t.reshape(-1) for t in workloads.generate_block(b, device)])
        ok = ok and dfw.check_status(stream) == dfw.OK and torch.equal(scratch[: d.n].view(torch.int16),
                                                                      ref.view(torch.int16))
    n_total = sum(d.n for d in devs_r)
    bits = lambda devs, aux: 8 * sum(d.compressed_bytes(with_aux=aux) for d in devs) / n_total  # noqa: E731
    alg = sum(d.algorithmic_bytes() for d in devs_r)
    peak, peak_kind = measured_peak_hbm()
    achieved = alg / (ms_r * 1e-3) / 1e9
    line = {
        "metric": "decoded bf16 weights/sec with the rANS variant (beside the Huffman plan on the same weights)",
        "value": world * n_total / (ms_r * 1e-3), "unit": "weights/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_r, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u8", "data": "synthetic",
        "config": {"workload": wdesc, "weights": n_total, "code_tables": len(devs_r), "mode": "rans",
                   "rans": "2^12 frequencies, 32 interleaved 32-bit states, blocks of 16384",
                   "l2": guard.label("every scope's rANS stream and raw bytes read, its bf16 written"),
                   "parallelism": f"replica{world}" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": None, "peak_source": peak_kind, "kernel": "rans_decode_kernel",
                     "algorithmic_bytes_per_step": alg},
        "rate_bits_per_weight": {"rans": bits(devs_r, True), "rans_no_aux": bits(devs_r, False),
                                 "huffman_lanes": bits(devs_h, True), "huffman_no_aux": bits(devs_h, False)},
        "huffman_lanes_ms_per_step": ms_h,
        "clocks": clocks, "gpu_launches": args.steps * len(devs_r), "verified_bit_exact": bool(ok),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0 if ok else 1


# ------------------------------------------------------------------ launch-cost mode

def run_launch_cost_mode(args, rank, world, device):
    """Decode time against size: one N(0, 0.02) tensor of 1, 2, ..., 32
    groups (2048 weights) per resident warp, each size timed with CUDA events
    around single launches; a least-squares line gives the per-launch fixed
    cost (intercept) and the per-group cost (slope)."""
    import lossless_entropy_coded_canonical_b200 as dfw
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    warps = sms * 32
    rows = []
    for k in (1, 2, 4, 8, 16, 32):
        n = warps * 2048 * k
        spec = workloads.BlockSpec("launch_cost", [workloads.TensorSpec("w", n, "normal", 77, 0.02)])
        ref = workloads.generate_block(spec, device)[0]
        enc = dfw.encode_multi([ref.cpu()], 32)
        dl = dfw.DeviceLanes.upload(enc, dfw.plan_lanes(enc), device)
        out = torch.empty(n, dtype=torch.bfloat16, device=device)
        for _ in range(args.warmup):
            dfw.decode_lanes(dl, out)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        torch.cuda.synchronize()
        for a, b in ev:
            a.record()
            dfw.decode_lanes(dl, out)
            b.record()
        torch.cuda.synchronize()
        ms = sorted(a.elapsed_time(b) for a, b in ev)
        exact = bool(torch.equal(out.view(torch.int16), ref.view(torch.int16)))
        rows.append({"groups_per_warp": k, "weights": n, "median_ms": ms[len(ms) // 2], "bit_exact": exact})
        del dl, out, ref
    ks = np.array([r["groups_per_warp"] for r in rows], float)
    ts = np.array([r["median_ms"] for r in rows])
    slope, icpt = np.linalg.lstsq(np.vstack([ks, np.ones_like(ks)]).T, ts, rcond=None)[0]
    if rank == 0:
        print(json.dumps({"mode": "launch-cost", "resident_warps": warps, "sizes": rows,
                          "fixed_ms_per_launch": float(icpt), "ms_per_group_per_warp": float(slope),
                          "verified_bit_exact": all(r["bit_exact"] for r in rows)}), flush=True)
    return 0 if all(r["bit_exact"] for r in rows) else 1


# ------------------------------------------------------------------ seq-cost mode

def run_seq_cost_mode(args, rank, world, device):
    """Cost of a scope inside a sequence: one Llama-3-8B-shaped transformer
    block decoded k = 1, 2, 4, 8, 16 times in one dfw_decode_lanes_seq call
    (the same resident scope repeated), CUDA events around each call; a
    least-squares line gives the fixed cost per call (intercept) and the
    cost per scope (slope), beside the same block decoded alone by
    dfw_decode_lanes (CUDA events around each launch)."""
    import lossless_entropy_coded_canonical_b200 as dfw
    blk = workloads.c5()[1]
    devs, _ = prepare_on_device([blk], device)
    d = devs[0]
    out = torch.empty(d.n, dtype=torch.bfloat16, device=device)
    rows = []
    for k in (1, 2, 4, 8, 16):
        seq = [d] * k
        for _ in range(args.warmup):
            dfw.decode_lanes_seq(seq, out)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        torch.cuda.synchronize()
        for a, b in ev:
            a.record()
            dfw.decode_lanes_seq(seq, out)
            b.record()
        torch.cuda.synchronize()
        ms = sorted(a.elapsed_time(b) for a, b in ev)
        rows.append({"scopes": k, "launches": dfw.decode_lanes_seq_launches(seq), "median_ms": ms[len(ms) // 2]})
    for _ in range(args.warmup):
        dfw.decode_lanes(d, out)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize()
    for a, b in ev:
        a.record()
        dfw.decode_lanes(d, out)
        b.record()
    torch.cuda.synchronize()
    single = sorted(a.elapsed_time(b) for a, b in ev)[args.steps // 2]
    ok = dfw.check_status() == dfw.OK and torch.equal(
        out.view(torch.int16), torch.cat([t.reshape(-1) for t in workloads.generate_block(blk, device)]).view(torch.int16))
    ks = np.array([r["scopes"] for r in rows], float)
    ts = np.array([r["median_ms"] for r in rows])
    slope, icpt = np.linalg.lstsq(np.vstack([ks, np.ones_like(ks)]).T, ts, rcond=None)[0]
    if rank == 0:
        print(json.dumps({"mode": "seq-cost", "scope": "llama3-8b-shaped transformer block (218103808 weights)",
                          "sizes": rows, "fixed_ms_per_call": float(icpt), "ms_per_scope": float(slope),
                          "single_launch_ms": single, "verified_bit_exact": bool(ok)}), flush=True)
    return 0 if ok else 1


# ------------------------------------------------------------------ main

def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="dfw", choices=["dfw", "reference"])
    ap.add_argument("--workload", default="c5")
    ap.add_argument("--window", type=int, default=8)
    ap.add_argument("--tile", type=int, default=256)
    ap.add_argument("--variant", default="lanes", choices=["window", "lanes"],
                    help="window: gap/out_start plan (count phase + scan); lanes: known-start chunks")
    ap.add_argument("--threads", type=int, default=0)
    ap.add_argument("--cap", type=int, default=32, help="code length cap of the encoding, 1..32")
    ap.add_argument("--seed", type=int, default=0,
                    help="offset added to every tensor's recipe seed (0: the workload's own seeds)")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--cpu-sample", type=int, default=32 * 1024 * 1024)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--graph", action="store_true",
                    help="decode step: capture the sequence once in a CUDA graph and replay it each step")
    ap.add_argument("--encode-api", default="multi", choices=["multi", "single"],
                    help="encode mode: one dfw_encode_device_multi call for all scopes, or dfw_encode_device each")
    ap.add_argument("--mode", default="decode", choices=["decode", "encode", "gemv", "rans", "launch-cost",
                                                         "seq-cost"],
                    help="decode: the decode path (default); encode: the GPU encoder; "
                         "gemv: decode fused with y = W x; rans: the rANS variant beside Huffman; "
                         "launch-cost: decode time against size (fixed cost per launch); "
                         "seq-cost: cost of a scope inside a sequence")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not 1 <= args.cap <= 32:
        ap.error("--cap must be in 1..32")
    global CAP
    CAP = args.cap
    blocks, wdesc = workload_blocks(args.workload)
    blocks = reseed(blocks, args.seed)
    if args.cap != 32 or args.seed:
        wdesc += f", cap {args.cap}, seed offset {args.seed}"
    n_total = sum(b.numel for b in blocks)

    if args.impl == "reference":
        return reference_arm(args, rank, world, blocks, n_total, wdesc)

    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=__import__("datetime").timedelta(seconds=600))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    import lossless_entropy_coded_canonical_b200 as dfw
    dfw.lib()
    dfw.check()
    if args.mode == "launch-cost":
        return run_launch_cost_mode(args, rank, world, device)
    if args.mode == "seq-cost":
        return run_seq_cost_mode(args, rank, world, device)
    if args.mode in ("encode", "gemv", "rans"):
        run = {"encode": run_encode_mode, "gemv": run_gemv_mode, "rans": run_rans_mode}[args.mode]
        rc = run(args, rank, world, blocks, wdesc, device)
        if world > 1:
            dist.destroy_process_group()
        return rc

    devs, results = prepare(blocks, device, args.window, args.tile, args.threads, args.variant)
    nmax = max(d.n for d in devs)
    scratch = torch.empty(nmax, dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(device)
    comp = sum(d.compressed_bytes(with_aux=True) for d in devs)
    comp_noaux = sum(d.compressed_bytes(with_aux=False) for d in devs)
    alg_bytes = sum(d.algorithmic_bytes() for d in devs)

    lanes = args.variant == "lanes"
    guard = L2Guard(device, alg_bytes)
    sampler = ClockSampler(local)
    per_step = []
    sampler.start()
    if lanes:  # the step: one sequence of launches over every scope
        total_ms, status = run_device_seq(devs, scratch, args.steps, args.warmup, stream, args.graph, guard,
                                          per_step)
    else:
        total_ms, per_launch, status = run_device(devs, scratch, args.steps, args.warmup, stream, guard)
    clocks = sampler.stop()
    ms_step = max_over_ranks(total_ms / args.steps)
    per_launch_step_ms = None
    if lanes:  # the kernel's roofline: the same launches one by one, each bracketed by CUDA events
        pl_ms, per_launch, st_pl = run_device(devs, scratch, args.steps, 3, stream, guard)
        per_launch_step_ms = max_over_ranks(pl_ms / args.steps)
        status = status if status != dfw.OK else st_pl
    ok = status == dfw.OK and verify(blocks, devs, scratch, device)

    # roofline of the step's kernel: algorithmic bytes per launch / mean
    # launch duration.  Known-start plan: the step is dfw_decode_lanes_seq,
    # one persistent launch per run of scopes (one for the whole 8B-shaped
    # model), timed by the CUDA events around each step; the per-scope kernel
    # launched one by one is reported beside it.  Windowed plan: one launch
    # per scope, events around each.
    launch_ms = np.array(per_launch)  # [steps, blocks]
    mean_launch_ms = launch_ms.mean(axis=0)
    per_scope_achieved = alg_bytes / (mean_launch_ms.sum() * 1e-3) / 1e9
    peak, peak_kind = measured_peak_hbm()
    if lanes:
        seq_launches = dfw.decode_lanes_seq_launches(devs)
        # a sequence of one scope runs the one-scope kernel (the closed-form
        # kernel for a scope whose code is a bitmap or the 8-bit identity)
        kernel = "decode_lanes_multi" if len(devs) > 1 else scope_kernel(devs[0])
        achieved = alg_bytes / (ms_step * 1e-3) / 1e9
        launches_per_step = seq_launches
        mean_kernel_ms = ms_step / seq_launches
        weights_per_launch = n_total / seq_launches
    else:
        kernel = "decode_tiles"
        achieved = per_scope_achieved
        launches_per_step = len(devs)
        mean_kernel_ms = float(mean_launch_ms.mean())
        weights_per_launch = n_total / len(devs)
    tpw = committed_traffic(kernel)
    traffic = None if tpw is None else tpw * weights_per_launch

    e2e = None
    if not args.no_e2e:
        e2e_ms, h2d, d2h, st2 = run_e2e(results, devs, device, args.e2e_steps, stream)
        e2e_ms = max_over_ranks(e2e_ms)
        ok = ok and st2 == dfw.OK
        e2e = {"value": world * n_total / (e2e_ms * 1e-3), "unit": "weights/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n_s, sec, _, _ = cpu_baseline_sample(blocks, args.cpu_sample, 3)
        scope = _sample_scope(blocks)
        cpu = {"value": n_s / sec, "unit": "weights/s", "cores": 1, "kind": "oracle",
               "sample": f"bit-serial decode of the first {n_s} weights of scope {scope.name} "
                         f"({', '.join(t.name for t in scope.tensors)}), median of 3, one host thread",
               "cpu": host_cpu()}
        if len(blocks) > 1:  # independent streams: the scopes
            per = max(1, args.cpu_sample // 8)
            n_a, sec_a, thr, k = cpu_baseline_all_cores(blocks, per, 3)
            cpu["all_cores"] = {"value": n_a / sec_a, "unit": "weights/s", "cores": thr,
                                "sample": f"{per} weights from each of the {k} code-table scopes, each encoded "
                                          f"on its own, decoded concurrently on {thr} threads, median of 3 "
                                          f"wall times"}

    value = world * n_total / (ms_step * 1e-3)
    eff_gbs = alg_bytes / (ms_step * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "weights/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u8", "data": "synthetic",
        "config": {"workload": wdesc, "weights": n_total, "code_tables": len(devs), "plan": args.variant,
                   "cap": CAP, "seed_offset": args.seed,
                   "window_bytes": args.window if args.variant == "window" else None,
                   "tile_windows": args.tile if args.variant == "window" else None,
                   "l2": guard.label("every scope's compressed form read, its bf16 written"),
                   "parallelism": f"replica{world}" if world > 1 else "single GPU",
                   "launch": ("one dfw_decode_lanes_seq per step: one persistent launch per run of up to 40 "
                              "scopes" + (", captured once in a CUDA graph and replayed" if args.graph else "")
                              if lanes else "one dfw_decode_block per scope")},
        "step_ms": step_stats(per_step),
        "effective_gbs": eff_gbs, "hbm_frac": eff_gbs / peak,
        "compression_ratio": 2 * n_total / comp, "compression_ratio_no_aux": 2 * n_total / comp_noaux,
        "bits_per_weight": 8 * comp / n_total,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic, "peak_source": peak_kind,
                     "kernel": kernel,
                     "algorithmic_bytes_per_step": alg_bytes,
                     "launches_per_step": launches_per_step,
                     "mean_launch_ms": mean_kernel_ms,
                     "timing": ("CUDA events around each timed step (the step is the kernel's launches)" if lanes
                                else "per-launch CUDA events around each scope's launch, launched one by one"),
                     "per_scope_kernel": ({"kernel": " + ".join(sorted({scope_kernel(d) for d in devs})),
                                           "achieved": per_scope_achieved,
                                           "frac": per_scope_achieved / peak,
                                           "mean_launch_ms": float(mean_launch_ms.mean()),
                                           "one_by_one_ms_per_step": per_launch_step_ms,
                                           "timing": "CUDA events around each scope's launch, launched one by one"}
                                          if lanes else None)},
        "cpu_baseline": cpu, "clocks": clocks, "e2e": e2e, "gpu_launches": args.steps * launches_per_step,
        "verified_bit_exact": bool(ok),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0 if ok else 1


def reference_arm(args, rank, world, blocks, n_total, wdesc):
    """The oracle as the reference arm: each of the --steps steps decodes a
    bounded sample of the workload on one host core (the sample shrinks when
    many steps are asked for, so the run stays within about two minutes).
    Rank 0 alone runs it."""
    if rank != 0:
        return 0
    budget_weights = int(120 * 9.0e7)  # ~2 min at the oracle's ~9e7 weights/s
    per_step = budget_weights // max(1, args.steps + args.warmup)
    sample = max(1 << 20, min(args.cpu_sample // 4, 8 * 1024 * 1024, per_step))
    n_s, _, enc, _ = cpu_baseline_sample(blocks, sample, 1)
    import oracle
    for _ in range(args.warmup):
        oracle.decode(enc)
    steps = args.steps
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle.decode(enc)
    sec = (time.perf_counter() - t0) / steps
    v = n_s / sec
    scope = _sample_scope(blocks)
    desc = f"bit-serial oracle decode of the first {n_s} weights of scope {scope.name} per step, one host thread"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": "weights/s", "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u8", "data": "synthetic",
        "config": {"workload": wdesc, "weights": n_total, "sample_weights": n_s},
        "cpu_baseline": {"value": v, "unit": "weights/s", "cores": 1, "kind": "oracle", "sample": desc,
                         "cpu": host_cpu()},
        "e2e": {"value": v, "unit": "weights/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
