"""The benchmark's measurement policy, on the CPU: when L2 is flushed between
timed steps and what the line says about it, the host record beside the
oracle baseline, the oracle's samples, and the reference arm's step count."""
import json
import os
import subprocess
import sys

import numpy as np
import torch

import bench
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_l2_guard_flushes_only_below_eight_times_l2():
    l2 = 126 << 20
    small = bench.L2Guard("cpu", 683_000_000)  # a Llama-2 block's step: 5.4x the L2
    big = bench.L2Guard("cpu", 26_974_239_280)  # the 8B-shaped model's step
    assert small.l2 == l2 and big.l2 == l2  # no CUDA device here: the B200's L2 size
    assert small.flushing and small.buf.numel() == 4 * l2
    assert not big.flushing and big.buf is None
    assert "flushed" in small.label("x") and "683 MB" in small.label("x")
    assert "larger than L2" in big.label("x") and "26974 MB" in big.label("x")
    assert bench.L2Guard("cpu", 8 * l2).flushing is False
    assert bench.L2Guard("cpu", 8 * l2 - 1).flushing is True


def test_timed_steps_calls_the_step_exactly_k_times():
    calls = []

    class _Ev:
        def __init__(self, **_):
            pass

        def record(self, *_):
            pass

        def elapsed_time(self, other):
            return 1.0

    real = torch.cuda.Event, torch.cuda.synchronize
    torch.cuda.Event, torch.cuda.synchronize = _Ev, (lambda *a: None)
    try:
        guard = bench.L2Guard("cpu", 1000)
        flushes = []
        guard.flush = lambda stream=None: flushes.append(1)
        assert bench.timed_steps(lambda: calls.append(1), 7, None, guard) == 7.0  # one pair of events per step
        assert len(calls) == 7 and len(flushes) == 7
        calls.clear()
        per = []
        assert bench.timed_steps(lambda: calls.append(1), 5, None, None, per) == 1.0  # first to last event
        assert len(calls) == 5 and per == [1.0] * 5  # an event between consecutive steps
        per.clear()
        calls.clear()
        assert bench.timed_steps(lambda: calls.append(1), 3, None, guard, per) == 3.0 and per == [1.0] * 3
    finally:
        torch.cuda.Event, torch.cuda.synchronize = real


def test_step_stats():
    s = bench.step_stats([3.0, 1.0, 2.0, 5.0])
    assert s == {"median": 2.5, "best": 1.0, "worst": 5.0, "steps": 4}
    assert bench.step_stats([]) is None


def test_closed_form_labels():
    import lossless_entropy_coded_canonical_b200 as dfw

    class _D:
        def __init__(self, lens, total_bits=1):
            self.table = dfw.Table()
            for s, v in lens.items():
                self.table.len[s] = v
            self.table.total_bits = total_bits

    assert bench.scope_kernel(_D({126: 1, 127: 1})) == "decode_closed"
    assert bench.scope_kernel(_D({s: 8 for s in range(256)})) == "decode_closed"
    assert bench.scope_kernel(_D({s: 8 for s in range(254)} | {254: 9, 255: 9})) == "decode_lanes"
    assert bench.scope_kernel(_D({1: 1, 2: 2, 3: 2})) == "decode_lanes"
    assert bench.scope_kernel(_D({}, total_bits=0)) == "fill_single"


def test_host_cpu_record():
    h = bench.host_cpu()
    assert h["nproc"] >= 1 and h["logical_cpus"] >= h["nproc"] and isinstance(h["model"], str)


def test_cpu_sample_follows_the_recipe():
    # a Llama-3 block: the first 5 M weights are all of q (4096 x 4096 = 16.8 M)
    blk = workloads.c5()[1]
    u = bench.cpu_sample(blk, 5_000_000)
    assert u.dtype == np.uint16 and u.size == 5_000_000
    # the sampled scope of the 34-scope model is its first transformer block
    assert bench._sample_scope(workloads.c5()).name == "layer0"
    assert bench._sample_scope([workloads.c1()]).name == "c1"
    # size-dependent bit-pattern tensors (their exponent counts depend on n) are
    # drawn whole with the recipe's size, then cut: the sample is a prefix of that draw
    blk4 = workloads.c4("b", 1 << 20)
    v = bench.cpu_sample(blk4, 1 << 19)
    whole = workloads.as_u16_numpy(workloads.generate(blk4.tensors[0], "cpu"))
    assert v.size == 1 << 19 and np.array_equal(v, whole[: 1 << 19])


def test_reference_arm_runs_exactly_the_steps_asked():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "c1",
                          "--steps", "4", "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["steps"] == 4 and line["warmup"] == 3
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["value"] == line["e2e"]["value"]


def test_seed_offset_and_cap_flags():
    blocks = workloads.c5()[:2]
    moved = bench.reseed(blocks, 7)
    assert [t.seed for b in moved for t in b.tensors] == [t.seed + 7 for b in blocks for t in b.tensors]
    assert [t.numel for b in moved for t in b.tensors] == [t.numel for b in blocks for t in b.tensors]
    assert bench.reseed(blocks, 0) is blocks
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--cap", "0"], capture_output=True,
                         text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 2 and "--cap" in out.stderr
