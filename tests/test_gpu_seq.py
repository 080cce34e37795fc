"""dfw_decode_lanes_seq: several scopes decoded one after another into one
output buffer by one persistent launch per run of scopes (runs chained as
programmatic dependents).

The result must be exactly that of dfw_decode_lanes called on each scope in
order (same bytes everywhere in the buffer, including what earlier, larger
scopes leave beyond a later scope's end), and the last scope's weights must
be the oracle's decode of that scope.  Repeated runs over a buffer refilled
with garbage would show a store that overtook the previous scope.
"""
import ctypes

import numpy as np
import pytest
import torch

import lossless_entropy_coded_canonical_b200 as dfw
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dfw.lib()
    dfw.check()


def _u16(spec) -> np.ndarray:
    return np.concatenate([workloads.as_u16_numpy(t) for t in workloads.generate_block(spec, "cpu")])


def _scopes():
    """Mixed scopes: Llama-3 and Llama-2 block shapes (scaled), heavy tails with
    zeros, long codes (escapes), incompressible data, one exponent, a scope
    that ends inside its first group."""
    rng = np.random.default_rng(5)
    single = ((rng.integers(0, 2, 100_003) << 15) | (121 << 7) | rng.integers(0, 128, 100_003)).astype(np.uint16)
    return [
        _u16(workloads.scaled(workloads.c5()[1], 1_500_000)),
        _u16(workloads.scaled(workloads.c3(), 2_000_000)),
        single,
        _u16(workloads.scaled(workloads.c2(), 1000)),
        _u16(workloads.scaled(workloads.c4("b"), 500_000)),
        _u16(workloads.scaled(workloads.c4("c"), 300_000)),
    ]


def _device(u: np.ndarray) -> dfw.DeviceLanes:
    enc = dfw.encode(u)
    return dfw.DeviceLanes.upload(enc, dfw.plan_lanes(enc), "cuda")


@pytest.fixture(scope="module")
def scopes():
    us = _scopes()
    return us, [_device(u) for u in us]


def _garbage(n: int) -> torch.Tensor:
    return torch.full((n,), 0x5A5A, dtype=torch.int16, device="cuda").view(torch.bfloat16)


def test_seq_matches_calls_in_order(oracle, scopes):
    us, devs = scopes
    nmax = max(u.size for u in us)
    for rot in range(len(us)):  # every scope comes last once
        order = list(range(rot + 1, len(us))) + list(range(rot + 1))
        got, want = _garbage(nmax), _garbage(nmax)
        dfw.decode_lanes_seq([devs[i] for i in order], got)
        for i in order:
            dfw.decode_lanes(devs[i], want)
        dfw.check()
        assert torch.equal(got.view(torch.int16), want.view(torch.int16)), f"order {order}"
        last = us[order[-1]]
        expect = oracle.decode(oracle.encode(last))
        assert np.array_equal(workloads.as_u16_numpy(got)[: last.size], expect), f"last scope {order[-1]}"


def test_seq_repeated_over_garbage(scopes):
    us, devs = scopes
    nmax = max(u.size for u in us)
    want = _garbage(nmax)
    for d in devs:
        dfw.decode_lanes(d, want)
    dfw.check()
    for _ in range(6):
        got = _garbage(nmax)
        dfw.decode_lanes_seq(devs, got)
        dfw.check()
        assert torch.equal(got.view(torch.int16), want.view(torch.int16))


def test_seq_full_size_llama3_blocks():
    """Three consecutive transformer blocks of the 8B-shaped model at full size,
    one buffer: the buffer ends as the last block's input, bit for bit."""
    blocks = workloads.c5()[1:4]
    devs, last = [], None
    for b in blocks:
        ts = workloads.generate_block(b, "cuda")
        enc = dfw.encode_multi([t.cpu() for t in ts], 32)
        devs.append(dfw.DeviceLanes.upload(enc, dfw.plan_lanes(enc), "cuda"))
        last = torch.cat([t.reshape(-1) for t in ts])
    out = _garbage(max(d.n for d in devs))
    for _ in range(2):
        dfw.decode_lanes_seq(devs, out)
        dfw.check()
        assert torch.equal(out.view(torch.int16)[: last.numel()], last.view(torch.int16))


def test_seq_rejects_bad_arguments_before_launch(scopes):
    us, devs = scopes
    lib = dfw.lib()
    out = _garbage(max(u.size for u in us) + 8)
    before = out.clone()
    # k = 0 does nothing
    assert lib.dfw_decode_lanes_seq(0, None, out.data_ptr(), None) == dfw.OK
    # misaligned output
    d = devs[0]
    arr = (dfw.LanesScope * 1)()
    arr[0] = dfw.LanesScope(d.stream.data_ptr(), d.mant.data_ptr(), d.lut.data_ptr(), d.chunk_bits.data_ptr(),
                            d.group_start.data_ptr(), ctypes.pointer(d.table), ctypes.pointer(d.info))
    assert lib.dfw_decode_lanes_seq(1, arr, out.data_ptr() + 2, None) == dfw.EALIGN
    # one bad scope among good ones: nothing runs
    bad_info = dfw.LanesInfo.from_buffer_copy(bytes(devs[1].info))
    bad_info.n_chunks += 1
    arr3 = (dfw.LanesScope * 3)()
    for i, (dd, info) in enumerate([(devs[0], devs[0].info), (devs[1], bad_info), (devs[2], devs[2].info)]):
        arr3[i] = dfw.LanesScope(dd.stream.data_ptr(), dd.mant.data_ptr(), dd.lut.data_ptr(),
                                 dd.chunk_bits.data_ptr(), dd.group_start.data_ptr(), ctypes.pointer(dd.table),
                                 ctypes.pointer(info))
    assert lib.dfw_decode_lanes_seq(3, arr3, out.data_ptr(), None) == dfw.EINVAL
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), before.view(torch.int16))
    dfw.check()


def test_seq_replays_from_a_cuda_graph(scopes):
    """The sequence captured once into a CUDA graph (its programmatic
    dependencies become graph edges) and replayed over garbage gives the
    eager result every time: the call makes no host synchronisation and no
    allocation, so a serving loop can capture it."""
    us, devs = scopes
    nmax = max(u.size for u in us)
    want = _garbage(nmax)
    dfw.decode_lanes_seq(devs, want)
    dfw.check()
    out = _garbage(nmax)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        dfw.decode_lanes_seq(devs, out)
    for _ in range(4):
        out.view(torch.int16).fill_(0x5A5A)
        g.replay()
        torch.cuda.synchronize()
        dfw.check()
        assert torch.equal(out.view(torch.int16), want.view(torch.int16))
    del g


def test_seq_longer_than_one_launch(oracle, scopes):
    """More scopes than one persistent launch serves (40): the call chains
    launches, each holding its stores until the previous has completed; the
    buffer must still end as the calls in order leave it."""
    us, devs = scopes
    order = [i % len(devs) for i in range(2 * 40 + 3)]
    seq = [devs[i] for i in order]
    assert dfw.decode_lanes_seq_launches(seq) >= 3
    nmax = max(u.size for u in us)
    got, want = _garbage(nmax), _garbage(nmax)
    dfw.decode_lanes_seq(seq, got)
    for d in seq:
        dfw.decode_lanes(d, want)
    dfw.check()
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))


def test_seq_corrupt_scope_in_the_middle(scopes):
    """A scope whose plan or fast table is corrupt writes nothing and is
    reported; the scopes around it decode as the calls in order would."""
    us, devs = scopes
    nmax = max(u.size for u in us)
    big, small = devs[1], devs[0]  # the corrupt one is the largest, so its region is visible at the end
    for what in ("chunk_bits", "lut"):
        bad = dfw.DeviceLanes(big.stream, big.mant, big.lut.clone(), big.chunk_bits.clone(), big.group_start,
                              big.table, big.info)
        if what == "chunk_bits":
            bad.chunk_bits[40] += 3
        else:
            bad.lut[9] = 0
        seq = [small, bad, small]
        got, want = _garbage(nmax), _garbage(nmax)
        dfw.decode_lanes_seq(seq, got)
        assert dfw.check_status() == dfw.ECORRUPT, what
        for d in seq:
            dfw.decode_lanes(d, want)
        assert dfw.check_status() == dfw.ECORRUPT, what
        assert torch.equal(got.view(torch.int16), want.view(torch.int16)), what
    # the context decodes correctly afterwards
    out = _garbage(nmax)
    dfw.decode_lanes_seq(devs, out)
    dfw.check()


@pytest.mark.parametrize("offset", [8, 16])
def test_seq_output_alignment(scopes, offset):
    """A 16-byte (not 32-byte) aligned output takes two 128-bit stores per 16
    weights; the bytes around the output stay untouched."""
    us, devs = scopes
    nmax = max(u.size for u in us)
    want = _garbage(nmax)
    for d in devs:
        dfw.decode_lanes(d, want)
    dfw.check()
    buf = torch.zeros(nmax + 64, dtype=torch.int16, device="cuda")
    out = buf[offset: offset + nmax].view(torch.bfloat16)
    out.view(torch.int16).fill_(0x5A5A)
    dfw.decode_lanes_seq(devs, out)
    dfw.check()
    assert torch.equal(out.view(torch.int16), want.view(torch.int16))
    assert not buf[:offset].any() and not buf[offset + nmax:].any()


def test_seq_one_scope_equals_single_decode(oracle, scopes):
    """Each scope alone through the sequence kernel equals the oracle's decode."""
    us, devs = scopes
    for u, d in zip(us, devs):
        out = _garbage(u.size)
        dfw.decode_lanes_seq([d], out)
        dfw.check()
        assert np.array_equal(workloads.as_u16_numpy(out), oracle.decode(oracle.encode(u)))


def test_seq_tiny_and_ragged_scopes(oracle):
    """Scopes smaller than one group (most warps own no group in them), sizes
    around the chunk and group edges, and a one-exponent scope among them: the
    buffer ends as the calls in order leave it, and every scope alone through
    the sequence kernel equals the oracle's decode."""
    rng = np.random.default_rng(11)
    sizes = [1, 63, 64, 65, 2047, 2048, 2049, 70_001]
    us = [_u16(workloads.BlockSpec("t", [workloads.TensorSpec("w", n, "normal", 500 + n, 0.02)])) for n in sizes]
    assert [u.size for u in us] == sizes
    us.insert(4, ((rng.integers(0, 2, 3000) << 15) | (118 << 7) | rng.integers(0, 128, 3000)).astype(np.uint16))
    devs = [_device(u) for u in us]
    nmax = max(u.size for u in us)
    for order in (list(range(len(us))), list(range(len(us)))[::-1]):
        got, want = _garbage(nmax), _garbage(nmax)
        dfw.decode_lanes_seq([devs[i] for i in order], got)
        for i in order:
            dfw.decode_lanes(devs[i], want)
        dfw.check()
        assert torch.equal(got.view(torch.int16), want.view(torch.int16)), order
    for u, d in zip(us, devs):
        out = _garbage(u.size)
        dfw.decode_lanes_seq([d], out)
        dfw.check()
        assert np.array_equal(workloads.as_u16_numpy(out), oracle.decode(oracle.encode(u)))


def test_seq_alternating_scopes_end_with_the_last(scopes):
    """Forty scopes in one launch, two contents of nearly the same size taking
    turns over the same bytes: a store of any scope that landed after the
    next scope's store of the same group would leave the wrong content."""
    us, devs = scopes
    a, b = devs[0], devs[1]  # 1.5 M and 2.0 M weights: ragged per-CTA group counts
    want_a, want_b = _garbage(max(a.n, b.n)), _garbage(max(a.n, b.n))
    for d in (b, a):
        dfw.decode_lanes(d, want_a)
    for d in (a, b):
        dfw.decode_lanes(d, want_b)
    dfw.check()
    for last, want in ((b, want_b), (a, want_a)):
        order = [a, b] * 20 if last is b else [b, a] * 20
        assert dfw.decode_lanes_seq_launches(order) == 1
        for _ in range(3):
            got = _garbage(max(a.n, b.n))
            dfw.decode_lanes_seq(order, got)
            dfw.check()
            assert torch.equal(got.view(torch.int16), want.view(torch.int16))


def test_seq_random_mixes(oracle):
    """Seeded random sequences of up to 45 scopes (so some take two launches):
    Gaussian blocks, long-code and incompressible tensors, closed forms, one
    exponent and empty scopes at random sizes, in random order with repeats.
    Each must leave the buffer exactly as separate decodes in order do."""
    rng = np.random.default_rng(2024)

    def make(kind: str, n: int) -> np.ndarray:
        r = np.random.default_rng(int(rng.integers(1 << 31)))
        if kind == "gauss":
            return np.concatenate([workloads.as_u16_numpy(t) for t in workloads.generate_block(
                workloads.scaled(workloads.c5()[1], max(n, 7 * 64)), "cpu")])
        if kind == "geometric":
            return workloads.as_u16_numpy(workloads.generate_block(workloads.c4("b", max(n, 4096)))[0])
        if kind == "uniform":
            return r.integers(0, 65536, n, dtype=np.uint64).astype(np.uint16)
        if kind == "bitmap":
            e = np.where(r.integers(0, 2, n) == 1, 140, 139).astype(np.uint64)
            return ((e << 7) | r.integers(0, 128, n).astype(np.uint64)).astype(np.uint16)
        if kind == "single":
            return ((r.integers(0, 2, n) << 15) | (118 << 7) | r.integers(0, 128, n)).astype(np.uint16)
        return np.zeros(0, np.uint16)

    kinds = ["gauss", "gauss", "geometric", "uniform", "bitmap", "single", "empty"]
    pool = []
    for i in range(12):
        kind = kinds[i % len(kinds)]
        u = make(kind, int(rng.integers(1, 300_000)))
        enc = dfw.encode(u)
        d = dfw.DeviceLanes.upload(enc, dfw.plan_lanes(enc), "cuda")
        if kind == "empty":
            d.mant = torch.zeros(16, dtype=torch.uint8, device="cuda")
        pool.append((u, d))
    nmax = max(u.size for u, _ in pool)
    for trial in range(6):
        k = int(rng.integers(2, 46))
        order = [int(i) for i in rng.integers(0, len(pool), k)]
        devs = [pool[i][1] for i in order]
        got, want = _garbage(nmax), _garbage(nmax)
        dfw.decode_lanes_seq(devs, got)
        for d in devs:
            if d.n:
                dfw.decode_lanes(d, want)
        dfw.check()
        assert torch.equal(got.view(torch.int16), want.view(torch.int16)), f"trial {trial}: {order}"
