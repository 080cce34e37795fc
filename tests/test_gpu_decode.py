"""GPU decode parity against the CPU oracle (needs a B200).

Element by element: the CUDA path decodes the oracle's own encoding (stream
and raw bytes produced by oracle.c) and must give exactly the oracle's
bit-serial decode, which the CPU pins tie to the input.  At the workloads'
full sizes, in the launch shape the benchmark times (W = 8, T = 256), every
weight is compared with the input on the device and sampled tiles with the
oracle's own decode from its own code positions.
"""
import numpy as np
import pytest
import torch

import lossless_entropy_coded_canonical_b200 as dfw
import workloads

pytestmark = pytest.mark.gpu

BENCH_SHAPE = (8, 256)
SHAPES = [(8, 128), (8, 256), (8, 512), (16, 128), (16, 256), (0, 0)]  # (0, 0): known-start plan


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from lossless_entropy_coded_canonical_b200.build import build
    build()
    dfw.check()  # clears any stale status


def encoded_from_oracle(oenc) -> dfw.Encoded:
    """The oracle's encoding wrapped in the library's table structure."""
    t = dfw.Table()
    t.version, t.cap, t.n = 1, 32, oenc.n
    t.total_bits = oenc.total_bits
    t.stream_bytes = oenc.stream.size
    for s in range(256):
        t.len[s] = int(oenc.lengths[s])
    if oenc.n and oenc.total_bits == 0:
        t.n_symbols, t.single_symbol = 1, oenc.single_symbol
    else:
        t.n_symbols = int(np.count_nonzero(oenc.lengths))
    mant = np.zeros(dfw.mant_bytes(oenc.n), np.uint8)
    mant[: oenc.n] = oenc.mant
    return dfw.Encoded(torch.from_numpy(oenc.stream.copy()), torch.from_numpy(mant), t)


def gpu_decode(enc: dfw.Encoded, W: int, T: int) -> np.ndarray:
    pl = dfw.plan(enc, W, T)
    dev = dfw.DeviceCompressed.upload(enc, pl)
    out = dfw.decode(dev)
    dfw.check()
    return workloads.as_u16_numpy(out)


def gpu_decode_lanes(enc: dfw.Encoded) -> np.ndarray:
    pl = dfw.plan_lanes(enc)
    dl = dfw.DeviceLanes.upload(enc, pl)
    out = dfw.decode_lanes(dl)
    dfw.check()
    return workloads.as_u16_numpy(out)


def oracle_parity(oracle, u: np.ndarray, W: int, T: int, cap: int = 32):
    """Windowed plan with shape (W, T), and (W == 0) the known-start plan."""
    oenc = oracle.encode(u, cap)
    expect = oracle.decode(oenc)
    enc = encoded_from_oracle(oenc)
    got = gpu_decode_lanes(enc) if W == 0 else gpu_decode(enc, W, T)
    assert got.shape == expect.shape
    bad = np.nonzero(got != expect)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first at {bad[:5]}"
    assert np.array_equal(expect, u)


def _u16(block):
    return np.concatenate([workloads.as_u16_numpy(t) for t in workloads.generate_block(block)])


SMALL = {
    "c1": lambda: _u16(workloads.c1()),
    "c2": lambda: _u16(workloads.scaled(workloads.c2(), 2_000_003)),
    "c3": lambda: _u16(workloads.scaled(workloads.c3(), 2_000_003)),
    "c4a": lambda: _u16(workloads.c4("a", 1_000_003)),
    "c4b": lambda: _u16(workloads.c4("b", 1_000_003)),
    "c4c": lambda: _u16(workloads.c4("c", 1_000_003)),
}


@pytest.mark.parametrize("W,T", SHAPES)
@pytest.mark.parametrize("name", list(SMALL))
def test_parity_small(oracle, name, W, T):
    oracle_parity(oracle, SMALL[name](), W, T)


@pytest.mark.parametrize("n", [1, 2, 7, 8, 9, 15, 16, 17, 31, 33, 255, 257, 4097, 65537])
def test_parity_edge_sizes(oracle, n):
    rng = np.random.default_rng(n)
    u = rng.integers(0, 65536, size=n, dtype=np.uint64).astype(np.uint16)
    oracle_parity(oracle, u, *BENCH_SHAPE)
    oracle_parity(oracle, u, 0, 0)
    # five exponents only: short codes, many codewords per window
    u2 = ((rng.integers(0, 2, n) << 15) | ((120 + rng.integers(0, 5, n)) << 7)
          | rng.integers(0, 128, n)).astype(np.uint16)
    oracle_parity(oracle, u2, 8, 128)
    oracle_parity(oracle, u2, 0, 0)


@pytest.mark.parametrize("n", [1, 7, 8, 9, 1000, 100_003])
def test_single_symbol(oracle, n):
    rng = np.random.default_rng(n)
    u = ((rng.integers(0, 2, n) << 15) | (119 << 7) | rng.integers(0, 128, n)).astype(np.uint16)
    oracle_parity(oracle, u, *BENCH_SHAPE)
    oracle_parity(oracle, u, 0, 0)


def test_empty():
    enc = dfw.encode(np.zeros(0, np.uint16))
    pl = dfw.plan(enc)
    dev = dfw.DeviceCompressed.upload(enc, pl)
    out = dfw.decode(dev)
    dfw.check()
    assert out.numel() == 0


@pytest.mark.parametrize("cap", [10, 12, 16, 32])
def test_cap_binding_tables(oracle, cap):
    """Geometric exponents (all 256 patterns: zeros, subnormals, Inf/NaN)
    with caps that bind, so every LUT level is exercised."""
    u = _u16(workloads.c4("b", 1_500_001))
    oracle_parity(oracle, u, 8, 256, cap)
    oracle_parity(oracle, u, 16, 256, cap)
    oracle_parity(oracle, u, 0, 0, cap)


def test_codes_straddle_tiles(oracle):
    """Long codes everywhere: many codewords cross window and tile edges."""
    rng = np.random.default_rng(11)
    counts = np.ones(256, np.int64)
    e = np.repeat(np.arange(256), counts * 200)
    rng.shuffle(e)
    u = ((e.astype(np.uint16) << 7) | rng.integers(0, 128, e.size).astype(np.uint16)).astype(np.uint16)
    oracle_parity(oracle, u, 8, 128, 32)
    oracle_parity(oracle, u[:-3], 16, 128, 12)
    oracle_parity(oracle, u[:-5], 0, 0, 32)


def test_product_encoder_roundtrip_on_gpu(oracle):
    u = SMALL["c2"]()
    enc = dfw.encode(u, 32)
    oenc = oracle.encode(u, 32)
    assert np.array_equal(enc.stream.numpy(), oenc.stream)
    assert np.array_equal(gpu_decode(enc, *BENCH_SHAPE), u)


def test_side_stream_and_reuse(oracle):
    u = SMALL["c1"]()
    enc = dfw.encode(u)
    pl = dfw.plan(enc)
    dev = dfw.DeviceCompressed.upload(enc, pl)
    s = torch.cuda.Stream()
    out = torch.empty(enc.n, dtype=torch.bfloat16, device="cuda")
    with torch.cuda.stream(s):
        for _ in range(3):
            dfw.decode(dev, out=out, stream=s)
    dfw.check(s)
    assert np.array_equal(workloads.as_u16_numpy(out), u)


# ------------------------------------------------------------ full sizes

def _full_parity(oracle, tensors, block=False, samples=6):
    """Product encode + plan in the bench shape, decode on the GPU; compare
    every weight with the input on the device, and sampled tiles with the
    oracle's decode started at the oracle's own code position."""
    enc = dfw.encode_multi(tensors, 32) if block else dfw.encode(torch.cat(tensors), 32)
    pl = dfw.plan(enc, *BENCH_SHAPE)
    dev = dfw.DeviceCompressed.upload(enc, pl)
    if block:
        scratch, views = dfw.decode_block(dev)
        dfw.check()
        for v, t in zip(views, tensors):
            assert torch.equal(v.view(torch.int16), t.to("cuda").view(torch.int16))
        out = scratch
    else:
        out = dfw.decode(dev)
        dfw.check()
        assert torch.equal(out.view(torch.int16), torch.cat(tensors).to("cuda").view(torch.int16))
    # oracle positions: its own aux over the product stream (identical bytes)
    oenc = oracle.Encoded(enc.stream.numpy(), enc.mant.numpy()[: enc.n], enc.lengths, enc.total_bits,
                          enc.n, -1)
    W, T = BENCH_SHAPE
    gap, out_start = oracle.aux(oenc, W, T)
    ntiles = out_start.size - 1
    rng = np.random.default_rng(123)
    picks = sorted(set([0, ntiles - 1] + list(rng.integers(0, ntiles, samples))))
    got_u16 = out.view(torch.int16)
    for b in picks:
        lo, hi = int(out_start[b]), int(out_start[b + 1])
        if hi == lo:
            continue
        start_bit = 8 * W * T * b + int(gap[T * b])
        syms = oracle.decode_symbols(oenc.stream, oenc.total_bits, oenc.lengths, start_bit, hi - lo)
        m = enc.mant.numpy()[lo:hi].astype(np.uint16)
        expect = ((m & 0x80) << 8) | (syms.astype(np.uint16) << 7) | (m & 0x7F)
        got = got_u16[lo:hi].cpu().numpy().view(np.uint16)
        assert np.array_equal(got, expect), f"tile {b}"
    return enc


def _full_lanes(tensors):
    """Known-start plan at full size: every weight compared with the input."""
    enc = dfw.encode_multi(tensors, 32)
    dl = dfw.DeviceLanes.upload(enc, dfw.plan_lanes(enc))
    out = dfw.decode_lanes(dl)
    dfw.check()
    assert torch.equal(out.view(torch.int16), torch.cat(tensors).to("cuda").view(torch.int16))


@pytest.mark.parametrize("name", ["c1", "c2", "c4a", "c4b", "c4bp", "c4c"])
def test_full_size_tensor_configs(oracle, name):
    block = {"c1": workloads.c1(), "c2": workloads.c2(), "c4a": workloads.c4("a"), "c4b": workloads.c4("b"),
             "c4bp": workloads.c4("bp"), "c4c": workloads.c4("c")}[name]
    ts = workloads.generate_block(block, "cuda")
    enc = _full_parity(oracle, [t.cpu() for t in ts])
    if name == "c4bp":
        assert int(enc.lengths.max()) == 32  # the cap binds
    if name == "c4c":
        assert np.all(enc.lengths == 8)
    _full_lanes([t.cpu() for t in ts])


def test_full_size_block_c3(oracle):
    ts = [t.cpu() for t in workloads.generate_block(workloads.c3(), "cuda")]
    _full_parity(oracle, ts, block=True)
    _full_lanes(ts)


def test_full_size_c5_blocks(oracle):
    """One transformer block and the embedding of the 8B-shaped model."""
    blocks = workloads.c5()
    for blk in (blocks[1], blocks[0]):
        ts = [t.cpu() for t in workloads.generate_block(blk, "cuda")]
        _full_parity(oracle, ts, block=True, samples=4)
        _full_lanes(ts)


# ------------------------------------------------------------ corruption

def _fresh(u):
    enc = dfw.encode(u)
    pl = dfw.plan(enc)
    return enc, pl, dfw.DeviceCompressed.upload(enc, pl)


def _status_after(dev):
    out = torch.zeros(dev.n, dtype=torch.bfloat16, device="cuda")
    dfw.decode(dev, out=out)
    return dfw.check_status(), out


def test_corrupt_gap_out_start_lut_stream_detected():
    u = SMALL["c1"]()
    enc, pl, dev = _fresh(u)
    assert _status_after(dev)[0] == dfw.OK
    dev.gap[1000] = 200  # that window now owns no codeword: counts disagree
    assert _status_after(dev)[0] == dfw.ECORRUPT
    dev.gap.copy_(pl.gap.to("cuda"))
    dev.out_start[7] += 3  # two tiles disagree with their counts
    assert _status_after(dev)[0] == dfw.ECORRUPT
    dev.out_start.copy_(pl.out_start.to("cuda"))
    dev.out_start[3] = dev.out_start[4] + 5  # out of order
    assert _status_after(dev)[0] == dfw.ECORRUPT
    dev.out_start.copy_(pl.out_start.to("cuda"))
    dev.lut[5] = 0  # a leaf of length 0
    assert _status_after(dev)[0] == dfw.ECORRUPT
    dev.lut.copy_(pl.lut.to("cuda"))
    half = dev.stream.numel() // 2
    dev.stream[half: half + 4096] = 0  # a run of zero bits decodes to too many codewords
    assert _status_after(dev)[0] == dfw.ECORRUPT
    dev.stream.copy_(enc.stream.to("cuda"))
    st, out = _status_after(dev)  # the context is still usable afterwards
    assert st == dfw.OK and np.array_equal(workloads.as_u16_numpy(out), u)


def test_bad_device_arguments_rejected_before_launch():
    u = SMALL["c1"]()
    enc, pl, dev = _fresh(u)
    out = torch.empty(enc.n + 8, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(dfw.DfwError) as ei:
        dfw.decode(dev, out=out[1:])  # 2-byte offset: not 16-byte aligned
    assert ei.value.status == dfw.EALIGN


def test_lanes_corrupt_aux_and_stream_detected():
    u = SMALL["c1"]()
    enc = dfw.encode(u)
    pl = dfw.plan_lanes(enc)
    dl = dfw.DeviceLanes.upload(enc, pl)

    def status():
        out = torch.zeros(dl.n, dtype=torch.bfloat16, device="cuda")
        dfw.decode_lanes(dl, out)
        return dfw.check_status(), out

    assert status()[0] == dfw.OK
    dl.chunk_bits[40] += 3  # chunk bits no longer add up to the group span
    assert status()[0] == dfw.ECORRUPT
    dl.chunk_bits.copy_(pl.chunk_bits.to("cuda"))
    dl.group_start[3] += 1  # group starts one bit late: its lanes end in the wrong place
    assert status()[0] == dfw.ECORRUPT
    dl.group_start.copy_(pl.group_start.to("cuda"))
    dl.lut[9] = 0  # a fast-table entry with no codewords and no escape mark
    assert status()[0] == dfw.ECORRUPT
    dl.lut.copy_(pl.lut.to("cuda"))
    half = dl.stream.numel() // 2
    dl.stream[half: half + 64] = 0  # zero bits: lanes end before their chunk bits say
    assert status()[0] == dfw.ECORRUPT
    dl.stream.copy_(enc.stream.to("cuda"))
    st, out = status()
    assert st == dfw.OK and np.array_equal(workloads.as_u16_numpy(out), u)


@pytest.mark.parametrize("offset", [0, 8, 16, 24])
def test_lanes_output_alignment(oracle, offset):
    """Known-start plan into an output that starts 0, 16, 32 or 48 bytes into
    a buffer: 32-byte aligned outputs take one 256-bit store per 16 weights,
    16-byte aligned ones two 128-bit stores; both must give the same bits
    and leave the bytes around the output untouched."""
    u = SMALL["c2"]()
    oenc = oracle.encode(u, 32)
    enc = encoded_from_oracle(oenc)
    dl = dfw.DeviceLanes.upload(enc, dfw.plan_lanes(enc))
    buf = torch.zeros(enc.n + 64, dtype=torch.bfloat16, device="cuda")
    out = buf[offset: offset + enc.n]
    dfw.decode_lanes(dl, out)
    dfw.check()
    assert np.array_equal(workloads.as_u16_numpy(out), oracle.decode(oenc))
    whole = workloads.as_u16_numpy(buf)
    assert not whole[:offset].any() and not whole[offset + enc.n:].any()
