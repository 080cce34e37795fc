"""libdfw host side (encoder, planner, LUT image) against the CPU oracle.

No GPU: these call only host entry points of libdfw.  Byte-for-byte
equality is required for the stream, the raw bytes, the lengths, gap[] and
out_start[].  The LUT image is checked by decoding streams with it (a
Python table walk) and comparing the symbols with the oracle's.
"""
import ctypes

import numpy as np
import pytest
import torch

import lossless_entropy_coded_canonical_b200 as dfw
import workloads


@pytest.fixture(scope="module", autouse=True)
def _built():
    from lossless_entropy_coded_canonical_b200.build import build
    build()


def _u16(block, n=None):
    b = workloads.scaled(block, n) if n else block
    return np.concatenate([workloads.as_u16_numpy(t) for t in workloads.generate_block(b)])


def _assert_same_encoding(enc, oenc):
    assert enc.n == oenc.n
    assert enc.total_bits == oenc.total_bits
    assert np.array_equal(enc.lengths, oenc.lengths)
    assert np.array_equal(enc.stream.numpy(), oenc.stream)
    assert np.array_equal(enc.mant.numpy()[: enc.n], oenc.mant)
    assert not enc.mant.numpy()[enc.n:].any()
    assert enc.mant.numel() == (enc.n + 15) // 16 * 16


CASES = {
    "c1": lambda: _u16(workloads.c1(), 300_001),
    "c2": lambda: _u16(workloads.c2(), 300_001),
    "c3": lambda: _u16(workloads.c3(), 300_001),
    "c4a": lambda: _u16(workloads.c4("a"), 300_001),
    "c4b": lambda: _u16(workloads.c4("b"), 300_001),
    "c4c": lambda: _u16(workloads.c4("c"), 300_001),
    "tiny": lambda: np.array([0x3F80, 0x3F80, 0xBF40, 0x3FC0, 0x3E80, 0xBF80, 0x3F81, 0x3F7F], np.uint16),
    "single": lambda: ((np.arange(1000) % 256 & 0x80) << 8 | (120 << 7) | (np.arange(1000) % 128)).astype(np.uint16),
    "empty": lambda: np.zeros(0, np.uint16),
}


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("threads", [1, 3, 8])
def test_encode_matches_oracle(oracle, name, threads):
    u = CASES[name]()
    enc = dfw.encode(u, 32, n_threads=threads)
    oenc = oracle.encode(u, 32)
    _assert_same_encoding(enc, oenc)
    if u.size:
        assert enc.table.n_symbols == len(set(((u >> 7) & 0xFF).tolist()))
    if oenc.total_bits == 0 and u.size:
        assert enc.table.single_symbol == oenc.single_symbol


@pytest.mark.parametrize("cap", [8, 9, 12, 16, 32])
def test_encode_caps_match_oracle(oracle, cap):
    u = _u16(workloads.c4("b"), 200_000)
    enc = dfw.encode(u, cap, n_threads=4)
    _assert_same_encoding(enc, oracle.encode(u, cap))


def test_encode_many_threads_and_odd_sizes(oracle):
    # chunk boundaries at every bit offset: many threads over a modest input
    u = _u16(workloads.c2(), 1_048_583)
    ref = oracle.encode(u, 32)
    for t in (2, 5, 16):
        _assert_same_encoding(dfw.encode(u, 32, n_threads=t), ref)


def test_encode_cap_errors():
    u = np.arange(65536, dtype=np.uint16)
    with pytest.raises(dfw.DfwError) as ei:
        dfw.encode(u, 7)
    assert ei.value.status == dfw.ECAP
    for cap in (0, 33):
        with pytest.raises(dfw.DfwError) as ei:
            dfw.encode(u, cap)
        assert ei.value.status == dfw.EINVAL


def test_encode_multi_matches_concatenation(oracle):
    block = workloads.scaled(workloads.c3(), 400_000)
    ts = workloads.generate_block(block)
    enc = dfw.encode_multi(ts, 32, n_threads=4)
    u = np.concatenate([workloads.as_u16_numpy(t) for t in ts])
    _assert_same_encoding(enc, oracle.encode(u, 32))
    sizes = [t.numel() for t in ts]
    assert list(enc.tensor_offsets) == list(np.concatenate([[0], np.cumsum(sizes)]))


def test_encode_multi_with_empty_tensor(oracle):
    ts = [torch.randn(1000).to(torch.bfloat16), torch.empty(0, dtype=torch.bfloat16),
          torch.randn(77).to(torch.bfloat16)]
    enc = dfw.encode_multi(ts, 32, n_threads=2)
    u = np.concatenate([workloads.as_u16_numpy(t) for t in ts])
    _assert_same_encoding(enc, oracle.encode(u, 32))
    assert list(enc.tensor_offsets) == [0, 1000, 1000, 1077]


@pytest.mark.parametrize("name", ["c1", "c2", "c4a", "c4b", "c4c", "tiny", "single"])
@pytest.mark.parametrize("W,T", [(8, 128), (8, 256), (8, 512), (16, 256)])
def test_plan_matches_oracle(oracle, name, W, T):
    u = CASES[name]()
    enc = dfw.encode(u, 32, n_threads=2)
    oenc = oracle.encode(u, 32)
    pl = dfw.plan(enc, W, T)
    gap, out_start = oracle.aux(oenc, W, T)
    assert pl.gap.numel() == pl.info.n_tiles * T
    assert np.array_equal(pl.gap.numpy()[: gap.size], gap)
    assert not pl.gap.numpy()[gap.size:].any()
    assert np.array_equal(pl.out_start.numpy().view(np.uint64), out_start)
    st = out_start.astype(np.int64)
    mx = int(np.max(np.diff(st))) if st.size > 1 else 0
    assert pl.info.max_tile_symbols == mx
    assert pl.info.n_windows == gap.size and pl.info.n_tiles + 1 == out_start.size


def test_plan_rejects_bad_shapes():
    enc = dfw.encode(CASES["c1"](), 32)
    for W, T in ((4, 256), (8, 100), (32, 256), (8, 1024), (16, 512)):
        with pytest.raises(dfw.DfwError) as ei:
            dfw.plan(enc, W, T)
        assert ei.value.status == dfw.EINVAL


def test_plan_detects_corrupt_stream():
    enc = dfw.encode(CASES["c1"](), 32)
    bad = dfw.Encoded(enc.stream.clone(), enc.mant, enc.table)
    bad.table = dfw.Table.from_buffer_copy(enc.table)
    bad.table.n = enc.table.n - 1  # the stream holds one codeword more than claimed
    with pytest.raises(dfw.DfwError) as ei:
        dfw.plan(bad)
    assert ei.value.status in (dfw.ECORRUPT, dfw.EINVAL)


def _lut_walk(lut, stream_u8, total_bits):
    """Decodes with the LUT image exactly as its format documents: key = next
    8 bits; leaf -> (symbol, total length); pointer -> subtable keyed by the
    following 8 bits."""
    bits = np.unpackbits(stream_u8)
    pad = np.zeros(64, np.uint8)
    bits = np.concatenate([bits, pad])
    syms = []
    pos = 0
    lut = lut.astype(np.uint64)
    while pos < total_bits:
        tab = 0
        level = 0
        while True:
            key = int(np.packbits(bits[pos + 8 * level: pos + 8 * level + 8])[0])
            e = int(lut[tab * 256 + key])
            if e & 0x80000000:
                tab = e & 0x3FFF
                level += 1
                assert level < 4
                continue
            syms.append(e & 0xFF)
            pos += (e >> 8) & 63
            break
    assert pos == total_bits
    return syms


def _split_lut(pl):
    img = pl.lut.numpy().view(np.uint32)
    nf = 1 << pl.info.fast_bits
    assert pl.info.lut_words == img.size == 2 * nf + 256 * pl.info.lut_tables
    return img[: 2 * nf].reshape(nf, 2), img[2 * nf:]


def _unrotate(r):
    """A fast-table symbol r = (e >> 1) | (e << 7) mod 256 back to e."""
    return ((r << 1) | (r >> 7)) & 0xFF


def _fast_window_walk(fast, hier, K, stream_u8, total_bits, W):
    """Emulates the device's phase 1 on every window: fast lookups of K bits,
    escapes through the byte hierarchy, and the window-end rule (a lookup that
    crosses the end keeps only codewords starting before it).  Returns the
    per-window symbol lists."""
    bits = np.concatenate([np.unpackbits(stream_u8), np.zeros(64, np.uint8)])
    wbits = 8 * W
    nwin = -(-total_bits // wbits)
    out = []
    # first codeword start per window, by a plain walk with the hierarchy
    starts, pos = [], 0

    def hier_one(pos):
        tab, level = 0, 0
        while True:
            key = int(np.packbits(bits[pos + 8 * level: pos + 8 * level + 8])[0])
            e = int(hier[tab * 256 + key])
            if e & 0x80000000:
                tab, level = e & 0x3FFF, level + 1
                continue
            return e & 0xFF, (e >> 8) & 63

    while pos < total_bits:
        starts.append(pos)
        pos += hier_one(pos)[1]
    starts = np.array(starts)
    for t in range(nwin):
        lo = wbits * t
        wend = min(wbits, total_bits - lo)
        after = starts[starts >= lo]
        p = int(after[0]) - lo if after.size else wend
        syms = []
        while p < wend:
            key = int(np.packbits(np.concatenate([bits[lo + p: lo + p + K], np.zeros(16 - K, np.uint8)])).view(">u2")[0]) >> (16 - K)
            e0, e1 = int(fast[key, 0]), int(fast[key, 1])
            if e1 & 0x80000000:
                s_, l_ = hier_one(lo + p)
                syms.append(s_)
                p += l_
                continue
            c = ((e1 >> 8) & 255) // 8
            cb = e1 & 255
            ends = (e1 >> 16) & 0xFFF
            take = c
            if p + cb > wend:
                r = wend - p
                take = min(c, 1 + bin(ends & ((1 << (r - 1)) - 1)).count("1"))
            # fast-table symbols are stored rotated right by one bit
            syms += [_unrotate((e0 >> (8 * i)) & 0xFF) for i in range(take)]
            p += cb
        out.append(syms)
    return out


@pytest.mark.parametrize("name", ["c1", "c4a", "c4b", "c4c", "tiny"])
@pytest.mark.parametrize("K", [8, 11, 12])
def test_lut_image_decodes_like_oracle(oracle, name, K):
    u = CASES[name]()[:20_000]
    enc = dfw.encode(u, 32 if name != "c4b" else 14)
    pl = dfw.plan(enc, 8, 128, fast_bits=K)
    assert pl.info.fast_bits == K
    fast, hier = _split_lut(pl)
    # the hierarchy alone decodes the stream
    syms = _lut_walk(hier, enc.stream.numpy(), enc.total_bits)
    e, _ = oracle.split(u)
    assert syms == list(e)
    # every fast entry satisfies what the kernel checks before use
    for key in range(1 << K):
        e0, e1 = int(fast[key, 0]), int(fast[key, 1])
        if e1 & 0x80000000:
            assert e1 == 0x80000000 | 255 and e0 == 0
            continue
        cb, c8, ends = e1 & 255, (e1 >> 8) & 255, (e1 >> 16) & 0xFFF
        assert c8 in (8, 16, 24, 32) and 1 <= cb <= K and 8 * cb >= c8
        assert bin(ends).count("1") * 8 == c8 and ends >> (cb - 1) == 1
        assert (e1 >> 28) & 7 == 0
        assert e0 >> c8 == 0 if c8 < 32 else True
    # the per-window walk the kernel performs gives the oracle's symbols in order
    W = 8
    wins = _fast_window_walk(fast, hier, K, enc.stream.numpy(), enc.total_bits, W)
    flat = [s for w in wins for s in w]
    assert flat == list(e)
    gap, out_start = oracle.aux(oracle.encode(u, 32 if name != "c4b" else 14), W, 128)
    counts = np.array([len(w) for w in wins])
    assert np.array_equal(np.concatenate([[0], np.cumsum(counts)])[::128][: out_start.size - 1],
                          out_start[:-1].astype(np.int64))


def test_plan_tables_for_cap_binding_case(oracle):
    # the Fibonacci workload's histogram needs codes of all lengths up to 32
    counts = workloads.fibonacci_counts(workloads.N64M)
    # build a small stream that uses the deepest codes, with the full-size table
    h = np.zeros(256, np.uint64)
    h[:] = counts
    ln = oracle.code_lengths(h, 32)
    assert int(ln.max()) == 32
    deep = [int(s) for s in np.argsort(-ln.astype(np.int64))[:6]]
    rng = np.random.default_rng(0)
    e = rng.choice(256, size=5000, p=counts / counts.sum())
    e[:6] = deep
    t = dfw.Table()
    t.version, t.cap, t.n = 1, 32, e.size
    for s in range(256):
        t.len[s] = int(ln[s])
    codes = oracle.canonical_codes(ln)
    bitstr = "".join(format(int(codes[x]), f"0{int(ln[x])}b") for x in e)
    t.total_bits = len(bitstr)
    t.stream_bytes = oracle.stream_bytes(t.total_bits)
    t.n_symbols = int(np.count_nonzero(ln))
    stream = np.zeros(t.stream_bytes, np.uint8)
    raw = np.packbits(np.array([int(c) for c in bitstr], np.uint8))
    stream[: raw.size] = raw
    enc = dfw.Encoded(torch.from_numpy(stream), torch.zeros((e.size + 15) // 16 * 16, dtype=torch.uint8), t)
    pl = dfw.plan(enc, 8, 256)
    assert pl.info.lut_tables > 4
    fast, hier = _split_lut(pl)
    assert _lut_walk(hier, stream, t.total_bits) == list(e)
    wins = _fast_window_walk(fast, hier, pl.info.fast_bits, stream, t.total_bits, 8)
    assert [s for w in wins for s in w] == list(e)
    oenc = oracle.Encoded(stream, np.zeros(e.size, np.uint8), ln, t.total_bits, e.size, -1)
    gap, out_start = oracle.aux(oenc, 8, 256)
    assert np.array_equal(pl.gap.numpy()[: gap.size], gap)
    assert np.array_equal(pl.out_start.numpy().view(np.uint64), out_start)


def test_bounds_helpers():
    assert dfw.mant_bytes(0) == 0 and dfw.mant_bytes(1) == 16 and dfw.mant_bytes(16) == 16
    assert dfw.stream_bound(10) >= 40 + 16


def test_decode_host_validation_without_gpu():
    # argument checks happen before any CUDA call
    enc = dfw.encode(CASES["c1"](), 32)
    pl = dfw.plan(enc)
    L = dfw.lib()
    info = dfw.PlanInfo.from_buffer_copy(pl.info)
    info.n_tiles += 1
    st = L.dfw_decode(None, None, None, None, None, ctypes.byref(enc.table), ctypes.byref(info), None, None)
    assert st == dfw.EINVAL
    bad = dfw.Table.from_buffer_copy(enc.table)
    bad.version = 99
    st = L.dfw_decode(None, None, None, None, None, ctypes.byref(bad), ctypes.byref(pl.info), None, None)
    assert st == dfw.EINVAL
    st = L.dfw_decode(None, None, None, None, None, ctypes.byref(enc.table), ctypes.byref(pl.info), None, None)
    assert st == dfw.EINVAL  # null device pointers
    st = L.dfw_decode(None, 8, None, None, None, ctypes.byref(enc.table), ctypes.byref(pl.info), 16, None)
    assert st == dfw.EALIGN
    offs = np.array([0, 5, enc.n + 1], np.uint64)
    st = L.dfw_decode_block(None, None, None, None, None, ctypes.byref(enc.table), ctypes.byref(pl.info),
                            offs.ctypes.data, 2, None, enc.n, None)
    assert st == dfw.EINVAL
    offs = np.array([0, enc.n], np.uint64)
    st = L.dfw_decode_block(None, None, None, None, None, ctypes.byref(enc.table), ctypes.byref(pl.info),
                            offs.ctypes.data, 1, None, enc.n - 1, None)
    assert st == dfw.ENOMEM


@pytest.mark.parametrize("name", ["c1", "c2", "c4a", "c4b", "c4c", "tiny", "single"])
def test_plan_lanes_matches_oracle(oracle, name):
    u = CASES[name]()
    enc = dfw.encode(u, 32, n_threads=2)
    oenc = oracle.encode(u, 32)
    pl = dfw.plan_lanes(enc)
    bits, starts = oracle.chunk_aux(oenc, 64, 32)
    assert pl.info.n_chunks == -(-u.size // 64) and pl.info.n_groups == starts.size - 1
    got_bits = pl.chunk_bits.numpy().view(np.uint16)[: bits.size]
    assert np.array_equal(got_bits.astype(np.uint32), bits)
    assert np.array_equal(pl.group_start.numpy().view(np.uint64), starts)
    spans = [((((int(starts[g + 1]) + 7) >> 3) + 8 + 15) & ~15) - ((int(starts[g]) >> 3) & ~15)
             for g in range(starts.size - 1)]
    if enc.total_bits:
        assert pl.info.max_group_bytes == max(spans + [16])
    fast, hier = _split_lut(dfw.Plan(pl.chunk_bits, pl.group_start, pl.lut, pl.info))


def test_plan_lanes_detects_corrupt_stream():
    enc = dfw.encode(CASES["c1"](), 32)
    bad = dfw.Encoded(enc.stream, enc.mant, dfw.Table.from_buffer_copy(enc.table))
    bad.table.n = enc.table.n + 1  # one codeword more than the stream holds
    with pytest.raises(dfw.DfwError) as ei:
        dfw.plan_lanes(bad)
    assert ei.value.status in (dfw.ECORRUPT, dfw.EINVAL)


# ---------------------------------------------------------------- rANS variant

def _rans_u16(name):
    if name == "edge":
        return np.random.default_rng(3).integers(0, 65536, size=70_001, dtype=np.uint64).astype(np.uint16)
    if name == "one":
        return np.full(33_333, 0x3F80, np.uint16)
    block = {"c1": workloads.c1(), "c2": workloads.c2(), "c3": workloads.c3(), "c4a": workloads.c4("a"),
             "c4b": workloads.c4("b"), "c4c": workloads.c4("c")}[name]
    return np.concatenate([workloads.as_u16_numpy(t)
                           for t in workloads.generate_block(workloads.scaled(block, 300_007))])


@pytest.mark.parametrize("name", ["c1", "c2", "c3", "c4a", "c4b", "c4c", "edge", "one"])
def test_rans_encoder_bytes_equal_oracle(oracle, name):
    u = _rans_u16(name)
    oenc = oracle.rans_encode(u, 12, 32, 16384)
    for nt in (1, 3):
        enc = dfw.rans_encode(torch.from_numpy(u.view(np.int16)), n_threads=nt)
        used = int(enc.table.stream_bytes)
        assert np.array_equal(enc.stream.numpy()[:used], oenc.stream)
        assert np.array_equal(enc.block_start.numpy().view(np.uint64), oenc.block_start)
        assert np.array_equal(np.frombuffer(bytes(enc.table.freq), np.uint16).astype(np.uint32), oenc.freq)
        assert np.array_equal(enc.mant.numpy()[: u.size], oenc.mant)
        assert enc.table.max_block_bytes == int(np.diff(oenc.block_start.astype(np.int64)).max())


def test_rans_encode_multi_equals_concatenation(oracle):
    a, b = _rans_u16("c1")[:40_000], _rans_u16("c2")[:30_001]
    enc = dfw.rans_encode([torch.from_numpy(a.view(np.int16)), torch.from_numpy(b.view(np.int16))])
    oenc = oracle.rans_encode(np.concatenate([a, b]), 12, 32, 16384)
    assert np.array_equal(enc.stream.numpy()[: int(enc.table.stream_bytes)], oenc.stream)
    assert enc.tensor_offsets.tolist() == [0, 40_000, 70_001]
