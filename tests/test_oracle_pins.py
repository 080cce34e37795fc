"""Pins the CPU oracle to facts fixed outside itself (no GPU needed).

Each check would fail under a plausible slip in the oracle: a dropped or
transposed bit, a wrong length, a non-optimal or over-long code, a wrong
canonical order, a wrong gap or output prefix.
  - round trip: decoding gives back the input bit for bit (closed form);
  - Kraft equality sum 2^-len = 1 as an exact integer identity;
  - H <= mean length < H + 1 when the cap does not bind (Shannon);
  - optimality against exhaustive search on tiny alphabets, and against an
    independent depth-by-depth dynamic program when the cap binds;
  - cost equality with a heap Huffman written here when the cap is slack;
  - closed forms: two symbols, 256 near-uniform symbols, one symbol;
  - hand-worked fixtures under tests/golden/ (RFC 1951 example, tie case,
    a complete tiny encoding);
  - gap / out_start recomputed from an independent codeword walk.
"""
import heapq
import itertools
import math
import os

import numpy as np
import pytest

import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------- helpers

def kraft_ok(lengths) -> bool:
    ln = [int(x) for x in lengths if x > 0]
    return sum(1 << (32 - x) for x in ln) == 1 << 32


def cost(counts, lengths) -> int:
    return int(sum(int(c) * int(l) for c, l in zip(counts, lengths)))


def heap_huffman_depths(weights):
    """Textbook Huffman (two lightest merged repeatedly); returns leaf depths."""
    items = [(w, i, (i,)) for i, w in enumerate(weights)]
    heapq.heapify(items)
    depth = [0] * len(weights)
    counter = len(weights)
    while len(items) > 1:
        w1, _, a = heapq.heappop(items)
        w2, _, b = heapq.heappop(items)
        for leaf in a + b:
            depth[leaf] += 1
        heapq.heappush(items, (w1 + w2, counter, a + b))
        counter += 1
    return depth


def exhaustive_min_cost(weights, cap):
    best = None
    k = len(weights)
    for ls in itertools.product(range(1, cap + 1), repeat=k):
        if sum(2.0 ** -l for l in ls) <= 1.0 + 1e-12:
            c = sum(w * l for w, l in zip(weights, ls))
            best = c if best is None else min(best, c)
    return best


def dp_min_cost(weights, cap):
    """Optimal length-limited cost by a dynamic program over depths.

    Weights sorted descending get non-decreasing lengths in some optimal code
    (exchange argument).  State at depth d: i symbols already placed
    (lengths < d) and `a` free nodes at depth d.  Placing j leaves at depth d
    leaves a - j internal nodes, i.e. 2(a - j) free nodes at depth d + 1.
    Each depth adds the weight of every symbol not yet placed above it.
    """
    w = sorted((int(x) for x in weights), reverse=True)
    k = len(w)
    suffix = [0] * (k + 1)
    for i in range(k - 1, -1, -1):
        suffix[i] = suffix[i + 1] + w[i]
    INF = float("inf")
    # depth 1: i = 0 placed, 2 free nodes
    cur = {(0, 2): suffix[0]}
    for d in range(1, cap + 1):
        nxt = {}
        for (i, a), c in cur.items():
            for j in range(0, min(a, k - i) + 1):
                ni = i + j
                if ni == k:
                    key = (k, 0)
                    if c < nxt.get(key, INF):
                        nxt[key] = c
                    continue
                na = min(2 * (a - j), k - ni)
                if na == 0 or d == cap:
                    continue
                nc = c + suffix[ni]
                if nc < nxt.get((ni, na), INF):
                    nxt[(ni, na)] = nc
        cur = nxt
    return min(c for (i, a), c in cur.items() if i == k)


def entropy_bits(counts) -> float:
    c = np.asarray([x for x in counts if x > 0], dtype=np.float64)
    p = c / c.sum()
    return float(-(p * np.log2(p)).sum())


def hist_from(counts_by_symbol: dict) -> np.ndarray:
    h = np.zeros(256, np.uint64)
    for s, c in counts_by_symbol.items():
        h[s] = c
    return h


def walk_code_starts(stream, total_bits, lengths):
    """Independent codeword walk: matches the left-aligned bits against every
    (code, length) pair of the canonical code built from RFC 1951's rule."""
    codes = {}
    ln = [int(x) for x in lengths]
    bl = [0] * 34
    for l in ln:
        if l:
            bl[l] += 1
    nxt = [0] * 34
    c = 0
    for b in range(1, 33):
        c = (c + bl[b - 1]) << 1
        nxt[b] = c
    for s in range(256):
        if ln[s]:
            codes[(ln[s], nxt[ln[s]])] = s
            nxt[ln[s]] += 1
    bits = np.unpackbits(np.asarray(stream, dtype=np.uint8))[:total_bits]
    starts, syms = [], []
    pos = 0
    while pos < total_bits:
        starts.append(pos)
        v = 0
        for l in range(1, 33):
            v = (v << 1) | int(bits[pos + l - 1])
            if (l, v) in codes:
                syms.append(codes[(l, v)])
                pos += l
                break
        else:
            raise AssertionError("no codeword matched")
    return starts, syms


def bf16_u16(values) -> np.ndarray:
    import torch
    return workloads.as_u16_numpy(torch.tensor(values, dtype=torch.float32).to(torch.bfloat16))


# ----------------------------------------------------------------- split / join

def test_split_join_closed_form(oracle):
    u = np.arange(65536, dtype=np.uint16)  # every bf16 pattern, NaNs included
    e, m = oracle.split(u)
    assert np.array_equal(e, ((u >> 7) & 0xFF).astype(np.uint8))
    assert np.array_equal(m >> 7, (u >> 15).astype(np.uint8))  # sign bit
    assert np.array_equal(m & 0x7F, (u & 0x7F).astype(np.uint8))  # mantissa bits
    # float semantics: exponent field of 1.0 is 127, of 2^-6 is 121, of -0.0 is 0
    e2, m2 = oracle.split(bf16_u16([1.0, 2.0 ** -6, -0.0, -3.0]))
    assert list(e2) == [127, 121, 0, 128]
    assert list(m2) == [0x00, 0x00, 0x80, 0x80 | 0x40]
    for x in (0x0000, 0x8000, 0x7F80, 0xFFC1, 0x3F80, 0x0001):
        ee, mm = oracle.split(np.array([x], np.uint16))
        assert oracle.join(int(ee[0]), int(mm[0])) == x


# ----------------------------------------------------------------- lengths

@pytest.mark.parametrize("seed", range(40))
def test_lengths_optimal_exhaustive_tiny(oracle, seed):
    rng = np.random.default_rng(seed)
    k = int(rng.integers(2, 7))
    syms = rng.choice(256, size=k, replace=False)
    w = [int(x) for x in rng.integers(1, 50, size=k)]
    h = hist_from(dict(zip(syms, w)))
    min_cap = max(1, math.ceil(math.log2(k)))
    for cap in range(min_cap, 7):
        ln = oracle.code_lengths(h, cap)
        got = [int(ln[s]) for s in syms]
        assert max(got) <= cap and min(got) >= 1
        assert kraft_ok(ln)
        assert cost(w, got) == exhaustive_min_cost(w, cap), (w, cap, got)
        assert np.count_nonzero(ln) == k


@pytest.mark.parametrize("seed", range(6))
def test_lengths_optimal_dp_binding_cap(oracle, seed):
    # Fibonacci-like weights force deep unconstrained trees; cap binds.
    rng = np.random.default_rng(100 + seed)
    k = int(rng.integers(8, 14))
    fib = [1, 1]
    while len(fib) < k:
        fib.append(fib[-1] + fib[-2])
    w = [f + int(rng.integers(0, 2)) for f in fib]
    syms = rng.choice(256, size=k, replace=False)
    h = hist_from(dict(zip(syms, w)))
    free_depth = max(heap_huffman_depths(w))
    for cap in range(math.ceil(math.log2(k)), free_depth + 2):
        ln = oracle.code_lengths(h, cap)
        got = [int(ln[s]) for s in syms]
        assert max(got) <= cap
        assert kraft_ok(ln)
        assert cost(w, got) == dp_min_cost(w, cap), (w, cap)


def test_dp_agrees_with_exhaustive():
    # pins the test's own dynamic program against brute force
    rng = np.random.default_rng(7)
    for _ in range(30):
        k = int(rng.integers(2, 7))
        w = [int(x) for x in rng.integers(1, 40, size=k)]
        for cap in range(max(1, math.ceil(math.log2(k))), 6):
            assert dp_min_cost(w, cap) == exhaustive_min_cost(w, cap)


@pytest.mark.parametrize("seed", range(10))
def test_lengths_match_heap_huffman_cost_when_cap_slack(oracle, seed):
    rng = np.random.default_rng(200 + seed)
    k = int(rng.integers(2, 257))
    syms = rng.choice(256, size=k, replace=False)
    w = [int(x) for x in rng.integers(1, 10 ** 6, size=k)]
    depths = heap_huffman_depths(w)
    assert max(depths) <= 32
    ln = oracle.code_lengths(hist_from(dict(zip(syms, w))), 32)
    got = [int(ln[s]) for s in syms]
    assert kraft_ok(ln)
    assert cost(w, got) == cost(w, depths)


def test_lengths_entropy_bounds_gaussian(oracle):
    import torch
    x = workloads.generate(workloads.scaled(workloads.c1(), 1 << 18).tensors[0])
    e, _ = oracle.split(workloads.as_u16_numpy(x))
    h = oracle.histogram(e)
    ln = oracle.code_lengths(h, 32)
    H = entropy_bits(h)
    mean = cost(h, ln) / int(h.sum())
    assert H <= mean < H + 1
    # the pages' ~1.5:1: about 8 + 2.6 bits per weight for N(0, sigma)
    bits_per_weight = 8 + mean
    assert 1.4 < 16 / bits_per_weight < 1.6


def test_histogram_counts(oracle):
    e = np.array([3, 3, 7, 255, 0, 3], np.uint8)
    h = oracle.histogram(e)
    assert h[3] == 3 and h[7] == 1 and h[255] == 1 and h[0] == 1 and int(h.sum()) == 6


def test_cap_binding_fibonacci_256(oracle):
    """Workload 4b' (64M weights): unconstrained Huffman depth is 33, so the
    32-bit cap binds; capped lengths must be <= 32, complete, and no cheaper
    than Huffman; cap 16 on the geometric workload 4b binds too."""
    counts = workloads.fibonacci_counts(workloads.N64M)
    free = heap_huffman_depths([int(c) for c in counts])
    assert max(free) == 33
    h = np.zeros(256, np.uint64)
    h[:] = counts  # rank r -> symbol r (any bijection gives the same multiset)
    ln = oracle.code_lengths(h, 32)
    assert int(ln.max()) == 32 and kraft_ok(ln)
    assert cost(counts, ln) >= cost(counts, free)
    assert cost(counts, ln) - cost(counts, free) < int(counts.sum()) // 1000
    g = workloads.geometric_counts(workloads.N64M)
    gfree = heap_huffman_depths([int(c) for c in g])
    assert max(gfree) <= 32  # the geometric workload does not bind at 32
    hg = np.zeros(256, np.uint64)
    hg[:] = g
    ln32 = oracle.code_lengths(hg, 32)
    assert cost(g, ln32) == cost(g, gfree)
    ln16 = oracle.code_lengths(hg, 16)
    assert int(ln16.max()) == 16 and kraft_ok(ln16)
    assert cost(g, ln16) > cost(g, gfree)


def test_cap_too_small_is_rejected(oracle):
    h = hist_from({s: 1 for s in range(5)})
    assert oracle.code_lengths_status(h, 2) == oracle.ECAP
    assert oracle.code_lengths_status(h, 3) == oracle.OK
    assert oracle.code_lengths_status(h, 0) == oracle.EINVAL
    assert oracle.code_lengths_status(h, 33) == oracle.EINVAL


def test_tie_rule_hand_worked(oracle):
    rows = [l.split() for l in open(os.path.join(GOLDEN, "tie_case.txt")) if l.strip() and not l.startswith("#")]
    cap = int([r for r in rows if r[0] == "cap"][0][1])
    table = [tuple(map(int, r)) for r in rows if r[0] != "cap"]
    h = hist_from({s: c for s, c, _ in table})
    ln = oracle.code_lengths(h, cap)
    assert [int(ln[s]) for s, _, _ in table] == [l for _, _, l in table]


def test_one_and_zero_symbols(oracle):
    ln = oracle.code_lengths(hist_from({42: 1000}), 32)
    assert int(ln.sum()) == 0
    ln = oracle.code_lengths(np.zeros(256, np.uint64), 32)
    assert int(ln.sum()) == 0


# ----------------------------------------------------------------- canonical codes

def test_canonical_rfc1951_example(oracle):
    rows = [l.split() for l in open(os.path.join(GOLDEN, "rfc1951_canonical.txt")) if l.strip() and not l.startswith("#")]
    ln = np.zeros(256, np.uint8)
    for s, l, _ in rows:
        ln[int(s)] = int(l)
    codes = oracle.canonical_codes(ln)
    for s, l, c in rows:
        assert format(int(codes[int(s)]), f"0{int(l)}b") == c


@pytest.mark.parametrize("seed", range(5))
def test_canonical_prefix_free_and_ordered(oracle, seed):
    rng = np.random.default_rng(300 + seed)
    k = int(rng.integers(2, 257))
    syms = rng.choice(256, size=k, replace=False)
    w = rng.integers(1, 10 ** 5, size=k)
    ln = oracle.code_lengths(hist_from(dict(zip(syms, w))), 32)
    codes = oracle.canonical_codes(ln)
    present = sorted((int(ln[s]), int(s)) for s in range(256) if ln[s])
    left = [int(codes[s]) << (32 - l) for l, s in present]
    # canonical: left-aligned codewords strictly increase in (length, symbol)
    # order, and consecutive intervals tile [0, 2^32) with no gap or overlap
    pos = 0
    for (l, s), v in zip(present, left):
        assert v == pos
        pos += 1 << (32 - l)
    assert pos == 1 << 32


# ----------------------------------------------------------------- encode / decode

def test_tiny_stream_hand_worked(oracle):
    rows = {}
    for line in open(os.path.join(GOLDEN, "tiny_stream.txt")):
        if line.strip() and not line.startswith("#"):
            k, *v = line.split()
            rows[k] = v
    u = np.array([int(x, 16) for x in rows["u16"]], np.uint16)
    e, m = oracle.split(u)
    assert list(e) == [int(x) for x in rows["exp"]]
    assert list(m) == [int(x, 16) for x in rows["mant"]]
    enc = oracle.encode(u, 32)
    for kv in rows["len"]:
        s, l = kv.split(":")
        assert enc.lengths[int(s)] == int(l)
    codes = oracle.canonical_codes(enc.lengths)
    for kv in rows["code"]:
        s, c = kv.split(":")
        assert format(int(codes[int(s)]), f"0{len(c)}b") == c
    assert enc.total_bits == int(rows["total_bits"][0])
    assert enc.stream.size == int(rows["stream_bytes"][0])
    head = [int(x, 16) for x in rows["stream_head"]]
    assert list(enc.stream[: len(head)]) == head
    assert not enc.stream[len(head):].any()
    assert np.array_equal(oracle.decode(enc), u)
    gap, out_start = oracle.aux(enc, 4, 1)
    assert list(gap) == [int(x) for x in rows["gap_W4"]]
    assert list(out_start) == [int(x) for x in rows["out_start_W4_T1"]]


def _roundtrip(oracle, u, cap=32):
    enc = oracle.encode(u, cap)
    out = oracle.decode(enc)
    assert np.array_equal(out, u)
    ln = enc.lengths
    if enc.total_bits:
        assert kraft_ok(ln)
        assert int(ln.max()) <= cap
        e, _ = oracle.split(u)
        assert enc.total_bits == cost(np.bincount(e, minlength=256), ln)
    return enc


@pytest.mark.parametrize("name", ["c1", "c2", "c3", "c4a", "c4b", "c4c"])
def test_roundtrip_workloads_scaled(oracle, name):
    block = {"c1": workloads.c1(), "c2": workloads.c2(), "c3": workloads.c3(), "c4a": workloads.c4("a"),
             "c4b": workloads.c4("b"), "c4c": workloads.c4("c")}[name]
    small = workloads.scaled(block, 200_003)
    u = np.concatenate([workloads.as_u16_numpy(t) for t in workloads.generate_block(small)])
    _roundtrip(oracle, u)


@pytest.mark.parametrize("n", [0, 1, 7, 8, 9, 31, 33, 1000])
def test_roundtrip_edge_sizes(oracle, n):
    rng = np.random.default_rng(n)
    u = rng.integers(0, 65536, size=n, dtype=np.uint64).astype(np.uint16)
    enc = _roundtrip(oracle, u)
    assert enc.stream.size == oracle.stream_bytes(enc.total_bits)


def test_roundtrip_all_patterns_and_caps(oracle):
    u = np.arange(65536, dtype=np.uint16)
    for cap in (8, 9, 12, 32):
        enc = _roundtrip(oracle, u, cap)
        assert int(enc.lengths.max()) == 8  # 256 equiprobable symbols
    with pytest.raises(oracle.OracleError):
        oracle.encode(u, 7)  # 256 symbols cannot fit in 7 bits


def test_single_symbol_closed_form(oracle):
    rng = np.random.default_rng(5)
    u = ((rng.integers(0, 256, 1000) & 0x80) << 8 | (121 << 7) | (rng.integers(0, 128, 1000))).astype(np.uint16)
    enc = oracle.encode(u)
    assert enc.total_bits == 0 and enc.single_symbol == 121
    assert enc.stream.size == 16 and not enc.stream.any()
    assert np.array_equal(oracle.decode(enc), u)


def test_two_exponent_closed_form(oracle):
    """4a: lengths {1, 1}; the smaller exponent gets codeword 0, so the stream
    is exactly the bitmap [e == 127], n bits long."""
    x = workloads.generate(workloads.c4("a", 1 << 16).tensors[0])
    u = workloads.as_u16_numpy(x)
    e, _ = oracle.split(u)
    enc = oracle.encode(u)
    assert enc.lengths[126] == 1 and enc.lengths[127] == 1 and np.count_nonzero(enc.lengths) == 2
    assert enc.total_bits == u.size
    assert np.array_equal(np.unpackbits(enc.stream)[: u.size], (e == 127).astype(np.uint8))


def test_uniform_closed_form(oracle):
    """4c: 256 near-equal counts (max < 2 min) give every symbol length 8, and
    canonical code of s is s, so the stream equals the exponent bytes."""
    x = workloads.generate(workloads.c4("c", 1 << 20).tensors[0])
    u = workloads.as_u16_numpy(x)
    e, _ = oracle.split(u)
    h = oracle.histogram(e)
    assert int(h.max()) < 2 * int(h.min())
    enc = oracle.encode(u)
    assert np.all(enc.lengths == 8)
    assert np.array_equal(enc.stream[: u.size], e)
    assert (16 * u.size) / (8 * enc.stream.size + 8 * u.size) < 1.0  # incompressible


def test_corrupt_stream_detected(oracle):
    x = workloads.generate(workloads.scaled(workloads.c1(), 5000).tensors[0])
    u = workloads.as_u16_numpy(x)
    enc = oracle.encode(u)
    rc, _ = oracle.decode_raw(enc.stream, enc.total_bits - 1, enc.lengths, -1, enc.mant, enc.n)
    assert rc == oracle.ECORRUPT
    rc, _ = oracle.decode_raw(enc.stream, enc.total_bits, enc.lengths, -1, enc.mant, enc.n + 1)
    assert rc == oracle.ECORRUPT


# ----------------------------------------------------------------- aux arrays

@pytest.mark.parametrize("W,T", [(4, 1), (4, 3), (8, 32), (16, 7), (32, 256)])
@pytest.mark.parametrize("kind", ["c1", "c4b"])
def test_aux_against_independent_walk(oracle, W, T, kind):
    block = workloads.scaled(workloads.c1() if kind == "c1" else workloads.c4("b"), 20_000)
    u = workloads.as_u16_numpy(workloads.generate(block.tensors[0]))
    enc = oracle.encode(u)
    starts, syms = walk_code_starts(enc.stream, enc.total_bits, enc.lengths)
    e, _ = oracle.split(u)
    assert syms == list(e)
    gap, out_start = oracle.aux(enc, W, T)
    nwin = -(-enc.total_bits // (8 * W))
    assert gap.size == nwin
    st = np.array(starts, dtype=np.int64)
    for t in range(nwin):
        lo = 8 * W * t
        after = st[st >= lo]
        first = int(after[0]) if after.size else enc.total_bits
        assert gap[t] == first - lo
        assert gap[t] < 32
    ntiles = -(-nwin // T)
    assert out_start.size == ntiles + 1
    for b in range(ntiles):
        assert out_start[b] == int(np.count_nonzero(st < 8 * W * T * b))
    assert out_start[-1] == u.size


def test_aux_window_without_code_start(oracle):
    """The last 32-bit window holds only the tail of a code that starts in
    the window before: its gap reaches total_bits and it owns no symbol.
    Exponents: 101 (2 bits), 29 x 127 (1 bit each), 100 (2 bits) ->
    codes at bits 0, 2..30, 31; total 33 bits; window 1 = bit 32 only."""
    e = np.array([101] + [127] * 29 + [100], dtype=np.uint16)
    u = (e << 7).astype(np.uint16)
    enc = oracle.encode(u)
    assert (enc.lengths[127], enc.lengths[100], enc.lengths[101]) == (1, 2, 2)
    assert enc.total_bits == 33
    gap, out_start = oracle.aux(enc, 4, 1)
    assert list(gap) == [0, 1]
    assert list(out_start) == [0, 31, 31]
    assert np.array_equal(oracle.decode(enc), u)


@pytest.mark.parametrize("M,G", [(64, 32), (4, 3), (1, 1), (7, 5)])
@pytest.mark.parametrize("kind", ["c1", "c4b", "single"])
def test_chunk_aux_against_independent_walk(oracle, M, G, kind):
    if kind == "single":
        u = ((np.arange(999) % 2) << 15 | (121 << 7)).astype(np.uint16)
    else:
        block = workloads.scaled(workloads.c1() if kind == "c1" else workloads.c4("b"), 10_007)
        u = workloads.as_u16_numpy(workloads.generate(block.tensors[0]))
    enc = oracle.encode(u)
    bits, starts = oracle.chunk_aux(enc, M, G)
    if enc.total_bits:
        st, _ = walk_code_starts(enc.stream, enc.total_bits, enc.lengths)
    else:
        st = [0] * u.size
    st = list(st) + [enc.total_bits]
    n_chunks = -(-u.size // M)
    n_groups = -(-n_chunks // G)
    assert bits.size == n_groups * G and starts.size == n_groups + 1
    for c in range(n_groups * G):
        if c < n_chunks:
            assert bits[c] == st[min(M * (c + 1), u.size)] - st[M * c]
        else:
            assert bits[c] == 0
    for g in range(n_groups):
        assert starts[g] == st[M * G * g]
    assert starts[-1] == enc.total_bits
    assert int(bits.sum()) == enc.total_bits


# ---------------------------------------------------------------- y = W x

def _u16_normal(rng, n: int) -> np.ndarray:
    """bf16 patterns of N(0, 0.02) draws (round to nearest even by hand)."""
    f = (rng.standard_normal(n) * 0.02).astype(np.float32).view(np.uint32)
    return ((f + 0x7FFF + ((f >> 16) & 1)) >> 16).astype(np.uint16)


def _bf16_of(v: float) -> int:
    """bf16 pattern of a float32-exact value whose low 16 bits are zero."""
    u = int(np.array([v], np.float32).view(np.uint32)[0])
    assert u & 0xFFFF == 0
    return u >> 16


def test_bf16_values_closed_forms(oracle):
    pats = np.array([0x3F80, 0xC000, 0x0001, 0x8000, 0x7F80, 0x4049, 0x3C23], np.uint16)
    want = [1.0, -2.0, 2.0 ** -133, -0.0, np.inf, 3.140625, 0.0099487304687500]
    got = oracle.bf16_values(pats)
    assert got[:5].tolist() == want[:5] and np.signbit(got[3])
    # 0x4049 = 2^1 * (1 + 0x49 / 128); 0x3C23 = 2^-7 * (1 + 0x23 / 128)
    assert got[5] == 2.0 * (1 + 0x49 / 128) == want[5]
    assert got[6] == 2.0 ** -7 * (1 + 0x23 / 128)


def test_gemv_hand_worked(oracle):
    """tests/golden/gemv_small.txt: a 2 x 64 case summed by hand."""
    kv = dict(line.split(":", 1) for line in open(os.path.join(GOLDEN, "gemv_small.txt"))
              if ":" in line and not line.startswith("#"))
    rows, cols = int(kv["rows"]), int(kv["cols"])
    want = [float(v) for v in kv["y"].split()]
    w = np.empty((rows, cols), np.uint16)
    w[0, :] = 0x3F80
    w[1, 0::2] = 0x3F00
    w[1, 1::2] = 0xBE80
    x = np.array([_bf16_of(j + 1) for j in range(cols)], np.uint16)
    assert oracle.gemv(w.reshape(-1), rows, cols, x).tolist() == want
    want_abs = [float(v) for v in kv["y_abs"].split()]
    assert oracle.gemv_abs(w.reshape(-1), rows, cols, x).tolist() == want_abs


def test_gemv_basis_vectors_pick_columns(oracle):
    rng = np.random.default_rng(5)
    rows, cols = 7, 128
    w = _u16_normal(rng, rows * cols)
    for j in (0, 1, 63, 64, 127):
        x = np.zeros(cols, np.uint16)
        x[j] = 0x3F80  # 1.0
        y = oracle.gemv(w, rows, cols, x)
        assert np.array_equal(y, oracle.bf16_values(w).reshape(rows, cols)[:, j])


def test_gemv_abs_against_exact_rationals(oracle):
    """gemv_abs is the exact sum of |w x| (up to float64 rounding), with
    negative weights and negative inputs present: a version that dropped the
    absolute value of either operand, took it of the sum instead of the terms,
    or used the wrong axis would miss these by far more than the rounding."""
    from fractions import Fraction
    rng = np.random.default_rng(8)
    rows, cols = 4, 128
    w, x = _u16_normal(rng, rows * cols), _u16_normal(rng, cols)
    wv = oracle.bf16_values(w).reshape(rows, cols)
    xv = oracle.bf16_values(x)
    assert (wv < 0).any() and (wv > 0).any() and (xv < 0).any() and (xv > 0).any()
    got = oracle.gemv_abs(w, rows, cols, x)
    assert got.shape == (rows,)
    for i in range(rows):
        exact = sum(abs(Fraction(float(wv[i, j])) * Fraction(float(xv[j]))) for j in range(cols))
        assert abs(Fraction(float(got[i])) - exact) <= Fraction(cols * 2.0 ** -53) * exact
        signed = abs(sum(Fraction(float(wv[i, j])) * Fraction(float(xv[j])) for j in range(cols)))
        assert exact > signed  # the terms have mixed signs: |sum| is strictly smaller
    # one row of all-negative weights against all-negative inputs: every term
    # is positive, so the signed product equals the absolute sum
    wn = np.full(cols, 0xBF80, np.uint16)  # -1.0
    xn = np.array([0x8000 | _bf16_of(j + 1) for j in range(cols)], np.uint16)  # -(j + 1)
    assert oracle.gemv_abs(wn, 1, cols, xn).tolist() == [cols * (cols + 1) / 2]
    assert oracle.gemv(wn, 1, cols, xn).tolist() == [cols * (cols + 1) / 2]


def test_gemv_against_exact_rationals(oracle):
    """Exact rational sums (fractions) of the same products: the float64
    result is within float64 rounding of them."""
    from fractions import Fraction
    rng = np.random.default_rng(6)
    rows, cols = 3, 192
    w, x = _u16_normal(rng, rows * cols), _u16_normal(rng, cols)
    y = oracle.gemv(w, rows, cols, x)
    scale = oracle.gemv_abs(w, rows, cols, x)
    wv = oracle.bf16_values(w).reshape(rows, cols)
    xv = oracle.bf16_values(x)
    for i in range(rows):
        exact = sum(Fraction(float(wv[i, j])) * Fraction(float(xv[j])) for j in range(cols))
        assert abs(Fraction(float(y[i])) - exact) <= Fraction(cols * 2.0 ** -53) * Fraction(float(scale[i]))


# ---------------------------------------------------------------- rANS variant

def test_rans_hand_worked(oracle):
    kv = dict(line.split(":", 1) for line in open(os.path.join(GOLDEN, "rans_tiny.txt"))
              if ":" in line and not line.startswith("#"))
    freq = np.zeros(256, np.uint32)
    freq[0], freq[1] = int(kv["freq0"]), int(kv["freq1"])
    e = np.array([int(v) for v in kv["symbols"].split()], np.uint8)
    stream, starts = oracle.rans_encode_symbols(e, freq, int(kv["scale_bits"]), int(kv["lanes"]), 16)
    want = np.array([int(b, 16) for b in kv["stream"].split()], np.uint8)
    assert np.array_equal(stream, want) and starts.tolist() == [0, 16]
    assert int(stream[:4].view(np.uint32)[0]) == int(kv["final_state"])
    rc, back = oracle.rans_decode_symbols(stream, starts, 2, freq, 8, 1, 16)
    assert rc == 0 and back.tolist() == [0, 1]


def test_rans_freqs_rules(oracle):
    h = np.zeros(256, np.uint64)
    h[[3, 9]] = [3000, 1000]  # proportional: exactly 3/4 and 1/4 of 4096
    f = oracle.rans_freqs(h, 12)
    assert f[3] == 3072 and f[9] == 1024 and f.sum() == 4096 and np.count_nonzero(f) == 2
    h = np.zeros(256, np.uint64)
    h[[0, 1, 2]] = [1, 1, 1]  # floors 1365 each, remainder 1 to the smallest of the tied most frequent
    f = oracle.rans_freqs(h, 12)
    assert f[:3].tolist() == [1366, 1365, 1365]
    h = np.zeros(256, np.uint64)
    h[0], h[1:201] = 10 ** 9, 1  # 200 rare symbols bumped to 1: the excess comes off the largest
    f = oracle.rans_freqs(h, 8)
    assert f.sum() == 256 and (f[1:201] == 1).all() and f[0] == 56 and not f[201:].any()
    h = np.zeros(256, np.uint64)
    h[77] = 5
    assert oracle.rans_freqs(h, 12)[77] == 4096


def test_rans_single_symbol_closed_form(oracle):
    e = np.full(5000, 77, np.uint8)
    freq = np.zeros(256, np.uint32)
    freq[77] = 4096
    stream, starts = oracle.rans_encode_symbols(e, freq, 12, 32, 4096)
    # every state stays at 65536 and no word is written: 2 blocks of 128 bytes
    assert starts.tolist() == [0, 128, 256]
    assert (stream.view(np.uint32) == 65536).all()


def test_rans_lanes_are_independent_coders(oracle):
    """With 32 interleaved states, the final state of lane j equals that of
    a one-state encoding of every 32nd exponent starting at j."""
    rng = np.random.default_rng(12)
    e = rng.choice(np.arange(6, dtype=np.uint8), size=4096, p=[0.4, 0.3, 0.15, 0.1, 0.04, 0.01])
    freq = oracle.rans_freqs(oracle.histogram(e), 12)
    stream, starts = oracle.rans_encode_symbols(e, freq, 12, 32, 4096)
    states = stream[:128].view(np.uint32)
    for j in (0, 1, 17, 31):
        s1, _ = oracle.rans_encode_symbols(e[j::32], freq, 12, 1, 128)
        assert int(s1[:4].view(np.uint32)[0]) == int(states[j])


def test_rans_rate_within_information_bounds(oracle):
    """Per lane, 16 (words) + log2(final state) - 16 is the information
    sum_i log2(M / f_i) of its exponents up to a rounding term of at most
    log2(1 / (1 - 2^-4)) < 0.1 bits per exponent (x >= 2^16 while f <= M)."""
    rng = np.random.default_rng(13)
    e = rng.choice(np.arange(5, dtype=np.uint8), size=32 * 2000, p=[0.5, 0.25, 0.15, 0.07, 0.03])
    freq = oracle.rans_freqs(oracle.histogram(e), 12)
    stream, starts = oracle.rans_encode_symbols(e, freq, 12, 32, e.size)
    info = np.log2(4096.0 / freq[e].astype(np.float64))
    words = (stream.size - 128) // 2  # padding < 16 bytes: at most 7 words of zeros
    total = 16 * words + np.log2(stream[:128].view(np.uint32).astype(np.float64)).sum() - 16 * 32
    assert info.sum() - 1.0 <= total <= info.sum() + 0.1 * e.size + 16 * 8


def _rans_case(name: str) -> np.ndarray:
    if name == "tiny":
        return np.array([0x3F80, 0x3F80, 0xBF00, 0x0001, 0x7F80, 0x3F80, 0xC000], np.uint16)
    block = {"c1": workloads.c1(), "c4a": workloads.c4("a"), "c4b": workloads.c4("b"),
             "c4c": workloads.c4("c")}[name]
    return np.concatenate([workloads.as_u16_numpy(t) for t in workloads.generate_block(workloads.scaled(block, 60_003))])


@pytest.mark.parametrize("name", ["c1", "c4a", "c4b", "c4c", "tiny"])
@pytest.mark.parametrize("lanes,block", [(32, 16384), (32, 8192), (1, 64), (8, 4096)])
def test_rans_roundtrip(oracle, name, lanes, block):
    u = _rans_case(name)
    enc = oracle.rans_encode(u, 12, lanes, block)
    assert np.array_equal(oracle.rans_decode(enc), u)


def test_rans_corrupt_state_detected(oracle):
    u = _rans_case("c1")[:50_000]
    enc = oracle.rans_encode(u)
    bad = enc.stream.copy()
    bad[4 * 5] ^= 0x40  # a bit of state 5 of block 0
    rc, _ = oracle.rans_decode_symbols(bad, enc.block_start, enc.n, enc.freq)
    assert rc == oracle.ECORRUPT
