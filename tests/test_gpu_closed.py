"""GPU decode of the two closed forms of the canonical code (needs a B200).

Two symbols with 1-bit codes make the stream a bitmap (code 0 is the smaller
symbol); all 256 symbols with 8-bit codes make code s the symbol s itself, so
stream byte i is exponent i.  The decoder reads such codes in place, 16
weights at a time, instead of walking the fast table.  Every case here is
compared element by element with the oracle's bit-serial decode of the
oracle's own encoding, and the table is checked to really be in the closed
form the case is about.
"""
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


def _encoded(oenc) -> dfw.Encoded:
    """The oracle's encoding in the library's table structure."""
    t = dfw.Table()
    t.version, t.cap, t.n = 1, 32, oenc.n
    t.total_bits = oenc.total_bits
    t.stream_bytes = oenc.stream.size
    for s in range(256):
        t.len[s] = int(oenc.lengths[s])
    t.n_symbols = int(np.count_nonzero(oenc.lengths))
    mant = np.zeros(dfw.mant_bytes(oenc.n), np.uint8)
    mant[: oenc.n] = oenc.mant
    return dfw.Encoded(torch.from_numpy(oenc.stream.copy()), torch.from_numpy(mant), t)


def _bitmap_data(n: int, pair, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    e = np.where(rng.integers(0, 2, n) == 1, pair[1], pair[0]).astype(np.uint64)
    return ((rng.integers(0, 2, n).astype(np.uint64) << 15) | (e << 7)
            | rng.integers(0, 128, n).astype(np.uint64)).astype(np.uint16)


def _identity_data(n: int, seed: int) -> np.ndarray:
    return np.random.default_rng(seed).integers(0, 65536, n, dtype=np.uint64).astype(np.uint16)


def _check_form(oenc, form: str):
    present = oenc.lengths[oenc.lengths > 0]
    if form == "bitmap":
        assert present.size == 2 and np.all(present == 1)
    else:
        assert present.size == 256 and np.all(present == 8)


def _decode_device(enc: dfw.Encoded, out: torch.Tensor | None = None) -> torch.Tensor:
    dl = dfw.DeviceLanes.upload(enc, dfw.plan_lanes(enc))
    out = dfw.decode_lanes(dl, out)
    dfw.check()
    return out


@pytest.mark.parametrize("n", [1, 2, 15, 16, 17, 31, 1023, 65537, 1_000_003])
@pytest.mark.parametrize("pair", [(126, 127), (0, 255), (3, 200)])
def test_bitmap_matches_oracle(oracle, n, pair):
    u = _bitmap_data(n, pair, n + pair[1])
    if np.unique((u >> 7) & 0xFF).size < 2:
        pytest.skip("the draw took one exponent only")
    oenc = oracle.encode(u, 32)
    _check_form(oenc, "bitmap")
    got = workloads.as_u16_numpy(_decode_device(_encoded(oenc)))
    expect = oracle.decode(oenc)
    assert np.array_equal(expect, u)
    bad = np.nonzero(got != expect)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first at {bad[:5]}"


@pytest.mark.parametrize("n", [65536 + 5, 262_147, 2_000_003])
def test_identity_matches_oracle(oracle, n):
    u = _identity_data(n, n)
    oenc = oracle.encode(u, 32)
    _check_form(oenc, "identity")
    # the closed form itself: the stream's first n bytes are the exponents
    assert np.array_equal(oenc.stream[:n], ((u >> 7) & 0xFF).astype(np.uint8))
    got = workloads.as_u16_numpy(_decode_device(_encoded(oenc)))
    bad = np.nonzero(got != u)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first at {bad[:5]}"


@pytest.mark.parametrize("form", ["bitmap", "identity"])
@pytest.mark.parametrize("offset", [0, 8, 16, 24])
def test_closed_output_alignment(oracle, form, offset):
    """16- and 32-byte aligned outputs give the same bits and leave the bytes
    around the output untouched."""
    n = 100_003
    u = _bitmap_data(n, (120, 130), 7) if form == "bitmap" else _identity_data(n, 7)
    oenc = oracle.encode(u, 32)
    _check_form(oenc, form)
    buf = torch.zeros(n + 64, dtype=torch.bfloat16, device="cuda")
    out = buf[offset: offset + n]
    _decode_device(_encoded(oenc), out)
    assert np.array_equal(workloads.as_u16_numpy(out), u)
    whole = workloads.as_u16_numpy(buf)
    assert not whole[:offset].any() and not whole[offset + n:].any()


def test_full_size_closed_configs():
    """The two edge configurations that are closed forms, at full size, from
    the product encoder: 4a (two exponents, a bitmap) and 4c (uniform 16-bit
    patterns, every code 8 bits)."""
    for form, block in (("bitmap", workloads.c4("a")), ("identity", workloads.c4("c"))):
        ts = workloads.generate_block(block, "cuda")
        enc = dfw.encode_multi([t.cpu() for t in ts], 32)
        lens = np.array([enc.table.len[s] for s in range(256)])
        present = lens[lens > 0]
        assert (present.size, int(present.max())) == ((2, 1) if form == "bitmap" else (256, 8))
        out = _decode_device(enc)
        assert torch.equal(out.view(torch.int16), torch.cat([t.reshape(-1) for t in ts]).view(torch.int16))


def test_closed_scopes_in_a_sequence(oracle):
    """Closed-form scopes among table scopes and a one-exponent scope, in
    every rotation: the buffer ends as separate decodes in order leave it.
    A closed scope alone runs the closed-form kernel."""
    rng = np.random.default_rng(11)
    single = ((rng.integers(0, 2, 70_001) << 15) | (121 << 7) | rng.integers(0, 128, 70_001)).astype(np.uint16)
    us = [
        _bitmap_data(300_007, (100, 101), 1),
        np.concatenate([workloads.as_u16_numpy(t) for t in
                        workloads.generate_block(workloads.scaled(workloads.c3(), 400_000), "cpu")]),
        _identity_data(200_003, 2),
        single,
        _bitmap_data(50_001, (7, 9), 3),
    ]
    devs = []
    for u in us:
        enc = dfw.encode(u)
        devs.append(dfw.DeviceLanes.upload(enc, dfw.plan_lanes(enc), "cuda"))
    nmax = max(u.size for u in us)
    for rot in range(len(us)):
        order = list(range(rot + 1, len(us))) + list(range(rot + 1))
        got = torch.full((nmax,), 0x5A5A, dtype=torch.int16, device="cuda").view(torch.bfloat16)
        want = got.clone()
        dfw.decode_lanes_seq([devs[i] for i in order], got)
        for i in order:
            dfw.decode_lanes(devs[i], want)
        dfw.check()
        assert torch.equal(got.view(torch.int16), want.view(torch.int16)), f"order {order}"
        last = us[order[-1]]
        assert np.array_equal(workloads.as_u16_numpy(got)[: last.size], last)
    for i in (0, 2):  # alone
        assert dfw.decode_lanes_seq_launches([devs[i]]) == 1
        got = torch.zeros(us[i].size, dtype=torch.bfloat16, device="cuda")
        dfw.decode_lanes_seq([devs[i]], got)
        dfw.check()
        assert np.array_equal(workloads.as_u16_numpy(got), us[i])
