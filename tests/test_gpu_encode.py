"""GPU encoder parity against the CPU oracle (needs a B200).

The encoder on the GPU (dfw_encode_device, then dfw_pack_device) must give the
oracle's encoding byte for byte: the stream with its padding, the raw bytes,
the code lengths and total bits, and the known-start aux (chunk bit counts and
group starts) that the oracle recomputes by walking its own stream.  The
result must then decode back to the input.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import lossless_entropy_coded_canonical_b200 as dfw
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dfw.lib()


def device_encode_parity(oracle, u: np.ndarray, cap: int = 32, fast_bits: int = 0):
    x = torch.from_numpy(np.ascontiguousarray(u).view(np.int16)).cuda()
    dl = dfw.encode_device(x, cap, fast_bits=fast_bits)
    dfw.check()
    oenc = oracle.encode(u, cap)
    assert int(dl.table.total_bits) == oenc.total_bits
    assert np.array_equal(np.frombuffer(bytes(dl.table.len), np.uint8), oenc.lengths)
    assert np.array_equal(dl.stream.cpu().numpy(), oenc.stream)
    mant = dl.mant.cpu().numpy()
    assert mant.size == dfw.mant_bytes(u.size)
    assert np.array_equal(mant[: u.size], oenc.mant) and not mant[u.size:].any()
    if u.size == 0:
        return dl
    bits, starts = oracle.chunk_aux(oenc, 64, 32)
    cb = dl.chunk_bits.cpu().numpy().view(np.uint16)
    assert np.array_equal(cb.astype(np.uint32), bits)
    assert np.array_equal(dl.group_start.cpu().numpy().view(np.uint64), starts)
    # the host planner, walking the device-made stream, agrees on the rest
    pl = dfw.plan_lanes(dfw.Encoded(dl.stream.cpu(), dl.mant.cpu(), dl.table), fast_bits=fast_bits)
    assert pl.info.max_group_bytes == dl.info.max_group_bytes
    assert pl.info.lut_words == dl.info.lut_words
    assert np.array_equal(pl.lut.numpy(), dl.lut.cpu().numpy())
    out = dfw.decode_lanes(dl)
    dfw.check()
    assert np.array_equal(workloads.as_u16_numpy(out), u)
    return dl


def _u16(block):
    return np.concatenate([workloads.as_u16_numpy(t) for t in workloads.generate_block(block)])


CASES = {
    "c1": lambda: _u16(workloads.c1()),
    "c2": lambda: _u16(workloads.scaled(workloads.c2(), 2_000_003)),
    "c3": lambda: _u16(workloads.scaled(workloads.c3(), 2_000_003)),
    "c4a": lambda: _u16(workloads.c4("a", 1_000_003)),
    "c4b": lambda: _u16(workloads.c4("b", 1_000_003)),
    "c4bp": lambda: _u16(workloads.c4("bp", 24_200_001)),  # needs n > F36 for its 34 Fibonacci counts
    "c4c": lambda: _u16(workloads.c4("c", 1_000_003)),
}


@pytest.mark.parametrize("name", list(CASES))
def test_device_encode_matches_oracle(oracle, name):
    device_encode_parity(oracle, CASES[name]())


@pytest.mark.parametrize("n", [0, 1, 2, 7, 8, 9, 63, 64, 65, 2047, 2048, 2049, 65537])
def test_device_encode_edge_sizes(oracle, n):
    rng = np.random.default_rng(1000 + n)
    u = rng.integers(0, 65536, size=n, dtype=np.uint64).astype(np.uint16)
    device_encode_parity(oracle, u)


@pytest.mark.parametrize("n", [1, 9, 100_003])
def test_device_encode_single_symbol(oracle, n):
    rng = np.random.default_rng(n)
    u = ((rng.integers(0, 2, n) << 15) | (119 << 7) | rng.integers(0, 128, n)).astype(np.uint16)
    dl = device_encode_parity(oracle, u)
    assert int(dl.table.total_bits) == 0 and int(dl.table.n_symbols) == 1


@pytest.mark.parametrize("cap", [10, 12, 16])
def test_device_encode_cap_binding(oracle, cap):
    device_encode_parity(oracle, CASES["c4b"](), cap)


def test_device_encode_long_codes_every_group(oracle):
    """The Fibonacci-like histogram (codewords up to 32 bits) with a 9-bit
    fast table: long codewords whose words cross group edges, and escapes
    when the result is decoded."""
    device_encode_parity(oracle, CASES["c4bp"](), 32, fast_bits=9)


def test_device_encode_cap_too_small():
    x = torch.arange(0, 300 * 128, 128, dtype=torch.int32).to(torch.int16).cuda()  # 256 distinct exponents
    with pytest.raises(dfw.DfwError) as ei:
        dfw.encode_device(x, 7)
    assert ei.value.status == dfw.ECAP


def test_device_encode_full_size_block_c3():
    """One Llama-2-7B-shaped block at full size: the device encoding equals the
    host encoder's (itself byte-identical to the oracle on every workload)."""
    ts = workloads.generate_block(workloads.c3(), "cuda")
    x = torch.cat([t.reshape(-1) for t in ts])
    dl = dfw.encode_device(x)
    dfw.check()
    enc = dfw.encode_multi([t.cpu() for t in ts], 32)
    assert torch.equal(dl.stream.cpu(), enc.stream)
    assert torch.equal(dl.mant.cpu(), enc.mant)
    pl = dfw.plan_lanes(enc)
    assert torch.equal(dl.chunk_bits.cpu(), pl.chunk_bits)
    assert torch.equal(dl.group_start.cpu(), pl.group_start)
    out = dfw.decode_lanes(dl)
    dfw.check()
    assert torch.equal(out.view(torch.int16), x.view(torch.int16))


@pytest.mark.parametrize("name", ["c1", "c4b", "random2049", "single", "c4bp"])
def test_pack_writes_every_stream_byte(oracle, name):
    """dfw_pack_device into a buffer full of garbage: its first stream_bytes
    bytes become the oracle's stream (codewords and zero padding), and the
    bytes past them stay as they were."""
    import ctypes
    rng = np.random.default_rng(31)
    u = {"random2049": lambda: rng.integers(0, 65536, size=2049, dtype=np.uint64).astype(np.uint16),
         "single": lambda: ((rng.integers(0, 2, 5000) << 15) | (120 << 7)).astype(np.uint16)}.get(
        name, lambda: CASES[name]())()
    x = torch.from_numpy(np.ascontiguousarray(u).view(np.int16)).cuda()
    dl = dfw.encode_device(x)
    sb = int(dl.table.stream_bytes)
    buf = torch.full((sb + 64,), 0xA5, dtype=torch.uint8, device="cuda")
    st = dfw.lib().dfw_pack_device(x.data_ptr(), ctypes.byref(dl.table), ctypes.byref(dl.info),
                                   dl.group_start.data_ptr(), buf.data_ptr(), buf.numel(), None)
    assert st == dfw.OK
    dfw.check()
    got = buf.cpu().numpy()
    assert np.array_equal(got[:sb], oracle.encode(u).stream)
    assert (got[sb:] == 0xA5).all()
