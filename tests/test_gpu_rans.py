"""GPU decode of the rANS variant against the oracle (needs a B200).

The GPU decodes the oracle's own rANS encoding (stream, block offsets,
frequencies and raw bytes produced by oracle.c) and must give exactly the
oracle's decode, which equals the input by the oracle's round-trip pin.
"""
from __future__ import annotations

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


def _device_from_oracle(oenc) -> dfw.DeviceRans:
    t = dfw.RansTable()
    t.version, t.scale_bits, t.lanes, t.block_syms = 1, oenc.scale_bits, oenc.lanes, oenc.block_syms
    t.n = oenc.n
    t.n_blocks = oenc.block_start.size - 1
    t.stream_bytes = int(oenc.block_start[-1])
    t.max_block_bytes = int(np.diff(oenc.block_start.astype(np.int64)).max()) if oenc.n else 0
    for s in range(256):
        t.freq[s] = int(oenc.freq[s])
    mant = np.zeros(dfw.mant_bytes(oenc.n), np.uint8)
    mant[: oenc.n] = oenc.mant
    stream = oenc.stream if oenc.stream.size else np.zeros(16, np.uint8)
    return dfw.DeviceRans(torch.from_numpy(stream.copy()).cuda(), torch.from_numpy(mant).cuda(),
                          torch.from_numpy(oenc.block_start.view(np.int64).copy()).cuda(), t)


def rans_parity(oracle, u):
    oenc = oracle.rans_encode(u, 12, 32, 16384)
    expect = oracle.rans_decode(oenc)
    assert np.array_equal(expect, u)
    dr = _device_from_oracle(oenc)
    out = dfw.rans_decode(dr)
    dfw.check()
    got = workloads.as_u16_numpy(out)
    bad = np.nonzero(got != expect)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first at {bad[:5]}"


def _u16(block):
    return np.concatenate([workloads.as_u16_numpy(t) for t in workloads.generate_block(block)])


CASES = {
    "c1": lambda: _u16(workloads.c1()),
    "c2": lambda: _u16(workloads.scaled(workloads.c2(), 2_000_003)),
    "c3": lambda: _u16(workloads.scaled(workloads.c3(), 2_000_003)),
    "c4a": lambda: _u16(workloads.c4("a", 1_000_003)),
    "c4b": lambda: _u16(workloads.c4("b", 1_000_003)),
    "c4c": lambda: _u16(workloads.c4("c", 1_000_003)),
}


@pytest.mark.parametrize("name", list(CASES))
def test_rans_gpu_matches_oracle(oracle, name):
    rans_parity(oracle, CASES[name]())


@pytest.mark.parametrize("n", [1, 31, 32, 33, 16383, 16384, 16385, 100_003])
def test_rans_gpu_edge_sizes(oracle, n):
    rng = np.random.default_rng(n)
    u = rng.integers(0, 65536, size=n, dtype=np.uint64).astype(np.uint16)
    rans_parity(oracle, u)


def test_rans_gpu_single_exponent(oracle):
    rng = np.random.default_rng(5)
    n = 50_001
    u = ((rng.integers(0, 2, n) << 15) | (119 << 7) | rng.integers(0, 128, n)).astype(np.uint16)
    rans_parity(oracle, u)


def test_rans_gpu_product_encoder_roundtrip():
    ts = [t.cpu() for t in workloads.generate_block(workloads.scaled(workloads.c3(), 5_000_011), "cuda")]
    enc = dfw.rans_encode(ts)
    out = dfw.rans_decode(dfw.DeviceRans.upload(enc))
    dfw.check()
    assert torch.equal(out.cpu().view(torch.int16), torch.cat([t.reshape(-1) for t in ts]).view(torch.int16))


def test_rans_gpu_corrupt_block_detected(oracle):
    u = CASES["c1"]()
    oenc = oracle.rans_encode(u, 12, 32, 16384)
    dr = _device_from_oracle(oenc)
    dr.stream[int(oenc.block_start[3]) + 4 * 7] ^= 0x10  # a bit of state 7 of block 3
    dfw.rans_decode(dr)
    assert dfw.check_status() == dfw.ECORRUPT
    dfw.check()  # cleared


def test_rans_gpu_short_block_detected(oracle):
    """Block 3's extent cut by 16 bytes (its last 8 words belong to block 4 as
    far as the decoder can tell): the states of block 3 ask for words past its
    end, those reloads are skipped, and the checks after the block report it;
    block 4, now read from 16 bytes early, fails its own checks."""
    u = CASES["c1"]()
    oenc = oracle.rans_encode(u, 12, 32, 16384)
    dr = _device_from_oracle(oenc)
    dr.block_start[4] -= 16
    out = dfw.rans_decode(dr)
    assert dfw.check_status() == dfw.ECORRUPT
    dfw.check()  # cleared
    got = workloads.as_u16_numpy(out)
    assert np.array_equal(got[: 3 * 16384], u[: 3 * 16384])  # blocks before it are untouched by the damage


def test_rans_gpu_full_size_block_c3():
    ts = [t.cpu() for t in workloads.generate_block(workloads.c3(), "cuda")]
    enc = dfw.rans_encode(ts)
    out = dfw.rans_decode(dfw.DeviceRans.upload(enc))
    dfw.check()
    assert torch.equal(out.view(torch.int16), torch.cat([t.reshape(-1) for t in ts]).cuda().view(torch.int16))
