"""The container (include/dfw.h, CONTAINER): an encoded tensor or block as
one byte buffer.  Pins: what comes back is the oracle's own encoding of the
input (stream bytes, raw bytes, code lengths) and the oracle decodes it to
the input; every byte of the buffer is covered by the FNV-1a hash (published
algorithm, computed independently here); a plan whose chunk bits disagree
with its group starts is refused even when the hash is made to match."""
import ctypes
import os

import numpy as np
import pytest
import torch

import lossless_entropy_coded_canonical_b200 as dfw
import workloads


def _u16(spec) -> np.ndarray:
    return np.concatenate([workloads.as_u16_numpy(t) for t in workloads.generate_block(spec, "cpu")])


def fnv1a64(b: bytes) -> int:
    h = 0xCBF29CE484222325
    for x in b:
        h = ((h ^ x) * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    return h


def _read(buf: np.ndarray):
    t, v = dfw.Table(), dfw.ContainerView()
    st = dfw.lib().dfw_container_read(buf.ctypes.data, buf.size, ctypes.byref(t), ctypes.byref(v))
    return st, t, v


CASES = {
    "tensor": lambda: [_u16(workloads.scaled(workloads.c1(), 70_001))],
    "block": lambda: [workloads.as_u16_numpy(t) for t in
                      workloads.generate_block(workloads.scaled(workloads.c3(), 150_000), "cpu")],
    "heavy_tails": lambda: [_u16(workloads.scaled(workloads.c2(), 40_000))],
    "long_codes": lambda: [_u16(workloads.scaled(workloads.c4("b"), 90_000))],
    "one_exponent": lambda: [((np.arange(5000) % 2 << 15) | (120 << 7) | (np.arange(5000) % 128)).astype(np.uint16)],
    "empty": lambda: [np.zeros(0, np.uint16)],
}


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("with_plan", [False, True])
def test_round_trip_is_the_oracles_encoding(oracle, tmp_path, name, with_plan):
    parts = CASES[name]()
    u = np.concatenate(parts) if parts else np.zeros(0, np.uint16)
    enc = dfw.encode_multi([torch.from_numpy(p.view(np.int16)) for p in parts], 32) if len(parts) > 1 \
        else dfw.encode(parts[0])
    pl = dfw.plan_lanes(enc) if with_plan else None
    path = os.path.join(tmp_path, "a.dfw")
    size = dfw.save(path, enc, pl)
    assert size == os.path.getsize(path)
    k = len(parts)
    assert size == dfw.lib().dfw_container_bytes(ctypes.byref(enc.table), k, int(with_plan))
    got, gpl = dfw.load(path)
    oenc = oracle.encode(u)
    assert np.array_equal(got.stream.numpy(), oenc.stream)
    assert np.array_equal(got.mant.numpy()[: u.size], oenc.mant)
    assert np.array_equal(got.lengths, oenc.lengths)
    assert got.n == u.size and got.total_bits == oenc.total_bits
    if k > 1:
        assert np.array_equal(got.tensor_offsets, np.cumsum([0] + [p.size for p in parts]).astype(np.uint64))
    if with_plan:
        assert gpl is not None
        m = 32 * int(pl.info.n_groups)  # (an empty tensor's plan keeps a one-entry placeholder)
        assert torch.equal(gpl.chunk_bits[:m], pl.chunk_bits[:m]) and torch.equal(gpl.group_start, pl.group_start)
        assert torch.equal(gpl.lut, pl.lut) and bytes(gpl.info) == bytes(pl.info)
    else:
        assert gpl is None


def _container(tmp_path, with_plan=True) -> np.ndarray:
    enc = dfw.encode(_u16(workloads.scaled(workloads.c1(), 50_000)))
    path = os.path.join(tmp_path, "c.dfw")
    dfw.save(path, enc, dfw.plan_lanes(enc) if with_plan else None)
    return np.fromfile(path, dtype=np.uint8)


def test_hash_covers_every_byte(tmp_path):
    buf = _container(tmp_path)
    assert _read(buf)[0] == dfw.OK
    assert int.from_bytes(buf[-8:].tobytes(), "little") == fnv1a64(buf[:-8].tobytes())
    rng = np.random.default_rng(0)
    for pos in list(rng.choice(buf.size - 8, 40, replace=False)) + [0, 9, 60, buf.size - 9]:
        b = buf.copy()
        b[pos] ^= 1 << int(rng.integers(0, 8))
        # a flipped version field reads as another format (refused as such)
        assert _read(b)[0] == (dfw.EINVAL if 8 <= pos < 12 else dfw.ECORRUPT), pos


def test_header_checks(tmp_path):
    buf = _container(tmp_path, with_plan=False)
    assert _read(buf[:-1])[0] == dfw.ECORRUPT  # truncated
    assert _read(np.concatenate([buf, np.zeros(16, np.uint8)]))[0] == dfw.ECORRUPT  # trailing bytes
    b = buf.copy()
    b[8] = 2  # another format version, hash made to match
    b[-8:] = np.frombuffer(fnv1a64(b[:-8].tobytes()).to_bytes(8, "little"), np.uint8)
    assert _read(b)[0] == dfw.EINVAL
    b = buf.copy()
    b[56 + 120] = 0  # a code length removed: no longer a complete code
    b[-8:] = np.frombuffer(fnv1a64(b[:-8].tobytes()).to_bytes(8, "little"), np.uint8)
    assert _read(b)[0] == dfw.ECORRUPT


def test_plan_must_agree_with_itself(tmp_path):
    buf = _container(tmp_path)
    st, t, v = _read(buf)
    assert st == dfw.OK and v.has_plan
    b = buf.copy()
    cb = b[v.chunk_bits_at: v.chunk_bits_at + 64].view(np.uint16)
    cb[3] += 1  # one chunk claims a bit more; group starts unchanged
    b[-8:] = np.frombuffer(fnv1a64(b[:-8].tobytes()).to_bytes(8, "little"), np.uint8)
    assert _read(b)[0] == dfw.ECORRUPT


@pytest.mark.gpu
def test_loaded_container_decodes_on_the_gpu(tmp_path):
    u = np.concatenate([workloads.as_u16_numpy(t) for t in
                        workloads.generate_block(workloads.scaled(workloads.c5()[1], 3_000_000), "cpu")])
    enc = dfw.encode(u)
    path = os.path.join(tmp_path, "g.dfw")
    dfw.save(path, enc, dfw.plan_lanes(enc))
    got, pl = dfw.load(path)
    out = dfw.decode_lanes(dfw.DeviceLanes.upload(got, pl, "cuda"))
    dfw.check()
    assert np.array_equal(workloads.as_u16_numpy(out), u)
