"""dfw_encode_device_multi: the encoder's first call for several tensors, each
with its own code, the host's share of one overlapped with the GPU's pass
over the next (needs a B200).

Every tensor's result must be the oracle's encoding of that tensor alone
(stream with padding, raw bytes, code lengths, chunk bit counts and group
starts), byte for byte what dfw_encode_device gives for it alone, and must
decode back to the input.  Argument errors are found before anything is
launched; a code error found half way leaves the stream idle.
"""
from __future__ import annotations

import ctypes

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


def _u16(block):
    return np.concatenate([workloads.as_u16_numpy(t) for t in workloads.generate_block(block)])


def _mixed() -> list[np.ndarray]:
    """Tensors of every kind in one call: Gaussian blocks, heavy tails,
    codewords up to 32 bits, one exponent, empty, sizes below one 8-weight
    load and just past one group."""
    rng = np.random.default_rng(77)
    single = ((rng.integers(0, 2, 100_003) << 15) | (119 << 7) | rng.integers(0, 128, 100_003)).astype(np.uint16)
    return [
        _u16(workloads.scaled(workloads.c1(), 300_001)),
        np.zeros(0, np.uint16),
        _u16(workloads.c4("b", 200_003)),
        rng.integers(0, 65536, size=1, dtype=np.uint64).astype(np.uint16),
        single,
        _u16(workloads.scaled(workloads.c2(), 150_001)),
        rng.integers(0, 65536, size=2049, dtype=np.uint64).astype(np.uint16),
        _u16(workloads.scaled(workloads.c3(), 1_000_003)),
        rng.integers(0, 65536, size=7, dtype=np.uint64).astype(np.uint16),
    ]


def _cuda_x(u: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(u).view(np.int16)).cuda()


def _same(a: dfw.DeviceLanes, b: dfw.DeviceLanes):
    assert bytes(a.table) == bytes(b.table) and bytes(a.info) == bytes(b.info)
    for f in ("stream", "mant", "chunk_bits", "group_start", "lut"):
        assert torch.equal(getattr(a, f), getattr(b, f)), f


def test_multi_is_each_tensors_own_encoding(oracle):
    us = _mixed()
    xs = [_cuda_x(u) for u in us]
    got = dfw.encode_device_multi(xs)
    dfw.check()
    assert len(got) == len(us)
    for i, (u, x, dl) in enumerate(zip(us, xs, got)):
        _same(dl, dfw.encode_device(x))
        oenc = oracle.encode(u)
        assert int(dl.table.total_bits) == oenc.total_bits, i
        assert np.array_equal(np.frombuffer(bytes(dl.table.len), np.uint8), oenc.lengths), i
        assert np.array_equal(dl.stream.cpu().numpy(), oenc.stream), i
        assert np.array_equal(dl.mant.cpu().numpy()[: u.size], oenc.mant), i
        if u.size:
            bits, starts = oracle.chunk_aux(oenc, 64, 32)
            assert np.array_equal(dl.chunk_bits.cpu().numpy().view(np.uint16).astype(np.uint32), bits), i
            assert np.array_equal(dl.group_start.cpu().numpy().view(np.uint64), starts), i
        out = dfw.decode_lanes(dl)
        dfw.check()
        assert np.array_equal(workloads.as_u16_numpy(out), u), i


def test_multi_pageable_staging_same_result():
    us = _mixed()[:6]
    xs = [_cuda_x(u) for u in us]
    for a, b in zip(dfw.encode_device_multi(xs), dfw.encode_device_multi(xs, pinned_staging=False)):
        _same(a, b)


@pytest.mark.parametrize("cap", [10, 16])
def test_multi_cap_binding(cap):
    us = [_u16(workloads.c4("b", 300_001)), _u16(workloads.c4("c", 200_001))]
    xs = [_cuda_x(u) for u in us]
    for x, dl in zip(xs, dfw.encode_device_multi(xs, cap)):
        _same(dl, dfw.encode_device(x, cap))
        assert max(bytes(dl.table.len)) <= cap


def _scopes(xs, outs):
    arr = (dfw.EncodeScope * len(xs))()
    for i, (x, (mant, cb, gs)) in enumerate(zip(xs, outs)):
        arr[i] = dfw.EncodeScope(x.data_ptr(), x.numel(), mant.data_ptr(), cb.data_ptr(), gs.data_ptr())
    return arr


def _outputs(x):
    n = x.numel()
    g = -(-(-(-n // 64)) // 32)
    return (torch.full((dfw.mant_bytes(n),), 0xAB, dtype=torch.uint8, device="cuda"),
            torch.full((32 * g,), 0x55, dtype=torch.int16, device="cuda"),
            torch.full((g + 1,), 7, dtype=torch.int64, device="cuda"))


def test_multi_checks_every_scope_before_launch():
    lib = dfw.lib()
    xs = [_cuda_x(u) for u in _mixed()[:4]]
    outs = [_outputs(x) for x in xs]
    before = [[t.clone() for t in o] for o in outs]
    k = len(xs)
    per = int(lib.dfw_encode_device_scratch_bytes(0))
    scratch = torch.empty(k * per, dtype=torch.uint8, device="cuda")
    staging = torch.empty(int(lib.dfw_encode_device_multi_staging_bytes(k)), dtype=torch.uint8, pin_memory=True)
    tables, infos = (dfw.Table * k)(), (dfw.LanesInfo * k)()

    def call(arr, cap=32, scratch_bytes=None, st_ptr=None, st_bytes=None, kk=k):
        return lib.dfw_encode_device_multi(kk, arr, cap, scratch.data_ptr(),
                                           scratch.numel() if scratch_bytes is None else scratch_bytes,
                                           staging.data_ptr() if st_ptr is None else st_ptr,
                                           staging.numel() if st_bytes is None else st_bytes, tables, infos, None)

    good = _scopes(xs, outs)
    assert lib.dfw_encode_device_multi(0, None, 32, None, 0, None, 0, None, None, None) == dfw.OK
    bad = _scopes(xs, outs)
    bad[2].d_mant += 1  # the third scope's raw-byte output misaligned
    assert call(bad) == dfw.EALIGN
    assert call(good, cap=0) == dfw.EINVAL
    assert call(good, cap=33) == dfw.EINVAL
    assert call(good, scratch_bytes=k * per - 1) == dfw.ENOMEM
    assert call(good, st_bytes=staging.numel() - 1) == dfw.ENOMEM
    assert call(good, st_ptr=staging.data_ptr() + 4) == dfw.EALIGN
    big = _scopes(xs, outs)
    big[1].n = 64 * 32 * (1 << 32)  # 2^32 chunks
    assert call(big) == dfw.EINVAL
    torch.cuda.synchronize()
    for o, b in zip(outs, before):
        for t, tb in zip(o, b):
            assert torch.equal(t, tb)
    # and the same arrays, corrected, encode
    assert call(good) == dfw.OK
    dfw.check()
    for i, x in enumerate(xs):
        one = dfw.encode_device(x)
        assert bytes(tables[i]) == bytes(one.table) and bytes(infos[i]) == bytes(one.info)
        if x.numel():
            assert torch.equal(outs[i][0], one.mant) and torch.equal(outs[i][2], one.group_start)


def test_multi_cap_error_half_way_leaves_stream_idle():
    """The second tensor has 256 distinct exponents, more than cap 7 allows:
    found only after its histogram pass, when the first tensor's work is
    already queued.  The call reports DFW_ECAP with nothing left running."""
    xs = [_cuda_x(_u16(workloads.scaled(workloads.c1(), 100_001))),
          torch.arange(0, 300 * 128, 128, dtype=torch.int32).to(torch.int16).cuda()]
    with pytest.raises(dfw.DfwError) as ei:
        dfw.encode_device_multi(xs, 7)
    assert ei.value.status == dfw.ECAP
    assert torch.cuda.current_stream().query()
    dfw.check()
    _same(dfw.encode_device_multi(xs[:1], 7)[0], dfw.encode_device(xs[0], 7))


def test_multi_full_size_llama3_blocks():
    """Embedding-sized tensor and two transformer blocks of the 8B-shaped
    model at full size, one call: each equals dfw_encode_device of it alone
    and decodes back to its input."""
    blocks = workloads.c5()
    xs = [torch.cat([t.reshape(-1) for t in workloads.generate_block(b, "cuda")]) for b in (blocks[0], *blocks[1:3])]
    got = dfw.encode_device_multi(xs)
    dfw.check()
    for x, dl in zip(xs, got):
        _same(dl, dfw.encode_device(x))
        out = dfw.decode_lanes(dl)
        dfw.check()
        assert torch.equal(out.view(torch.int16), x.view(torch.int16))
        del out
