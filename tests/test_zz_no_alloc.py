"""The encoder entry point that allocates no device memory.

dfw_encode_device_noalloc serves callers that cannot allocate device memory
when they encode (a runtime that reserves all of the GPU's memory at start-up,
or code that must not call cudaMalloc); its scratch is an array inside the
library rather than a caller buffer.  Two calls in a row on different inputs
must each give exactly what dfw_encode_device gives with its own scratch
buffer: same raw bytes, chunk bit counts, group starts, code table and plan
info, and, after dfw_pack_device, the same stream.  The second call passing
also shows that the shared array is cleared between calls.  A second test
checks the property itself: after a warm-up call, a call leaves the device's
free memory and torch's allocator unchanged.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import lossless_entropy_coded_canonical_b200 as dfw
import workloads
from lossless_entropy_coded_canonical_b200 import LanesInfo, Table

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dfw.lib()


def _encode_via_abi(x: torch.Tensor, noalloc: bool):
    """One encode through the C ABI; outputs start as garbage so that any
    byte the call fails to write shows up in the comparison."""
    lib = dfw.lib()
    n, dev = x.numel(), x.device
    n_groups = -(-(-(-n // 64)) // 32)
    mant = torch.full((dfw.mant_bytes(n),), 0xA5, dtype=torch.uint8, device=dev)
    chunk_bits = torch.full((32 * n_groups,), -1, dtype=torch.int16, device=dev)
    group_start = torch.full((n_groups + 1,), -1, dtype=torch.int64, device=dev)
    table, info = Table(), LanesInfo()
    sh = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    if noalloc:
        st = lib.dfw_encode_device_noalloc(x.data_ptr(), n, 32, mant.data_ptr(), chunk_bits.data_ptr(),
                                           group_start.data_ptr(), ctypes.byref(table), ctypes.byref(info), sh)
    else:
        scratch = torch.empty(int(lib.dfw_encode_device_scratch_bytes(n)), dtype=torch.uint8, device=dev)
        st = lib.dfw_encode_device(x.data_ptr(), n, 32, mant.data_ptr(), chunk_bits.data_ptr(),
                                   group_start.data_ptr(), scratch.data_ptr(), scratch.numel(),
                                   ctypes.byref(table), ctypes.byref(info), sh)
    assert st == dfw.OK, dfw.lib().dfw_strerror(st)
    stream = torch.empty(int(table.stream_bytes), dtype=torch.uint8, device=dev)
    st = lib.dfw_pack_device(x.data_ptr(), ctypes.byref(table), ctypes.byref(info), group_start.data_ptr(),
                             stream.data_ptr(), stream.numel(), sh)
    assert st == dfw.OK, dfw.lib().dfw_strerror(st)
    torch.cuda.synchronize()
    return {"mant": mant.cpu(), "chunk_bits": chunk_bits.cpu(), "group_start": group_start.cpu(),
            "stream": stream.cpu(), "table": bytes(table), "info": bytes(info)}


def test_noalloc_matches_regular_entry_point_two_calls_in_a_row():
    a = torch.cat([t.reshape(-1) for t in workloads.generate_block(workloads.c1(), "cuda")])
    b = torch.cat([t.reshape(-1) for t in
                   workloads.generate_block(workloads.scaled(workloads.c2(), 3_000_017), "cuda")])
    got = [_encode_via_abi(a, noalloc=True), _encode_via_abi(b, noalloc=True)]  # two calls in a row
    want = [_encode_via_abi(a, noalloc=False), _encode_via_abi(b, noalloc=False)]
    for g, w in zip(got, want):
        for key in ("mant", "chunk_bits", "group_start", "stream"):
            assert torch.equal(g[key], w[key]), key
        assert g["table"] == w["table"] and g["info"] == w["info"]
    # the two inputs differ, so a stale histogram in the shared array would show
    assert got[0]["table"] != got[1]["table"]
    # and the result decodes back to the input
    for x, g in zip((a, b), got):
        t = Table.from_buffer_copy(g["table"])
        info = LanesInfo.from_buffer_copy(g["info"])
        lut = torch.empty(int(info.lut_words), dtype=torch.int32)
        assert dfw.lib().dfw_lanes_lut(ctypes.byref(t), ctypes.byref(info), lut.data_ptr()) == dfw.OK
        dl = dfw.DeviceLanes(g["stream"].cuda(), g["mant"].cuda(), lut.cuda(), g["chunk_bits"].cuda(),
                             g["group_start"].cuda(), t, info)
        out = dfw.decode_lanes(dl)
        dfw.check()
        assert np.array_equal(workloads.as_u16_numpy(out), workloads.as_u16_numpy(x))


def test_noalloc_call_allocates_no_device_memory():
    """What the entry point exists for: once a warm-up call has placed the
    library's code and array on the device, a call changes neither the
    device's free memory (cudaMemGetInfo) nor torch's allocator, and its
    result still equals the regular entry point's.  The outputs are
    allocated before the measurement starts."""
    lib = dfw.lib()
    x = torch.cat([t.reshape(-1) for t in workloads.generate_block(workloads.c1(), "cuda")])
    n, dev = x.numel(), x.device
    n_groups = -(-(-(-n // 64)) // 32)
    mant = torch.empty(dfw.mant_bytes(n), dtype=torch.uint8, device=dev)
    chunk_bits = torch.empty(32 * n_groups, dtype=torch.int16, device=dev)
    group_start = torch.empty(n_groups + 1, dtype=torch.int64, device=dev)
    table, info = Table(), LanesInfo()
    sh = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)

    def call():
        st = lib.dfw_encode_device_noalloc(x.data_ptr(), n, 32, mant.data_ptr(), chunk_bits.data_ptr(),
                                           group_start.data_ptr(), ctypes.byref(table), ctypes.byref(info), sh)
        assert st == dfw.OK, lib.dfw_strerror(st)
        torch.cuda.synchronize()

    call()  # warm-up: module loading may place code and the array on the device here
    free0, alloc0 = torch.cuda.mem_get_info(dev)[0], torch.cuda.memory_allocated(dev)
    call()
    free1, alloc1 = torch.cuda.mem_get_info(dev)[0], torch.cuda.memory_allocated(dev)
    assert alloc1 == alloc0
    assert free1 == free0
    want = _encode_via_abi(x, noalloc=False)
    assert torch.equal(mant.cpu(), want["mant"]) and torch.equal(group_start.cpu(), want["group_start"])
    assert bytes(table) == want["table"] and bytes(info) == want["info"]
