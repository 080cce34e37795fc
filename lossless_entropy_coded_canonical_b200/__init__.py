"""Lossless entropy-coded bf16 weights, decoded on B200 (sm_100a).

Thin Python binding over libdfw (include/dfw.h).  Every step of encoding,
planning and decoding runs in the native library; this module only marshals
torch tensors into pointers and sizes.  PyTorch provides host/device memory
and CUDA streams.  There is no fallback path: if libdfw.so is missing, the
first call raises ImportError.

Typical use::

    enc = encode(weights_bf16_cpu)            # host: split, code, pack
    pl = plan(enc)                            # host: gap/out_start aux + LUT
    dev = DeviceCompressed.upload(enc, pl)    # H2D (caller's memory: torch)
    w = decode(dev)                           # GPU: bit-exact bf16 tensor
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import numpy as np
import torch

from ._abi import (EALIGN, ECAP, ECORRUPT, ECUDA, EINVAL, ENOMEM, OK, ST_COUNT, ST_LUT, ST_RANGE, ST_TIMEOUT,
                   ContainerView, DfwError, EncodeScope, LanesInfo, LanesScope, PlanInfo, RansTable, Table, check as _check, lib)

__all__ = ["encode", "encode_multi", "plan", "DeviceCompressed", "decode", "decode_block", "check",
           "plan_lanes", "LanesPlan", "DeviceLanes", "decode_lanes", "decode_lanes_seq", "LanesInfo",
           "encode_device", "encode_device_multi", "encode_device_scratch_bytes", "decode_gemv_lanes",
           "rans_encode", "RansEncoded", "DeviceRans", "rans_decode", "RansTable", "save", "load",
           "Encoded", "Plan", "Table", "PlanInfo", "DfwError", "lib", "mant_bytes", "stream_bound",
           "OK", "EINVAL", "ECAP", "ENOMEM", "ECORRUPT", "EALIGN", "ECUDA"]


def _ptr(t) -> int:
    if isinstance(t, torch.Tensor):
        return t.data_ptr()
    return int(t.ctypes.data)


def _as_u16_host(x) -> torch.Tensor:
    if isinstance(x, np.ndarray):
        x = torch.from_numpy(np.ascontiguousarray(x).view(np.int16))
    if x.is_cuda:
        raise ValueError("encode takes host tensors")
    if x.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise TypeError(f"expected bf16 bit patterns, got {x.dtype}")
    return x.contiguous().reshape(-1)


def _stream_handle(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(int(stream.cuda_stream))


def mant_bytes(n: int) -> int:
    return int(lib().dfw_mant_bytes(n))


def stream_bound(n: int) -> int:
    return int(lib().dfw_stream_bound(n))


@dataclass
class Encoded:
    """Host result of dfw_encode / dfw_encode_multi."""
    stream: torch.Tensor  # uint8[table.stream_bytes]
    mant: torch.Tensor  # uint8[mant_bytes(n)]
    table: Table
    tensor_offsets: np.ndarray | None = None  # uint64[k + 1] for a block

    @property
    def n(self) -> int:
        return int(self.table.n)

    @property
    def total_bits(self) -> int:
        return int(self.table.total_bits)

    @property
    def lengths(self) -> np.ndarray:
        return np.frombuffer(bytes(self.table.len), dtype=np.uint8).copy()


def _encode_call(fn, n, args_before, args_after, cap, n_threads, pin) -> tuple:
    mant = torch.empty(mant_bytes(n), dtype=torch.uint8, pin_memory=pin)
    table = Table()
    cap_bytes = n + 4096  # enough for <= 8 bits/weight; retried with the exact size otherwise
    stream = torch.empty(cap_bytes, dtype=torch.uint8, pin_memory=pin)
    st = fn(*args_before, cap, _ptr(stream), cap_bytes, _ptr(mant), mant.numel(), ctypes.byref(table),
            *args_after, n_threads)
    if st == ENOMEM and table.stream_bytes > cap_bytes:
        cap_bytes = int(table.stream_bytes)
        stream = torch.empty(cap_bytes, dtype=torch.uint8, pin_memory=pin)
        st = fn(*args_before, cap, _ptr(stream), cap_bytes, _ptr(mant), mant.numel(), ctypes.byref(table),
                *args_after, n_threads)
    _check(st, "dfw_encode")
    used = int(table.stream_bytes)
    if used < cap_bytes // 2:  # do not keep a mostly empty (possibly pinned) buffer alive
        stream = torch.empty(used, dtype=torch.uint8, pin_memory=pin).copy_(stream[:used])
    return stream[:used], mant, table


def encode(bf16, cap: int = 32, n_threads: int = 0, pin: bool = False) -> Encoded:
    """Encodes one host bf16 tensor (any shape; flattened)."""
    u = _as_u16_host(bf16)
    stream, mant, table = _encode_call(lib().dfw_encode, u.numel(), [_ptr(u), u.numel()], [], cap, n_threads, pin)
    return Encoded(stream, mant, table)


def encode_multi(tensors, cap: int = 32, n_threads: int = 0, pin: bool = False) -> Encoded:
    """Encodes k host bf16 tensors with one shared code table (one block)."""
    us = [_as_u16_host(t) for t in tensors]
    k = len(us)
    ptrs = (ctypes.c_void_p * k)(*[_ptr(u) for u in us])
    sizes = (ctypes.c_uint64 * k)(*[u.numel() for u in us])
    offs = np.zeros(k + 1, dtype=np.uint64)
    n = int(sum(u.numel() for u in us))
    stream, mant, table = _encode_call(lib().dfw_encode_multi, n, [ptrs, sizes, k], [_ptr(offs)], cap,
                                       n_threads, pin)
    return Encoded(stream, mant, table, offs)


@dataclass
class Plan:
    """Host result of dfw_plan: aux arrays, LUT image and plan shape."""
    gap: torch.Tensor  # uint8[n_tiles * tile_windows]: n_windows gaps, then zero padding
    out_start: torch.Tensor  # int64 view of uint64[n_tiles + 1]
    lut: torch.Tensor  # int32 view of uint32[lut_words]
    info: PlanInfo


def plan(enc: Encoded, window_bytes: int = 8, tile_windows: int = 256, pin: bool = False,
         fast_bits: int = 0) -> Plan:
    info = PlanInfo()
    info.fast_bits = fast_bits  # 0 = library default
    _check(lib().dfw_plan_query(ctypes.byref(enc.table), window_bytes, tile_windows, ctypes.byref(info)),
           "dfw_plan_query")
    gap = torch.empty(int(info.n_tiles) * int(info.tile_windows), dtype=torch.uint8, pin_memory=pin)
    out_start = torch.empty(int(info.n_tiles) + 1, dtype=torch.int64, pin_memory=pin)
    lut = torch.empty(int(info.lut_words), dtype=torch.int32, pin_memory=pin)
    _check(lib().dfw_plan(_ptr(enc.stream), ctypes.byref(enc.table), _ptr(gap), _ptr(out_start), _ptr(lut),
                          ctypes.byref(info)), "dfw_plan")
    return Plan(gap, out_start, lut, info)


@dataclass
class DeviceCompressed:
    """A compressed tensor or block resident in device memory."""
    stream: torch.Tensor
    mant: torch.Tensor
    lut: torch.Tensor
    gap: torch.Tensor
    out_start: torch.Tensor
    table: Table
    info: PlanInfo
    tensor_offsets: np.ndarray | None = None

    @staticmethod
    def upload(enc: Encoded, pl: Plan, device="cuda", non_blocking: bool = False) -> "DeviceCompressed":
        mv = lambda t: t.to(device, non_blocking=non_blocking)  # noqa: E731
        return DeviceCompressed(mv(enc.stream), mv(enc.mant), mv(pl.lut), mv(pl.gap), mv(pl.out_start),
                                enc.table, pl.info, enc.tensor_offsets)

    @property
    def n(self) -> int:
        return int(self.table.n)

    def compressed_bytes(self, with_aux: bool = True) -> int:
        b = int(self.table.stream_bytes) + self.n + 256  # stream + raw bytes + length table
        if with_aux:
            b += self.gap.numel() + 8 * self.out_start.numel() + 4 * self.lut.numel()
        return b

    def algorithmic_bytes(self) -> int:
        """Bytes a decode must move: coded stream + gap + out_start read,
        one raw byte read and one bf16 written per weight."""
        return (int(self.table.stream_bytes) + self.gap.numel() + 8 * self.out_start.numel()
                + 4 * self.lut.numel() + self.n + 2 * self.n)


def _decode_args(dc: DeviceCompressed):
    return (_ptr(dc.stream), _ptr(dc.mant), _ptr(dc.lut), _ptr(dc.gap), _ptr(dc.out_start),
            ctypes.byref(dc.table), ctypes.byref(dc.info))


def decode(dc: DeviceCompressed, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Decodes into ``out`` (bf16, n elements, on the device) asynchronously."""
    if out is None:
        out = torch.empty(dc.n, dtype=torch.bfloat16, device=dc.mant.device)
    if out.numel() < dc.n or not out.is_contiguous():
        raise ValueError("out must be a contiguous tensor of at least n elements")
    _check(lib().dfw_decode(*_decode_args(dc), _ptr(out), _stream_handle(stream)), "dfw_decode")
    return out


def decode_block(dc: DeviceCompressed, scratch: torch.Tensor | None = None, stream=None):
    """Decodes a block (k tensors, one table) into one scratch buffer; returns
    (scratch, [view of tensor i])."""
    offs = dc.tensor_offsets if dc.tensor_offsets is not None else np.array([0, dc.n], np.uint64)
    k = offs.size - 1
    if scratch is None:
        scratch = torch.empty(dc.n, dtype=torch.bfloat16, device=dc.mant.device)
    _check(lib().dfw_decode_block(*_decode_args(dc), _ptr(offs), k, _ptr(scratch), scratch.numel(),
                                  _stream_handle(stream)), "dfw_decode_block")
    views = [scratch[int(offs[i]): int(offs[i + 1])] for i in range(k)]
    return scratch, views


@dataclass
class LanesPlan:
    """Host result of dfw_plan_lanes (known-start chunks)."""
    chunk_bits: torch.Tensor  # int16 view of uint16[32 * n_groups]
    group_start: torch.Tensor  # int64 view of uint64[n_groups + 1]
    lut: torch.Tensor  # int32 view of uint32[lut_words]
    info: LanesInfo


def plan_lanes(enc: Encoded, pin: bool = False, fast_bits: int = 0) -> LanesPlan:
    info = LanesInfo()
    info.fast_bits = fast_bits
    _check(lib().dfw_plan_lanes_query(ctypes.byref(enc.table), ctypes.byref(info)), "dfw_plan_lanes_query")
    cb = torch.empty(max(32 * int(info.n_groups), 1), dtype=torch.int16, pin_memory=pin)
    gs = torch.empty(int(info.n_groups) + 1, dtype=torch.int64, pin_memory=pin)
    lut = torch.empty(int(info.lut_words), dtype=torch.int32, pin_memory=pin)
    _check(lib().dfw_plan_lanes(_ptr(enc.stream), ctypes.byref(enc.table), _ptr(cb), _ptr(gs), _ptr(lut),
                                ctypes.byref(info)), "dfw_plan_lanes")
    return LanesPlan(cb, gs, lut, info)


@dataclass
class DeviceLanes:
    """A compressed tensor or block resident in device memory, known-start plan."""
    stream: torch.Tensor
    mant: torch.Tensor
    lut: torch.Tensor
    chunk_bits: torch.Tensor
    group_start: torch.Tensor
    table: Table
    info: LanesInfo
    tensor_offsets: np.ndarray | None = None

    @staticmethod
    def upload(enc: Encoded, pl: LanesPlan, device="cuda", non_blocking: bool = False) -> "DeviceLanes":
        mv = lambda t: t.to(device, non_blocking=non_blocking)  # noqa: E731
        return DeviceLanes(mv(enc.stream), mv(enc.mant), mv(pl.lut), mv(pl.chunk_bits), mv(pl.group_start),
                           enc.table, pl.info, enc.tensor_offsets)

    @property
    def n(self) -> int:
        return int(self.table.n)

    def compressed_bytes(self, with_aux: bool = True) -> int:
        b = int(self.table.stream_bytes) + self.n + 256
        if with_aux:
            b += 2 * self.chunk_bits.numel() + 8 * self.group_start.numel() + 4 * self.lut.numel()
        return b

    def algorithmic_bytes(self) -> int:
        """Stream + chunk_bits + group_start + LUT read, one raw byte read and
        one bf16 written per weight."""
        return (int(self.table.stream_bytes) + 2 * self.chunk_bits.numel() + 8 * self.group_start.numel()
                + 4 * self.lut.numel() + self.n + 2 * self.n)


def decode_lanes(dl: DeviceLanes, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Decodes with the known-start plan into ``out`` (bf16, n elements)."""
    if out is None:
        out = torch.empty(dl.n, dtype=torch.bfloat16, device=dl.mant.device)
    if out.numel() < dl.n or not out.is_contiguous():
        raise ValueError("out must be a contiguous tensor of at least n elements")
    _check(lib().dfw_decode_lanes(_ptr(dl.stream), _ptr(dl.mant), _ptr(dl.lut), _ptr(dl.chunk_bits),
                                  _ptr(dl.group_start), ctypes.byref(dl.table), ctypes.byref(dl.info), _ptr(out),
                                  _stream_handle(stream)), "dfw_decode_lanes")
    return out


def _scope_array(dls):
    arr = (LanesScope * len(dls))()
    for i, d in enumerate(dls):
        arr[i] = LanesScope(_ptr(d.stream), _ptr(d.mant), _ptr(d.lut), _ptr(d.chunk_bits), _ptr(d.group_start),
                            ctypes.pointer(d.table), ctypes.pointer(d.info))
    return arr


def decode_lanes_seq(dls, out: torch.Tensor, stream=None) -> torch.Tensor:
    """Decodes the scopes ``dls`` one after another into ``out``
    (``dfw_decode_lanes_seq``): the same result as ``decode_lanes`` on each
    in order, from one persistent launch per run of up to
    ``DFW_SEQ_MAX_SCOPES`` scopes.  ``out`` must hold the largest scope;
    returns it."""
    dls = list(dls)
    if not dls:
        return out
    if out.numel() < max(d.n for d in dls) or not out.is_contiguous():
        raise ValueError("out must be a contiguous tensor holding the largest scope")
    arr = _scope_array(dls)
    _check(lib().dfw_decode_lanes_seq(len(dls), arr, _ptr(out), _stream_handle(stream)), "dfw_decode_lanes_seq")
    return out


def decode_lanes_seq_launches(dls) -> int:
    """Kernel launches ``decode_lanes_seq`` makes for these scopes
    (``dfw_decode_lanes_seq_launches``; host only)."""
    dls = list(dls)
    n = ctypes.c_int(0)
    _check(lib().dfw_decode_lanes_seq_launches(len(dls), _scope_array(dls) if dls else None, ctypes.byref(n)),
           "dfw_decode_lanes_seq_launches")
    return int(n.value)


def decode_gemv_lanes(dl: DeviceLanes, xs, cols, ys=None, partial: torch.Tensor | None = None,
                      tensor_offsets=None, stream=None):
    """y_i = W_i x_i for every tensor of a scope, decoded on the fly
    (``dfw_decode_gemv_lanes``): the decoded weights are never written.
    ``xs``: one bf16 CUDA vector per tensor (cols[i] entries); ``cols``:
    columns per tensor (multiples of 64); returns fp32 ``ys`` (one per row)."""
    offs = dl.tensor_offsets if tensor_offsets is None else tensor_offsets
    if offs is None:
        offs = np.array([0, dl.n], dtype=np.uint64)
    offs = np.ascontiguousarray(np.asarray(offs, dtype=np.uint64))
    k = offs.size - 1
    cols = np.ascontiguousarray(np.asarray(cols, dtype=np.uint32))
    if len(xs) != k or cols.size != k:
        raise ValueError("one x and one column count per tensor")
    dev = dl.mant.device
    if ys is None:
        ys = [torch.empty(int(offs[i + 1] - offs[i]) // int(cols[i]), dtype=torch.float32, device=dev)
              for i in range(k)]
    if partial is None:
        partial = torch.empty(max(1, dl.n // 64), dtype=torch.float32, device=dev)
    xs = [x.contiguous() for x in xs]
    xp = (ctypes.c_void_p * k)(*[x.data_ptr() for x in xs])
    yp = (ctypes.c_void_p * k)(*[y.data_ptr() for y in ys])
    _check(lib().dfw_decode_gemv_lanes(_ptr(dl.stream), _ptr(dl.mant), _ptr(dl.lut), _ptr(dl.chunk_bits),
                                       _ptr(dl.group_start), ctypes.byref(dl.table), ctypes.byref(dl.info), k,
                                       _ptr(offs), _ptr(cols), xp, yp, _ptr(partial), partial.numel(),
                                       _stream_handle(stream)), "dfw_decode_gemv_lanes")
    return ys


def encode_device(x: torch.Tensor, cap: int = 32, fast_bits: int = 0, stream=None,
                  scratch: torch.Tensor | None = None) -> DeviceLanes:
    """Encodes a bf16 tensor that is already on the GPU (``dfw_encode_device``
    then ``dfw_pack_device``): the same stream bytes as :func:`encode`, the
    known-start plan made on the way, and the LUT image built on the host and
    uploaded.  Returns a :class:`DeviceLanes` ready for :func:`decode_lanes`.
    ``scratch`` (uint8, at least ``encode_device_scratch_bytes()``) may be
    passed to reuse one buffer across calls."""
    x, mant, chunk_bits, group_start = _device_outputs(x)
    dev, n = x.device, x.numel()
    need = encode_device_scratch_bytes()
    if scratch is None:
        scratch = torch.empty(need, dtype=torch.uint8, device=dev)
    if scratch.numel() * scratch.element_size() < need:
        raise ValueError(f"scratch needs {need} bytes")
    table, info = Table(), LanesInfo()
    info.fast_bits = fast_bits
    sh = _stream_handle(stream)
    _check(lib().dfw_encode_device(_ptr(x), n, cap, _ptr(mant), _ptr(chunk_bits), _ptr(group_start),
                                   _ptr(scratch), scratch.numel() * scratch.element_size(), ctypes.byref(table),
                                   ctypes.byref(info), sh), "dfw_encode_device")
    return _pack_device(x, mant, chunk_bits, group_start, table, info, sh)


def _device_outputs(x: torch.Tensor):
    if not x.is_cuda:
        raise ValueError("encode_device takes a CUDA tensor")
    if x.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise TypeError(f"expected bf16 bit patterns, got {x.dtype}")
    x = x.contiguous().reshape(-1)
    n = x.numel()
    n_groups = -(-(-(-n // 64)) // 32)
    return (x, torch.empty(mant_bytes(n), dtype=torch.uint8, device=x.device),
            torch.empty(32 * n_groups, dtype=torch.int16, device=x.device),
            torch.empty(n_groups + 1, dtype=torch.int64, device=x.device))


def _pack_device(x, mant, chunk_bits, group_start, table, info, sh) -> DeviceLanes:
    """Second call (dfw_pack_device) and the LUT image, after the first."""
    stream_buf = torch.empty(int(table.stream_bytes), dtype=torch.uint8, device=x.device)
    _check(lib().dfw_pack_device(_ptr(x), ctypes.byref(table), ctypes.byref(info), _ptr(group_start),
                                 _ptr(stream_buf), stream_buf.numel(), sh), "dfw_pack_device")
    lut = torch.empty(int(info.lut_words), dtype=torch.int32)
    _check(lib().dfw_lanes_lut(ctypes.byref(table), ctypes.byref(info), _ptr(lut.numpy())), "dfw_lanes_lut")
    return DeviceLanes(stream_buf, mant, lut.to(x.device), chunk_bits, group_start, table, info, None)


def encode_device_multi(xs, cap: int = 32, fast_bits: int = 0, stream=None,
                        pinned_staging: bool = True) -> list[DeviceLanes]:
    """Encodes several bf16 tensors already on the GPU, each with its own
    code (``dfw_encode_device_multi``, then ``dfw_pack_device`` per tensor):
    the host builds tensor i's code while the GPU runs tensor i + 1's
    histogram pass.  Each result equals :func:`encode_device` of that tensor
    alone.  ``pinned_staging=False`` reads the histograms back through
    pageable memory (same results, no overlap)."""
    outs = [_device_outputs(x) for x in xs]
    k = len(outs)
    if k == 0:
        return []
    dev = outs[0][0].device
    arr = (EncodeScope * k)()
    for i, (x, mant, cb, gs) in enumerate(outs):
        if x.device != dev:
            raise ValueError("all tensors must be on one device")
        arr[i] = EncodeScope(_ptr(x), x.numel(), _ptr(mant), _ptr(cb), _ptr(gs))
    scratch = torch.empty(k * encode_device_scratch_bytes(), dtype=torch.uint8, device=dev)
    staging = torch.empty(int(lib().dfw_encode_device_multi_staging_bytes(k)), dtype=torch.uint8,
                          pin_memory=pinned_staging)
    tables, infos = (Table * k)(), (LanesInfo * k)()
    for i in range(k):
        infos[i].fast_bits = fast_bits
    sh = _stream_handle(stream)
    _check(lib().dfw_encode_device_multi(k, arr, cap, _ptr(scratch), scratch.numel(), staging.data_ptr(),
                                         staging.numel(), tables, infos, sh), "dfw_encode_device_multi")
    res = []
    for i, (x, mant, cb, gs) in enumerate(outs):
        t, inf = Table.from_buffer_copy(tables[i]), LanesInfo.from_buffer_copy(infos[i])
        res.append(_pack_device(x, mant, cb, gs, t, inf, sh))
    return res


def encode_device_scratch_bytes() -> int:
    return int(lib().dfw_encode_device_scratch_bytes(0))


# ---------------------------------------------------------------- rANS variant

@dataclass
class RansEncoded:
    """Host result of dfw_rans_encode."""
    stream: torch.Tensor       # uint8[table.stream_bytes]
    mant: torch.Tensor         # uint8[mant_bytes(n)]
    block_start: torch.Tensor  # int64 view of uint64[n_blocks + 1]
    table: RansTable
    tensor_offsets: np.ndarray | None = None

    @property
    def n(self) -> int:
        return int(self.table.n)


def rans_encode(tensors, n_threads: int = 0, pin: bool = False) -> RansEncoded:
    """Encodes one host bf16 tensor, or several with one table, with the rANS
    variant of the exponent coder (``dfw_rans_encode``)."""
    if isinstance(tensors, (torch.Tensor, np.ndarray)):
        tensors = [tensors]
    us = [_as_u16_host(t) for t in tensors]
    k = len(us)
    n = int(sum(u.numel() for u in us))
    ptrs = (ctypes.c_void_p * max(k, 1))(*[_ptr(u) for u in us])
    sizes = (ctypes.c_uint64 * max(k, 1))(*[u.numel() for u in us])
    table = RansTable()
    cap = int(lib().dfw_rans_stream_bound(n))
    stream = torch.empty(max(cap, 16), dtype=torch.uint8, pin_memory=pin)
    mant = torch.empty(mant_bytes(n), dtype=torch.uint8, pin_memory=pin)
    nb = (n + 16383) // 16384
    starts = torch.empty(nb + 1, dtype=torch.int64, pin_memory=pin)
    _check(lib().dfw_rans_encode(ptrs, sizes, k, _ptr(stream), stream.numel(), _ptr(mant), mant.numel(),
                                 _ptr(starts), ctypes.byref(table), n_threads), "dfw_rans_encode")
    used = int(table.stream_bytes)
    stream = torch.empty(max(used, 16), dtype=torch.uint8, pin_memory=pin).copy_(
        torch.cat([stream[:used], torch.zeros(max(0, 16 - used), dtype=torch.uint8)]))
    offs = np.concatenate([[0], np.cumsum([u.numel() for u in us])]).astype(np.uint64)
    return RansEncoded(stream, mant, starts, table, offs)


@dataclass
class DeviceRans:
    """An rANS-coded tensor or block resident in device memory."""
    stream: torch.Tensor
    mant: torch.Tensor
    block_start: torch.Tensor
    table: RansTable
    tensor_offsets: np.ndarray | None = None

    @staticmethod
    def upload(enc: RansEncoded, device="cuda") -> "DeviceRans":
        return DeviceRans(enc.stream.to(device), enc.mant.to(device), enc.block_start.to(device), enc.table,
                          enc.tensor_offsets)

    @property
    def n(self) -> int:
        return int(self.table.n)

    def compressed_bytes(self, with_aux: bool = True) -> int:
        b = int(self.table.stream_bytes) + self.n + 512
        return b + (8 * self.block_start.numel() if with_aux else 0)

    def algorithmic_bytes(self) -> int:
        """Stream + block offsets read, one raw byte read and one bf16
        written per weight."""
        return int(self.table.stream_bytes) + 8 * self.block_start.numel() + 3 * self.n


def rans_decode(dr: DeviceRans, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(dr.n, dtype=torch.bfloat16, device=dr.mant.device)
    if out.numel() < dr.n or not out.is_contiguous():
        raise ValueError("out must be a contiguous tensor of at least n elements")
    _check(lib().dfw_rans_decode(_ptr(dr.stream), _ptr(dr.mant), _ptr(dr.block_start), ctypes.byref(dr.table),
                                 _ptr(out), _stream_handle(stream)), "dfw_rans_decode")
    return out


def check(stream=None) -> None:
    """Synchronises the stream and raises DfwError if a decode saw corruption."""
    _check(lib().dfw_check(_stream_handle(stream)), "dfw_check")


def check_status(stream=None) -> int:
    return int(lib().dfw_check(_stream_handle(stream)))


def status_bits(stream=None) -> tuple[int, int]:
    """(status, bits): dfw_check's result and the device status bits it read
    and cleared (ST_COUNT, ST_LUT, ST_RANGE, ST_TIMEOUT)."""
    bits = ctypes.c_uint32(0)
    st = int(lib().dfw_status_bits(_stream_handle(stream), ctypes.byref(bits)))
    return st, int(bits.value)


# ------------------------------------------------------------------ container

def save(path, enc: Encoded, plan: LanesPlan | None = None) -> int:
    """Writes an encoded tensor or block (and optionally its known-start
    plan) to ``path`` as one container (dfw_container_write); returns the
    number of bytes written."""
    k = 1 if enc.tensor_offsets is None else int(enc.tensor_offsets.size - 1)
    offs = None if enc.tensor_offsets is None else np.ascontiguousarray(enc.tensor_offsets, dtype=np.uint64)
    size = int(lib().dfw_container_bytes(ctypes.byref(enc.table), k, plan is not None))
    if size == 0:
        raise DfwError(EINVAL, "dfw_container_bytes")
    out = np.empty(size, dtype=np.uint8)
    cb = gs = None
    if plan is not None:
        cb, gs = _ptr(plan.chunk_bits.contiguous()), _ptr(plan.group_start.contiguous())
    _check(lib().dfw_container_write(ctypes.byref(enc.table), k, None if offs is None else _ptr(offs),
                                     _ptr(enc.stream.contiguous()), _ptr(enc.mant.contiguous()), cb, gs,
                                     _ptr(out), size), "dfw_container_write")
    with open(path, "wb") as f:
        f.write(out.tobytes())
    return size


def load(path):
    """Reads a container written by :func:`save`; returns (Encoded, LanesPlan
    or None), host tensors viewing the file's bytes (the LUT is rebuilt from
    the code lengths)."""
    with open(path, "rb") as f:
        buf = np.frombuffer(f.read(), dtype=np.uint8).copy()
    table, view = Table(), ContainerView()
    _check(lib().dfw_container_read(_ptr(buf), buf.size, ctypes.byref(table), ctypes.byref(view)),
           "dfw_container_read")
    raw = torch.from_numpy(buf)
    n, k = int(table.n), int(view.k)
    offs = buf[view.offsets_at: view.offsets_at + 8 * (k + 1)].view(np.uint64).copy()
    stream = raw[view.stream_at: view.stream_at + int(table.stream_bytes)]
    mant = raw[view.mant_at: view.mant_at + mant_bytes(n)]
    enc = Encoded(stream, mant, table, offs if k > 1 else None)
    if not view.has_plan:
        return enc, None
    info = LanesInfo()
    _check(lib().dfw_plan_lanes_query(ctypes.byref(table), ctypes.byref(info)), "dfw_plan_lanes_query")
    ng = int(info.n_groups)
    cb = torch.from_numpy(buf[view.chunk_bits_at: view.chunk_bits_at + 64 * ng].view(np.int16).copy())
    gs = torch.from_numpy(buf[view.group_start_at: view.group_start_at + 8 * (ng + 1)].view(np.int64).copy())
    if cb.numel() == 0:
        cb = torch.zeros(1, dtype=torch.int16)
    # the largest group span, as dfw_plan_lanes reports it
    g = gs.numpy().view(np.uint64)
    if ng:
        b0 = (g[:-1] >> np.uint64(3)) & ~np.uint64(15)
        b1 = (((g[1:] + np.uint64(7)) >> np.uint64(3)) + np.uint64(8 + 15)) & ~np.uint64(15)
        info.max_group_bytes = max(16, int((b1 - b0).max()))
    else:
        info.max_group_bytes = 16
    lut = torch.empty(int(info.lut_words), dtype=torch.int32)
    _check(lib().dfw_lanes_lut(ctypes.byref(table), ctypes.byref(info), _ptr(lut)), "dfw_lanes_lut")
    return enc, LanesPlan(cb, gs, lut, info)
