"""CPU oracle for entropy-coded bf16 weights -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never imports,
links or executes anything here, and nothing here imports the product.

``oracle.c`` holds the arithmetic (plain C, one bit at a time); this module
compiles it with gcc on first use (or via :func:`build`) and marshals numpy
arrays through ctypes.  See the header comment of ``oracle.c`` for the
sources and the readings R1..R6 the oracle follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

OK, EINVAL, ECAP, ENOMEM, ECORRUPT = 0, 1, 2, 3, 4

_lib = None


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compiles oracle.c into liboracle.so next to it (plain -O2, untuned)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-shared", "-fPIC", "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u8p = ctypes.POINTER(ctypes.c_uint8)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        u32p = ctypes.POINTER(ctypes.c_uint32)
        u64p = ctypes.POINTER(ctypes.c_uint64)
        u64 = ctypes.c_uint64
        lib.oracle_split.argtypes = [u16p, u64, u8p, u8p]
        lib.oracle_split.restype = None
        lib.oracle_join.argtypes = [ctypes.c_uint8, ctypes.c_uint8]
        lib.oracle_join.restype = ctypes.c_uint16
        lib.oracle_histogram.argtypes = [u8p, u64, u64p]
        lib.oracle_histogram.restype = None
        lib.oracle_code_lengths.argtypes = [u64p, ctypes.c_int, u8p]
        lib.oracle_code_lengths.restype = ctypes.c_int
        lib.oracle_canonical_codes.argtypes = [u8p, u32p]
        lib.oracle_canonical_codes.restype = None
        lib.oracle_stream_bytes.argtypes = [u64]
        lib.oracle_stream_bytes.restype = u64
        lib.oracle_pack.argtypes = [u8p, u64, u8p, u32p, u8p, u64, u64p]
        lib.oracle_pack.restype = ctypes.c_int
        lib.oracle_encode.argtypes = [u16p, u64, ctypes.c_int, u8p, u64, u8p, u8p, u64p]
        lib.oracle_encode.restype = ctypes.c_int
        lib.oracle_decode.argtypes = [u8p, u64, u8p, ctypes.c_int, u8p, u64, u16p]
        lib.oracle_decode.restype = ctypes.c_int
        lib.oracle_decode_symbols.argtypes = [u8p, u64, u8p, u64, u64, u8p]
        lib.oracle_decode_symbols.restype = ctypes.c_int
        lib.oracle_n_windows.argtypes = [u64, u64]
        lib.oracle_n_windows.restype = u64
        lib.oracle_aux.argtypes = [u8p, u64, u8p, u64, u64, u64, u8p, u64p]
        lib.oracle_aux.restype = ctypes.c_int
        lib.oracle_chunk_aux.argtypes = [u8p, u64, u8p, u64, u64, u64, u32p, u64p]
        lib.oracle_chunk_aux.restype = ctypes.c_int
        lib.oracle_rans_freqs.argtypes = [u64p, ctypes.c_int, u32p]
        lib.oracle_rans_freqs.restype = ctypes.c_int
        lib.oracle_rans_encode.argtypes = [u8p, u64, u32p, ctypes.c_int, ctypes.c_uint32, ctypes.c_uint32, u8p, u64,
                                           u64p, u64p]
        lib.oracle_rans_encode.restype = ctypes.c_int
        lib.oracle_rans_decode.argtypes = [u8p, u64p, u64, u32p, ctypes.c_int, ctypes.c_uint32, ctypes.c_uint32, u8p]
        lib.oracle_rans_decode.restype = ctypes.c_int
        _lib = lib
    return _lib


def _p(a: np.ndarray, ct):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ct))


def _check(rc: int, what: str):
    if rc != OK:
        raise OracleError(f"{what} failed with status {rc}")


def _u16(x) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(x))
    if a.dtype != np.uint16:
        a = a.view(np.uint16) if a.dtype.itemsize == 2 else a.astype(np.uint16)
    return a.reshape(-1)


def split(u) -> tuple[np.ndarray, np.ndarray]:
    u = _u16(u)
    e = np.empty(u.size, np.uint8)
    m = np.empty(u.size, np.uint8)
    _load().oracle_split(_p(u, ctypes.c_uint16), u.size, _p(e, ctypes.c_uint8), _p(m, ctypes.c_uint8))
    return e, m


def join(e: int, m: int) -> int:
    return int(_load().oracle_join(e, m))


def histogram(e: np.ndarray) -> np.ndarray:
    e = np.ascontiguousarray(e, dtype=np.uint8)
    h = np.zeros(256, np.uint64)
    _load().oracle_histogram(_p(e, ctypes.c_uint8), e.size, _p(h, ctypes.c_uint64))
    return h


def code_lengths(hist, cap: int = 32) -> np.ndarray:
    h = np.ascontiguousarray(np.asarray(hist, dtype=np.uint64).reshape(256))
    ln = np.zeros(256, np.uint8)
    _check(_load().oracle_code_lengths(_p(h, ctypes.c_uint64), cap, _p(ln, ctypes.c_uint8)), "code_lengths")
    return ln


def code_lengths_status(hist, cap: int) -> int:
    h = np.ascontiguousarray(np.asarray(hist, dtype=np.uint64).reshape(256))
    ln = np.zeros(256, np.uint8)
    return int(_load().oracle_code_lengths(_p(h, ctypes.c_uint64), cap, _p(ln, ctypes.c_uint8)))


def canonical_codes(lengths) -> np.ndarray:
    ln = np.ascontiguousarray(np.asarray(lengths, dtype=np.uint8).reshape(256))
    c = np.zeros(256, np.uint32)
    _load().oracle_canonical_codes(_p(ln, ctypes.c_uint8), _p(c, ctypes.c_uint32))
    return c


def stream_bytes(total_bits: int) -> int:
    return int(_load().oracle_stream_bytes(total_bits))


class Encoded:
    """The oracle's encoding of one tensor (or one concatenation)."""

    def __init__(self, stream, mant, lengths, total_bits, n, single_symbol):
        self.stream = stream
        self.mant = mant
        self.lengths = lengths
        self.total_bits = total_bits
        self.n = n
        self.single_symbol = single_symbol

    @property
    def n_symbols(self) -> int:
        return int(np.count_nonzero(self.lengths)) if self.total_bits else (1 if self.n else 0)


def encode(u, cap: int = 32) -> Encoded:
    u = _u16(u)
    n = u.size
    cap_bytes = 4 * n + 128
    stream = np.zeros(cap_bytes, np.uint8)
    mant = np.zeros(max(n, 1), np.uint8)
    ln = np.zeros(256, np.uint8)
    tb = np.zeros(1, np.uint64)
    _check(
        _load().oracle_encode(_p(u, ctypes.c_uint16), n, cap, _p(stream, ctypes.c_uint8), cap_bytes,
                              _p(mant, ctypes.c_uint8), _p(ln, ctypes.c_uint8), _p(tb, ctypes.c_uint64)),
        "encode")
    total_bits = int(tb[0])
    single = -1
    if n and total_bits == 0:
        single = int((u[0] >> 7) & 0xFF)
    return Encoded(stream[: stream_bytes(total_bits)].copy(), mant[:n].copy(), ln, total_bits, n, single)


def decode(enc: Encoded) -> np.ndarray:
    out = np.zeros(max(enc.n, 1), np.uint16)
    mant = np.ascontiguousarray(enc.mant if enc.n else np.zeros(1, np.uint8), dtype=np.uint8)
    stream = np.ascontiguousarray(enc.stream if enc.stream.size else np.zeros(1, np.uint8), dtype=np.uint8)
    ln = np.ascontiguousarray(enc.lengths, dtype=np.uint8)
    _check(_load().oracle_decode(_p(stream, ctypes.c_uint8), enc.total_bits, _p(ln, ctypes.c_uint8),
                                 enc.single_symbol, _p(mant, ctypes.c_uint8), enc.n, _p(out, ctypes.c_uint16)),
           "decode")
    return out[: enc.n]


def decode_raw(stream, total_bits, lengths, single_symbol, mant, n) -> tuple[int, np.ndarray]:
    """Decode returning (status, out) without raising (for corrupt inputs)."""
    out = np.zeros(max(n, 1), np.uint16)
    mant = np.ascontiguousarray(mant if n else np.zeros(1, np.uint8), dtype=np.uint8)
    stream = np.ascontiguousarray(stream if len(stream) else np.zeros(1, np.uint8), dtype=np.uint8)
    ln = np.ascontiguousarray(lengths, dtype=np.uint8)
    rc = _load().oracle_decode(_p(stream, ctypes.c_uint8), total_bits, _p(ln, ctypes.c_uint8), single_symbol,
                               _p(mant, ctypes.c_uint8), n, _p(out, ctypes.c_uint16))
    return int(rc), out[:n]


def decode_symbols(stream, total_bits, lengths, start_bit: int, count: int) -> np.ndarray:
    out = np.zeros(max(count, 1), np.uint8)
    stream = np.ascontiguousarray(stream, dtype=np.uint8)
    ln = np.ascontiguousarray(lengths, dtype=np.uint8)
    _check(_load().oracle_decode_symbols(_p(stream, ctypes.c_uint8), total_bits, _p(ln, ctypes.c_uint8),
                                         start_bit, count, _p(out, ctypes.c_uint8)), "decode_symbols")
    return out[:count]


def n_windows(total_bits: int, W: int) -> int:
    return int(_load().oracle_n_windows(total_bits, W))


def aux(enc: Encoded, W: int, T: int) -> tuple[np.ndarray, np.ndarray]:
    """(gap[n_windows] u8, out_start[n_tiles + 1] u64) for window W bytes, T windows per tile."""
    nwin = n_windows(enc.total_bits, W)
    ntiles = (nwin + T - 1) // T
    gap = np.zeros(max(nwin, 1), np.uint8)
    out_start = np.zeros(ntiles + 1, np.uint64)
    stream = np.ascontiguousarray(enc.stream if enc.stream.size else np.zeros(1, np.uint8), dtype=np.uint8)
    ln = np.ascontiguousarray(enc.lengths, dtype=np.uint8)
    _check(_load().oracle_aux(_p(stream, ctypes.c_uint8), enc.total_bits, _p(ln, ctypes.c_uint8), enc.n, W, T,
                              _p(gap, ctypes.c_uint8), _p(out_start, ctypes.c_uint64)), "aux")
    return gap[:nwin], out_start


def chunk_aux(enc: Encoded, M: int = 64, G: int = 32) -> tuple[np.ndarray, np.ndarray]:
    """(chunk_bits[n_groups * G] u32, group_start[n_groups + 1] u64) for
    chunks of M codewords and groups of G chunks (reading R7)."""
    n_chunks = (enc.n + M - 1) // M
    n_groups = (n_chunks + G - 1) // G
    bits = np.zeros(max(n_groups * G, 1), np.uint32)
    starts = np.zeros(n_groups + 1, np.uint64)
    stream = np.ascontiguousarray(enc.stream if enc.stream.size else np.zeros(1, np.uint8), dtype=np.uint8)
    ln = np.ascontiguousarray(enc.lengths, dtype=np.uint8)
    _check(_load().oracle_chunk_aux(_p(stream, ctypes.c_uint8), enc.total_bits, _p(ln, ctypes.c_uint8), enc.n, M, G,
                                    _p(bits, ctypes.c_uint32), _p(starts, ctypes.c_uint64)), "chunk_aux")
    return bits[: n_groups * G], starts


# ---------------------------------------------------------------- y = W x

def bf16_values(u) -> np.ndarray:
    """Exact float64 values of bf16 bit patterns: a bf16 is the upper half of
    an IEEE binary32 whose lower 16 bits are zero."""
    u = np.ascontiguousarray(_u16(u))
    return (u.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def gemv(w, rows: int, cols: int, x) -> np.ndarray:
    """y = W x in float64 for the row-major bf16 matrix W (rows x cols bit
    patterns, e.g. the oracle's decode) and the bf16 vector x (cols).  Every
    product of two bf16 values is exact in float64 (8 + 8 significand bits);
    the sums use numpy's float64 matrix product as a library step."""
    W = bf16_values(w).reshape(rows, cols)
    return W @ bf16_values(x)


def gemv_abs(w, rows: int, cols: int, x) -> np.ndarray:
    """sum_j |W[i, j] x[j]| per row: the scale of the rounding-error bound of
    any fp32 summation of the products."""
    W = np.abs(bf16_values(w).reshape(rows, cols))
    return W @ np.abs(bf16_values(x))


# ---------------------------------------------------------------- rANS variant

RANS_SCALE_BITS = 12
RANS_LANES = 32
RANS_BLOCK = 8192


def rans_freqs(hist, scale_bits: int = RANS_SCALE_BITS) -> np.ndarray:
    """Quantised frequencies summing to 2^scale_bits (reading R9 of oracle.c)."""
    h = np.ascontiguousarray(hist, dtype=np.uint64)
    f = np.zeros(256, np.uint32)
    _check(_load().oracle_rans_freqs(_p(h, ctypes.c_uint64), scale_bits, _p(f, ctypes.c_uint32)), "rans_freqs")
    return f


class RansEncoded:
    """The oracle's rANS encoding: stream bytes, block byte offsets, the
    quantised frequencies, the raw bytes and the coding parameters."""

    def __init__(self, stream, block_start, freq, mant, n, scale_bits, lanes, block_syms):
        self.stream, self.block_start, self.freq, self.mant = stream, block_start, freq, mant
        self.n, self.scale_bits, self.lanes, self.block_syms = n, scale_bits, lanes, block_syms


def rans_encode_symbols(e, freq, scale_bits=RANS_SCALE_BITS, lanes=RANS_LANES, block_syms=RANS_BLOCK):
    e = np.ascontiguousarray(e, dtype=np.uint8)
    freq = np.ascontiguousarray(freq, dtype=np.uint32)
    n = e.size
    n_blocks = (n + block_syms - 1) // block_syms
    cap = 2 * n + n_blocks * (4 * lanes + 16) + 16
    out = np.zeros(cap, np.uint8)
    starts = np.zeros(n_blocks + 1, np.uint64)
    nb = np.zeros(1, np.uint64)
    _check(_load().oracle_rans_encode(_p(e if n else np.zeros(1, np.uint8), ctypes.c_uint8), n,
                                      _p(freq, ctypes.c_uint32), scale_bits, lanes, block_syms,
                                      _p(out, ctypes.c_uint8), cap, _p(starts, ctypes.c_uint64),
                                      _p(nb, ctypes.c_uint64)), "rans_encode")
    return out[: int(nb[0])].copy(), starts


def rans_decode_symbols(stream, block_start, n, freq, scale_bits=RANS_SCALE_BITS, lanes=RANS_LANES,
                        block_syms=RANS_BLOCK):
    e = np.zeros(max(n, 1), np.uint8)
    stream = np.ascontiguousarray(stream if len(stream) else np.zeros(1, np.uint8), dtype=np.uint8)
    starts = np.ascontiguousarray(block_start, dtype=np.uint64)
    freq = np.ascontiguousarray(freq, dtype=np.uint32)
    rc = _load().oracle_rans_decode(_p(stream, ctypes.c_uint8), _p(starts, ctypes.c_uint64), n,
                                    _p(freq, ctypes.c_uint32), scale_bits, lanes, block_syms, _p(e, ctypes.c_uint8))
    return int(rc), e[:n]


def rans_encode(u, scale_bits=RANS_SCALE_BITS, lanes=RANS_LANES, block_syms=RANS_BLOCK) -> RansEncoded:
    e, m = split(u)
    freq = rans_freqs(histogram(e), scale_bits)
    stream, starts = rans_encode_symbols(e, freq, scale_bits, lanes, block_syms)
    return RansEncoded(stream, starts, freq, m, e.size, scale_bits, lanes, block_syms)


def rans_decode(enc: RansEncoded) -> np.ndarray:
    rc, e = rans_decode_symbols(enc.stream, enc.block_start, enc.n, enc.freq, enc.scale_bits, enc.lanes,
                                enc.block_syms)
    _check(rc, "rans_decode")
    return (((enc.mant.astype(np.uint16) & 0x80) << 8) | (e.astype(np.uint16) << 7)
            | (enc.mant.astype(np.uint16) & 0x7F)).astype(np.uint16)
