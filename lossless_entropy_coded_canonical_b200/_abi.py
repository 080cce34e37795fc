"""ctypes declarations of the libdfw C ABI (include/dfw.h)."""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdfw.so")

OK, EINVAL, ECAP, ENOMEM, ECORRUPT, EALIGN, ECUDA = range(7)
ST_COUNT, ST_LUT, ST_RANGE, ST_TIMEOUT, ST_CHECK = 1, 2, 4, 8, 16  # device status bits (include/dfw.h DFW_ST_*)
FORMAT_VERSION = 1
MAX_CAP = 32


class DfwError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = lib().dfw_strerror(status).decode() if _lib is not None else str(status)
        super().__init__(f"{what}: {msg} (status {status})")


class Table(ctypes.Structure):
    _fields_ = [("version", ctypes.c_uint32), ("cap", ctypes.c_uint32), ("n", ctypes.c_uint64),
                ("total_bits", ctypes.c_uint64), ("stream_bytes", ctypes.c_uint64),
                ("n_symbols", ctypes.c_uint32), ("single_symbol", ctypes.c_uint32),
                ("len", ctypes.c_uint8 * 256)]


class PlanInfo(ctypes.Structure):
    _fields_ = [("window_bytes", ctypes.c_uint32), ("tile_windows", ctypes.c_uint32),
                ("n_windows", ctypes.c_uint64), ("n_tiles", ctypes.c_uint64),
                ("max_tile_symbols", ctypes.c_uint64), ("lut_words", ctypes.c_uint32),
                ("lut_tables", ctypes.c_uint32), ("fast_bits", ctypes.c_uint32), ("reserved", ctypes.c_uint32)]


class LanesInfo(ctypes.Structure):
    _fields_ = [("n_chunks", ctypes.c_uint64), ("n_groups", ctypes.c_uint64), ("chunk_symbols", ctypes.c_uint32),
                ("group_chunks", ctypes.c_uint32), ("max_group_bytes", ctypes.c_uint32), ("lut_words", ctypes.c_uint32),
                ("lut_tables", ctypes.c_uint32), ("fast_bits", ctypes.c_uint32)]


class LanesScope(ctypes.Structure):
    """dfw_lanes_scope: one scope of dfw_decode_lanes_seq."""
    _fields_ = [("d_stream", ctypes.c_void_p), ("d_mant", ctypes.c_void_p), ("d_lut", ctypes.c_void_p),
                ("d_chunk_bits", ctypes.c_void_p), ("d_group_start", ctypes.c_void_p),
                ("table", ctypes.POINTER(Table)), ("info", ctypes.POINTER(LanesInfo))]


class EncodeScope(ctypes.Structure):
    """dfw_encode_scope: one scope of dfw_encode_device_multi."""
    _fields_ = [("d_bf16", ctypes.c_void_p), ("n", ctypes.c_uint64), ("d_mant", ctypes.c_void_p),
                ("d_chunk_bits", ctypes.c_void_p), ("d_group_start", ctypes.c_void_p)]


class ContainerView(ctypes.Structure):
    """dfw_container_view: where dfw_container_read found each section."""
    _fields_ = [("k", ctypes.c_int32), ("has_plan", ctypes.c_int32), ("offsets_at", ctypes.c_uint64),
                ("stream_at", ctypes.c_uint64), ("mant_at", ctypes.c_uint64), ("chunk_bits_at", ctypes.c_uint64),
                ("group_start_at", ctypes.c_uint64)]


class RansTable(ctypes.Structure):
    _fields_ = [("version", ctypes.c_uint32), ("scale_bits", ctypes.c_uint32), ("lanes", ctypes.c_uint32),
                ("block_syms", ctypes.c_uint32), ("n", ctypes.c_uint64), ("n_blocks", ctypes.c_uint64),
                ("stream_bytes", ctypes.c_uint64), ("max_block_bytes", ctypes.c_uint32),
                ("reserved", ctypes.c_uint32), ("freq", ctypes.c_uint16 * 256)]


_lib = None

# name -> (restype, argtypes); the symbols include/dfw.h declares
_vp, _u64, _i = ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int
_TP, _IP, _LP = ctypes.POINTER(Table), ctypes.POINTER(PlanInfo), ctypes.POINTER(LanesInfo)
_RP = ctypes.POINTER(RansTable)
SIGNATURES = {
    "dfw_stream_bound": (_u64, [_u64]),
    "dfw_mant_bytes": (_u64, [_u64]),
    "dfw_encode": (_i, [_vp, _u64, _i, _vp, _u64, _vp, _u64, _TP, _i]),
    "dfw_encode_multi": (_i, [_vp, _vp, _i, _i, _vp, _u64, _vp, _u64, _TP, _vp, _i]),
    "dfw_plan_query": (_i, [_TP, ctypes.c_uint32, ctypes.c_uint32, _IP]),
    "dfw_plan": (_i, [_vp, _TP, _vp, _vp, _vp, _IP]),
    "dfw_decode": (_i, [_vp, _vp, _vp, _vp, _vp, _TP, _IP, _vp, _vp]),
    "dfw_decode_block": (_i, [_vp, _vp, _vp, _vp, _vp, _TP, _IP, _vp, _i, _vp, _u64, _vp]),
    "dfw_plan_lanes_query": (_i, [_TP, _LP]),
    "dfw_plan_lanes": (_i, [_vp, _TP, _vp, _vp, _vp, _LP]),
    "dfw_decode_lanes": (_i, [_vp, _vp, _vp, _vp, _vp, _TP, _LP, _vp, _vp]),
    "dfw_decode_lanes_seq": (_i, [_i, _vp, _vp, _vp]),
    "dfw_decode_lanes_seq_launches": (_i, [_i, _vp, _vp]),
    "dfw_status_bits": (_i, [_vp, ctypes.POINTER(ctypes.c_uint32)]),
    "dfw_checks_report": (_i, [ctypes.POINTER(ctypes.c_uint32), ctypes.POINTER(ctypes.c_uint32)]),
    "dfw_container_bytes": (_u64, [_TP, _i, _i]),
    "dfw_container_write": (_i, [_TP, _i, _vp, _vp, _vp, _vp, _vp, _vp, _u64]),
    "dfw_container_read": (_i, [_vp, _u64, _TP, ctypes.POINTER(ContainerView)]),
    "dfw_selftest_wait_timeout": (_i, [_vp]),
    "dfw_decode_gemv_lanes": (_i, [_vp, _vp, _vp, _vp, _vp, _TP, _LP, _i, _vp, _vp, _vp, _vp, _vp, _u64, _vp]),
    "dfw_encode_device_scratch_bytes": (_u64, [_u64]),
    "dfw_encode_device": (_i, [_vp, _u64, _i, _vp, _vp, _vp, _vp, _u64, _TP, _LP, _vp]),
    "dfw_pack_device": (_i, [_vp, _TP, _LP, _vp, _vp, _u64, _vp]),
    "dfw_lanes_lut": (_i, [_TP, _LP, _vp]),
    "dfw_encode_device_multi_staging_bytes": (_u64, [ctypes.c_uint32]),
    "dfw_encode_device_multi": (_i, [ctypes.c_uint32, _vp, _i, _vp, _u64, _vp, _u64, _vp, _vp, _vp]),
    "dfw_encode_device_noalloc": (_i, [_vp, _u64, _i, _vp, _vp, _vp, _TP, _LP, _vp]),
    "dfw_rans_stream_bound": (_u64, [_u64]),
    "dfw_rans_encode": (_i, [_vp, _vp, _i, _vp, _u64, _vp, _u64, _vp, _RP, _i]),
    "dfw_rans_decode": (_i, [_vp, _vp, _vp, _RP, _vp, _vp]),
    "dfw_check": (_i, [_vp]),
    "dfw_strerror": (ctypes.c_char_p, [_i]),
}


def lib_path() -> str:
    """The library this process uses: libdfw.so, or with DFW_LIBRARY=checks
    in the environment the checks build libdfw_checks.so (every copy range,
    shared-memory extent and output index checked before use)."""
    if os.environ.get("DFW_LIBRARY", "") == "checks":
        return os.path.join(os.path.dirname(LIB_PATH), "libdfw_checks.so")
    return LIB_PATH


def lib():
    """Loads the library from the package directory; fails loudly if absent."""
    global _lib
    if _lib is None:
        path = lib_path()
        if not os.path.exists(path):
            raise ImportError(f"{os.path.basename(path)} is not built ({path}); run "
                              "`python -m lossless_entropy_coded_canonical_b200.build`")
        handle = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def check(status: int, what: str):
    if status != OK:
        raise DfwError(status, what)
