"""The C-ABI library loads without a GPU and exports every function that
include/dfw.h declares, with matching Python declarations."""
import os
import re
import subprocess

import lossless_entropy_coded_canonical_b200 as dfw
from lossless_entropy_coded_canonical_b200 import _abi
from lossless_entropy_coded_canonical_b200.build import LIB, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(dfw_[a-z_0-9]+)\s*\(", src))
    return names


def test_library_exports_every_declared_symbol():
    build()
    out = subprocess.run(["nm", "-D", "--defined-only", LIB], capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    declared = declared_functions()
    assert declared, "no declarations found"
    missing = declared - exported
    assert not missing, f"declared but not exported: {sorted(missing)}"
    assert declared == set(_abi.SIGNATURES), "Python signatures out of step with the header"
    lib = dfw.lib()
    for name in declared:
        assert getattr(lib, name) is not None


def test_strerror_covers_every_status():
    for st in range(7):
        assert dfw.lib().dfw_strerror(st).decode() not in ("", "unknown status")
    assert dfw.lib().dfw_strerror(99).decode() == "unknown status"


def test_struct_layouts_match_header():
    import ctypes
    assert ctypes.sizeof(dfw.Table) == 4 + 4 + 8 + 8 + 8 + 4 + 4 + 256
    assert ctypes.sizeof(dfw.PlanInfo) == 4 + 4 + 8 + 8 + 8 + 4 + 4 + 4 + 4
