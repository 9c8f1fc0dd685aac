"""The C-ABI library loads without a GPU and exports every declared symbol."""

import ctypes
import os
import subprocess
import sys

from _util import HEADER, ROOT, header_functions

LIB = os.path.join(ROOT, "walsh_hadamard_sparse_b200", "libqwha.so")


def _ensure_built():
    if not os.path.exists(LIB):
        subprocess.check_call([sys.executable, os.path.join(ROOT, "walsh_hadamard_sparse_b200", "build.py")])


def test_library_exports_every_header_symbol():
    _ensure_built()
    h = ctypes.CDLL(LIB)
    names = header_functions()
    assert len(names) >= 12
    missing = [n for n in names if not hasattr(h, n)]
    assert not missing, f"declared in include/qwha.h but not exported: {missing}"


def test_binding_covers_header():
    _ensure_built()
    import walsh_hadamard_sparse_b200._lib as L

    assert set(header_functions()) == set(L.exported_symbols())


def test_status_strings_and_host_checks():
    _ensure_built()
    import walsh_hadamard_sparse_b200._lib as L

    h = L.lib()
    assert h.qwha_status_string(0) == b"ok"
    assert b"sm_100a" in h.qwha_version()
    # argument checks run on the host before any CUDA call: no GPU needed
    assert h.qwha_fwht(0, None, None, 4, 256, 3, None) == 1  # had_block not a power of two
    assert b"had_block" in h.qwha_last_error()
    assert h.qwha_fwht(0, None, None, 4, 96, 64, None) == 1  # 64 does not divide 96
    assert h.qwha_fwht(0, None, None, 4, 256, 256, None) == 1  # NULL x
    assert h.qwha_fwht(0, ctypes.c_void_p(8), ctypes.c_void_p(4096), 4, 256, 256, None) == 2  # misaligned
    assert h.qwha_fwht(7, None, None, 4, 256, 256, None) == 1  # bad dtype
    assert h.qwha_fwht(0, None, None, 0, 256, 256, None) == 0  # nothing to do
    tile = int(next(l.split()[2] for l in open(HEADER) if l.startswith("#define QWHA_TILE")))
    assert h.qwha_plan_tiles(4096, 14336) == -(-4096 // tile) * -(-14336 // tile)
