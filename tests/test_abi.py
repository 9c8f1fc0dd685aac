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


def test_host_checks_of_init_variants_and_refinement():
    """The selection, refinement and split-AdaAlloc entry points reject bad arguments on the host, before any CUDA
    call (no GPU needed), and name the problem."""
    _ensure_built()
    import walsh_hadamard_sparse_b200._lib as L

    h = L.lib()
    P = ctypes.c_void_p
    dummy = P(4096)
    # p above d_out * d_in
    assert h.qwha_init_select_global(dummy, 4, 8, 8, 33, 0, 7, dummy, dummy, dummy, dummy, dummy, 1 << 20, None) == 1
    # unknown selection rule
    assert h.qwha_init_select_global(dummy, 4, 8, 8, 8, 5, 7, dummy, dummy, dummy, dummy, dummy, 1 << 20, None) == 1
    # d_in not a multiple of 8 (row strides of the tensor-core operands)
    assert h.qwha_calib_hessian(dummy, 16, 12, dummy, None) == 1
    assert h.qwha_calib_hessian(dummy, 0, 64, dummy, None) == 1  # no calibration rows
    assert h.qwha_refine_values(dummy, 4, 12, 4, dummy, ctypes.c_float(0.0), dummy, dummy, 8, dummy, dummy, 1 << 20,
                                None) == 1
    assert h.qwha_refine_values(dummy, 4, 64, 64, dummy, ctypes.c_float(-1.0), dummy, dummy, 8, dummy, dummy, 1 << 20,
                                None) == 1  # negative damping
    assert b"damp" in h.qwha_last_error()
    # workspace below the need
    assert h.qwha_refine_values(dummy, 4, 64, 64, dummy, ctypes.c_float(0.0), dummy, dummy, 8, dummy, dummy, 16,
                                None) == 4
    # split AdaAlloc: bad remainder mode, p out of range
    assert h.qwha_init_budgets(dummy, 4, 8, 16, 2, 9, dummy, dummy, dummy, 1 << 20, None) == 1
    assert h.qwha_init_budgets(dummy, 4, 8, 4, 2, 0, dummy, dummy, dummy, 1 << 20, None) == 1  # p < 2 * d_out
    assert h.qwha_init_select(dummy, 4, 96, 64, dummy, dummy, 8, dummy, dummy, None) == 1  # 64 does not divide 96
    assert h.qwha_workspace_size(7, 64, 64, 100, 0, 0) > 0 and h.qwha_workspace_size(6, 64, 64, 100, 0, 0) > 0


def test_sparse_forward_needs_entry_workspace():
    """The sparse products write their (staged-row, value) pairs, ordered for the shared-memory gather, into the
    caller's workspace (8 bytes per coefficient, plus the padding of the groups of segments), so the adapter-only
    sparse forward needs a workspace too; without one it is refused on the host, before any CUDA call (no GPU
    needed)."""
    _ensure_built()
    import walsh_hadamard_sparse_b200._lib as L

    h = L.lib()
    d, p, T = 64, 100, 16
    need = h.qwha_workspace_size(0, d, d, p, T, 0)  # QWHA_OP_FWD, adapter only
    assert need >= 8 * p
    assert h.qwha_workspace_size(0, d, d, p, T, 1) >= need + 4 * T * d  # plus the fp32 adapter term
    assert h.qwha_workspace_size(1, d, d, p, T, 0) >= 8 * p + 4 * T * d  # QWHA_OP_BWD: entries and dZ
    a = L.QwhaAdapter(d_in=d, d_out=d, had_block=d, algo=0, p=p, row_ptr=4096, col_idx=8192, coef=12288)
    buf = ctypes.c_void_p(16384)
    rc = h.qwha_adapter_fwd(ctypes.byref(a), None, 1, buf, T, ctypes.c_float(1.0), buf, buf, None, 0, None)
    assert rc == 4 and b"workspace" in h.qwha_last_error()


def test_debug_hooks_round_trip_on_the_host():
    """The test hooks only change host-side state: the wait limit is returned on the next set, and arming and
    disarming the injected failures needs no GPU."""
    _ensure_built()
    import walsh_hadamard_sparse_b200._lib as L

    h = L.lib()
    old = h.qwha_debug_wait_limit_ns(12345)
    assert old == 2_000_000_000
    assert h.qwha_debug_wait_limit_ns(old) == 12345
    h.qwha_debug_fail_cuda_checks(3)
    h.qwha_debug_fail_cuda_checks(0)
    assert h.qwha_fwht(0, None, None, 4, 256, 3, None) == 1  # host checks are not CUDA checks: unaffected


def test_sparse_workspace_covers_the_sliced_layout_and_the_transposes():
    """The sizes qwha_workspace_size reports cover the worst case of what the sparse kernels place there (no GPU):
    the sliced SpMM's entries (every group of 16 or 32 segments padded to its longest segment, at most the
    coefficients plus 32 entries per column of the row width, plus one step a group) and ranking tables, and in the
    backward the transposed dY and Z of the coefficient gradient (bf16, tokens rounded up to 64), which share a
    region with dZ."""
    _ensure_built()
    import walsh_hadamard_sparse_b200._lib as L

    h = L.lib()
    for d_out, d_in, p, T in ((2600, 8192, 65100, 50), (4616, 4096, 125296, 40), (64, 4096, 3, 1), (4096, 64, 4096, 129)):
        fwd = h.qwha_workspace_size(0, d_out, d_in, p, T, 0)
        bwd = h.qwha_workspace_size(1, d_out, d_in, p, T, 0)
        ent_fwd = 8 * (p + 32 * (d_in + 2) + 32 * ((d_out + 15) // 16))  # forward: segments are rows, width d_in
        ent_bwd = 8 * (p + 32 * (d_out + 2) + 32 * ((d_in + 15) // 16))  # gather: segments are columns, width d_out
        assert fwd >= max(ent_fwd, ent_bwd), (d_out, d_in)
        t64 = (T + 63) // 64 * 64
        region = max(4 * T * d_in, 2 * (d_out + d_in) * t64)  # dZ, or before it the transposed dY and Z
        assert bwd >= 16 * p * 4 + region + max(ent_fwd, ent_bwd), (d_out, d_in)
