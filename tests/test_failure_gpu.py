"""Failure detection without a GPU fault.

A bounded device-side wait that runs out is made to happen by lowering the
library's wait limit to 0 through its test hook: the row transform's first
waits then give up, the kernel sets the device error word, lets its own copies
in flight land and exits, and qwha_check_stream_status reports
QWHA_ERR_TIMEOUT. The context stays usable: the next call, with the limit put
back, gives the normal result. A failed CUDA call is injected on the host: the
entry point returns QWHA_ERR_CUDA and names the failure, and the library keeps
working afterwards. Nothing here faults, traps or hangs the GPU."""

import ctypes

import numpy as np
import pytest

import oracle
from _util import TOL_BF16, bf16_dev, host, rel_fro
from workloads import f32_to_bf16_bits, rng_for

pytestmark = pytest.mark.gpu

QWHA_OK, QWHA_ERR_CUDA, QWHA_ERR_TIMEOUT = 0, 5, 6


def _lib():
    import walsh_hadamard_sparse_b200._lib as L

    return L.lib()


def _stream():
    import torch

    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _input(rows, n):
    x = rng_for(70, "failure", rows, n).standard_normal((rows, n)).astype(np.float32)
    return x, bf16_dev(f32_to_bf16_bits(x))


def test_wait_that_runs_out_reports_timeout_and_the_context_recovers():
    import torch
    import walsh_hadamard_sparse_b200 as W

    h = _lib()
    rows, n = 8192, 4096
    xh, x = _input(rows, n)
    z_ref = W.fwht(x, n)
    assert h.qwha_check_stream_status(_stream()) == QWHA_OK
    z = torch.zeros_like(x)
    old = h.qwha_debug_wait_limit_ns(0)
    try:
        assert old == 2_000_000_000
        W.fwht(x, n, out=z)  # enqueued; the waits give up on the device
        rc = h.qwha_check_stream_status(_stream())
        msg = h.qwha_last_error()
    finally:
        assert h.qwha_debug_wait_limit_ns(old) == 0
    assert rc == QWHA_ERR_TIMEOUT, (rc, msg)
    assert b"gave up" in msg
    assert h.qwha_check_stream_status(_stream()) == QWHA_OK  # the word was cleared
    z2 = W.fwht(x, n)
    assert h.qwha_check_stream_status(_stream()) == QWHA_OK
    assert torch.equal(z2.view(torch.int16), z_ref.view(torch.int16))
    sel = np.arange(0, rows, 911)
    want = oracle.fwht(xh[sel].astype(np.float64), n)
    assert rel_fro(host(z2[torch.as_tensor(sel).cuda()]), want) <= TOL_BF16


def test_injected_cuda_failure_is_reported_and_the_library_recovers():
    import torch
    import walsh_hadamard_sparse_b200 as W

    h = _lib()
    rows, n = 512, 1024
    _, x = _input(rows, n)
    z_ref = W.fwht(x, n)
    torch.cuda.synchronize()
    h.qwha_debug_fail_cuda_checks(1)
    try:
        with pytest.raises(W.QwhaError) as ei:
            W.fwht(x, n)
    finally:
        h.qwha_debug_fail_cuda_checks(0)
    assert ei.value.status == QWHA_ERR_CUDA
    assert "injected failure" in str(ei.value)
    z = W.fwht(x, n)
    assert h.qwha_check_stream_status(_stream()) == QWHA_OK
    assert torch.equal(z.view(torch.int16), z_ref.view(torch.int16))
