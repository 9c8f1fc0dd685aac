"""The allocation-free coefficient gradient (qwha_coef_grad_noalloc).

Some callers cannot allocate device memory or pass a workspace (a framework
custom-op slot that only hands over inputs and outputs; a step that must not
call cudaMalloc). For them the library keeps the gradient's partial sums in a
static device array of its own. These tests call that entry point through the
C ABI and compare it with the dc of qwha_adapter_bwd on the same inputs, on two
calls in a row with different inputs (the shared array keeps the previous
call's contents, so the second call checks that it is cleared). Both run the
same coefficient-gradient kernels in the same order, so the results must agree
bit for bit; sampled entries are also checked against the oracle. The file is
named to be collected last."""

import ctypes

import numpy as np
import pytest

import oracle
from _util import TOL_BF16, TOL_F32, bf16_dev, rel_fro, to_dev
from workloads import bf16_bits_to_f32, f32_to_bf16_bits, random_pattern, rng_for

pytestmark = pytest.mark.gpu


def _noalloc_dc(a, dY, Z, T, alpha, dc):
    import torch
    import walsh_hadamard_sparse_b200._lib as L

    cs = a.c_struct()
    dt = 0 if dY.dtype == torch.float32 else 1
    rc = L.lib().qwha_coef_grad_noalloc(ctypes.byref(cs), dt, ctypes.c_void_p(dY.data_ptr()),
                                        ctypes.c_void_p(Z.data_ptr()), T, float(alpha),
                                        ctypes.c_void_p(dc.data_ptr()),
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc


def _act(a, dtype):
    return bf16_dev(f32_to_bf16_bits(a)) if dtype == "bf16" else to_dev(a)


@pytest.mark.parametrize(
    "d_in,d_out,n,T,p,dtype",
    [
        (1024, 768, 1024, 300, 768 * 24, "bf16"),
        (256, 256, 256, 64, 1024, "f32"),
        (4096, 4096, 4096, 8192, 524288, "bf16"),  # the q_proj layer's size
    ],
)
def test_noalloc_dc_matches_adapter_bwd_twice(d_in, d_out, n, T, p, dtype):
    import torch
    import walsh_hadamard_sparse_b200 as W

    g = rng_for(50, "noalloc", d_in, d_out, T, p)
    rp, ci, cf = random_pattern(d_out, d_in, p=p, rng=g)
    a = W.plan_build(W.Adapter(d_in, d_out, n, p, to_dev(rp), to_dev(ci), to_dev(cf)))
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    rows = oracle.csr_rows(rp)
    for call in range(2):  # two calls in a row, different inputs each time
        X = g.standard_normal((T, d_in)).astype(np.float32)
        dYh = g.standard_normal((T, d_out)).astype(np.float32)
        if dtype == "bf16":
            X, dYh = bf16_bits_to_f32(f32_to_bf16_bits(X)), bf16_bits_to_f32(f32_to_bf16_bits(dYh))
        Xd, dYd = _act(X, dtype), _act(dYh, dtype)
        Z = W.fwht(Xd, n)
        ref, _ = W.adapter_bwd(a, dYd, Z, 0.9, want_dx=False)
        dc = torch.full((p,), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc_dc(a, dYd, Z, T, 0.9, dc) == 0
        torch.cuda.synchronize()
        assert torch.equal(dc.view(torch.int32), ref.view(torch.int32)), call
        sel = np.sort(g.choice(p, min(p, 48), replace=False))
        want = oracle.adapter_bwd_dc(X, dYh, rows[sel], ci[sel], n, 0.9)
        assert rel_fro(dc.cpu().numpy()[sel], want) <= tol, call


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import torch
    import walsh_hadamard_sparse_b200 as W
    import walsh_hadamard_sparse_b200._lib as L

    buf = torch.zeros(1024, dtype=torch.int32, device="cuda")
    a = W.Adapter(4096, 4096, 4096, 4096 * 4096 // 2, buf, buf, buf.float(), buf, buf, buf, buf, buf, buf)
    dc = torch.zeros(16, device="cuda")
    x = torch.zeros(16, device="cuda", dtype=torch.bfloat16)
    rc = _noalloc_dc(a, x, x, 8192, 1.0, dc)
    assert rc == 4  # QWHA_ERR_WORKSPACE, nothing launched
    assert b"static scratch" in L.lib().qwha_last_error()
    torch.cuda.synchronize()
    assert torch.count_nonzero(dc).item() == 0
