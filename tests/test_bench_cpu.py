"""The bench's roofline bookkeeping on the host (no GPU): which measured peak a stage is compared
with, the work the fractions are computed from, and the DRAM traffic the line reports."""

import importlib.util
import os

from _util import ROOT


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


PEAKS = {"hbm_gbs": 6540.2, "bf16_tflops": 1609.6, "bf16_tflops_sustained": 1360.5, "sm_max_mhz": 1965.0,
         "_source": "measured"}


def test_tensor_peak_follows_the_timed_region():
    """A short timed region (the driver's 20 steps, ~15 ms) is compared with the burst GEMM peak; a region of a
    second or more (at the power cap) with the sustained one."""
    b = _bench()
    peak, unit, note = b.peak_for("tensor", PEAKS, 0.015)
    assert (peak, unit) == (1609.6, "TFLOP/s") and "burst" in note
    peak, _, note = b.peak_for("tensor", PEAKS, 3.0)
    assert peak == 1360.5 and "sustained" in note
    assert b.peak_for("hbm", PEAKS, 0.015)[:2] == (6540.2, "GB/s")
    alu, unit, _ = b.peak_for("alu", PEAKS)
    assert unit == "TFLOP/s" and abs(alu - 148 * 128 * 2 * 1965e6 / 1e12) < 1e-9


def test_stage_work_of_the_q_proj_step():
    """Algorithmic work per call: 2 T d_in d_out per GEMM, 2 p T for the sparse products (and for the dc GEMM's
    method work), 4 bytes per element for the bf16 transform."""
    b = _bench()
    spec = b.CONFIGS["q_proj"][0]
    T, di, do, p = spec.T, spec.d_in, spec.d_out, spec.p
    for st in ("gemm_fwd", "gemm_bwd", "gemm_dc"):
        kind, work, _ = b.stage_work(st, spec, T, spec.bits, "dense")
        assert kind == "tensor" and work == 2.0 * T * di * do
    for st in ("spmm_fwd", "sddmm_dc", "gather_bwd"):
        kind, work, _ = b.stage_work(st, spec, T, spec.bits, "sparse")
        assert kind == "alu" and work == 2.0 * p * T
    kind, work, nbytes = b.stage_work("fwht_fwd", spec, T, spec.bits, "sparse")
    assert kind == "hbm" and work == nbytes == 4.0 * T * di
    mkind, mwork = b.METHOD_WORK["gemm_dc"](spec, T)
    assert mkind == "alu" and mwork == 2.0 * p * T


def test_traffic_is_reported_only_for_unchanged_kernels():
    """The per-launch DRAM bytes come from the committed capture and are dropped (None) for a stage whose kernel
    sources hash differently from the capture's."""
    import json

    b = _bench()
    d = json.load(open(os.path.join(ROOT, "profiles", "ncu_traffic.json")))
    for path in ("dense", "sparse"):
        for stage, rec in d[path].items():
            expect = rec["dram_bytes_per_launch"] if rec["source_sha"] == b.source_sha(b.KERNEL_SOURCES[stage]) else None
            assert b.ncu_traffic(path, stage) == expect
    assert b.ncu_traffic("dense", "no_such_stage") is None
