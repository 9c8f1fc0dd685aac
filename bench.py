#!/usr/bin/env python
"""Throughput of one Walsh-Hadamard-adapted linear layer (forward + backward) on B200.

A step is one pass of the whole hot path over one batch of seeded synthetic
tokens: the forward (Z = X H and Y = X W_Q^T + alpha Z F^T) and the backward
(dc at E and dX = dY W_Q + alpha dY F H) of one adapted layer with its base
GEMMs, and, with N > 1 GPUs, the data-parallel sum of the coefficient
gradients (NCCL all-reduce). The headline runs the dense algorithm (the
adapter folded into W_eff = W_Q + alpha F H and three tcgen05 GEMMs, dc from
the sampled epilogue of dY^T Z); the same run times the sparse algorithm
(segment SpMM, tiled SDDMM, CSC gather on the FMA units) under paths.sparse.
The workload is the LLaMA-7B q_proj shape: d_in = d_out = 4096, 8192 tokens
per GPU (16 x 512), 4-bit group-128 round-to-nearest base weight, p = 524288
coefficients chosen by AdaAlloc. AdaAlloc and the whole-matrix selection
rules (one-off per layer) are timed separately.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun every rank runs its own tokens; rank 0 prints one JSON line.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import CONFIGS, layer_inputs, rank_rows  # noqa: E402

METRIC = "WHA adapter fwd+bwd tokens/s per layer; achieved HBM GB/s vs B200 peak"
UNIT = "tokens/s"
WORKLOAD = "q_proj"
FLUSH_BYTES = 512 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}
ALU_LANES_PER_SM = 128  # fp32 FMA lanes per SM (4 partitions x 32)

# the stages of a step that exist only because of the adapter (the rest is the frozen layer's own GEMMs)
ADAPTER_STAGES = {"dense": ["weff", "gemm_dc"],
                  "sparse": ["fwht_fwd", "spmm_fwd", "sddmm_dc", "gather_bwd", "fwht_bwd"]}

KERNEL_SOURCES = {
    "fwht_fwd": ["fwht.cu", "fwht_body.cuh", "bulk.cuh"], "fwht_bwd": ["fwht.cu", "fwht_body.cuh", "bulk.cuh"],
    "spmm_fwd": ["sparse.cu"], "gather_bwd": ["sparse.cu"], "sddmm_dc": ["sparse.cu"], "dequant": ["dequant.cu"],
    "gemm_fwd": ["gemm.cu", "fwht_body.cuh"], "gemm_bwd": ["gemm.cu", "fwht_body.cuh"],
    "gemm_dc": ["gemm.cu", "fwht_body.cuh"], "weff": ["fwht.cu", "dense.cu", "fwht_body.cuh", "bulk.cuh"],
    "init_alloc": ["init.cu"], "plan_build": ["plan.cu"],
}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        d["_source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["_source"] = "fallback"
    return d


def source_sha(files):
    h = hashlib.sha256()
    for f in files + ["common.cuh"]:
        h.update(open(os.path.join(ROOT, "walsh_hadamard_sparse_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(path_name, stage):
    """DRAM bytes (read + write) per launch of `stage` on the `path_name` path ("dense" or "sparse"), from the
    committed ncu summary, if the kernel's sources are unchanged since it was taken; else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path)).get(path_name, {}).get(stage)
    if not d or d.get("source_sha") != source_sha(KERNEL_SOURCES.get(stage, [])):
        return None
    return d.get("dram_bytes_per_launch")


# --------------------------------------------------------------------------- work per stage


def stage_work(stage, spec, T, bits, algo="dense"):
    """(bound, algorithmic work per stage call, HBM bytes per stage call) for the layer of `spec` at T tokens on
    the `algo` path. bound is hbm (work = bytes), tensor or alu (work = FLOP); None for stages without a model."""
    di, do, p = spec.d_in, spec.d_out, spec.p
    # the sparse path's GEMMs also read the fp32 adapter term in their epilogue; the dense forward GEMM's launch
    # also writes Z = X H (bf16) from its extra warps
    addend = (4.0 * T * do if stage == "gemm_fwd" else 4.0 * T * di) if algo == "sparse" else 0.0
    if algo == "dense" and stage == "gemm_fwd":
        addend = 2.0 * T * di
    qbytes = do * di * bits / 8 + (do * di / spec.group) * 5
    w = {
        # forward transform: read X, write Z (bf16)
        "fwht_fwd": ("hbm", 4.0 * T * di, 4.0 * T * di),
        # backward transform: read dZ (fp32), write dX_adapter (fp32)
        "fwht_bwd": ("hbm", 8.0 * T * di, 8.0 * T * di),
        "dequant": ("hbm", qbytes + 2.0 * do * di, qbytes + 2.0 * do * di),
        # sparse products: 2 p T FLOP; bytes = activations in and out + the index arrays
        "spmm_fwd": ("alu", 2.0 * p * T, 2.0 * T * di + 4.0 * T * do + 8.0 * p),
        "gather_bwd": ("alu", 2.0 * p * T, 2.0 * T * do + 4.0 * T * di + 12.0 * p),
        "sddmm_dc": ("alu", 2.0 * p * T, 2.0 * T * (di + do) + 8.0 * p),
        "gemm_fwd": ("tensor", 2.0 * T * di * do, 2.0 * T * di + 2.0 * do * di + 2.0 * T * do + addend),
        "gemm_bwd": ("tensor", 2.0 * T * di * do, 2.0 * T * do + 2.0 * do * di + 2.0 * T * di + addend),
        "gemm_dc": ("tensor", 2.0 * T * di * do, 2.0 * T * (di + do) + 12.0 * p),
        # W_eff = W_Q + alpha F H: codes + CSR in, bf16 out
        "weff": ("hbm", qbytes + 8.0 * p + 2.0 * do * di, qbytes + 8.0 * p + 2.0 * do * di),
    }
    return w.get(stage)


SUSTAINED_AFTER_S = 1.0  # timed regions at least this long are compared with the sustained (power-capped) GEMM peak


def fp32_fma_tflops(peaks):
    mhz = peaks.get("sm_max_mhz", 1965.0)
    return 148 * ALU_LANES_PER_SM * 2 * mhz * 1e6 / 1e12


def peak_for(kind, peaks, region_s=0.0):
    """(peak, unit, note) for a kernel whose timed region lasted region_s seconds: the burst cuBLAS bf16 figure for
    regions shorter than SUSTAINED_AFTER_S, the sustained one (a seconds-long loop under the power cap) otherwise."""
    if kind == "hbm":
        return peaks["hbm_gbs"], "GB/s", "HBM copy bandwidth, " + peaks["_source"]
    if kind == "tensor":
        if region_s >= SUSTAINED_AFTER_S:
            return (peaks["bf16_tflops_sustained"], "TFLOP/s",
                    f"cuBLAS bf16 sustained ({region_s:.2f} s timed region), " + peaks["_source"])
        return (peaks["bf16_tflops"], "TFLOP/s",
                f"cuBLAS bf16 burst ({region_s:.3f} s timed region), " + peaks["_source"])
    return fp32_fma_tflops(peaks), "TFLOP/s", "fp32 FMA: 148 SMs x 128 lanes x 2 x max SM clock (derived)"


# the method's own work of a stage that the tensor cores do as a larger dense product: the dense dc GEMM computes
# all d_out x d_in entries of dY^T Z and keeps the p at E, whose sums (2 p T FLOP) are the SDDMM's work
METHOD_WORK = {"gemm_dc": lambda spec, T: ("alu", 2.0 * spec.p * T)}


# --------------------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi samples during the timed region (read-only queries)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self):
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"qwha_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            v = [x.strip() for x in line.split(",")]
            if len(v) < 10:
                continue
            try:
                rows.append(dict(sm=float(v[1]), mx=float(v[2]), util=float(v[4]), hw=v[6], hwt=v[7], swt=v[8],
                                 pcap=v[9]))
            except ValueError:
                continue
        load = [r for r in rows if r["util"] >= 50] or rows
        if not load:
            return None
        reasons = set()
        for r in load:
            for k, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                            ("pcap", "sw_power_cap")):
                if r[k].lower() in ("active", "1", "yes"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load), "sm_max_mhz": max(r["mx"] for r in load),
                "reasons": sorted(reasons), "samples": len(load)}


# --------------------------------------------------------------------------- CPU oracle


_ORACLE_INIT = {}


def oracle_tokens_per_s(spec, d, X, dY, tokens, threads=0):
    """The oracle's forward + backward over `tokens` token rows (dc over all p entries); returns (tokens/s, s, cores).
    E and c come from the oracle's own AdaAlloc on the same dW_Q (computed once, untimed)."""
    import oracle

    cores = oracle.set_threads(threads)
    if spec.name not in _ORACLE_INIT:
        _ORACLE_INIT[spec.name] = oracle.init_alloc(d["dWq"], spec.p, spec.had_block, spec.min_per_row, spec.remainder)
    init = _ORACLE_INIT[spec.name]
    rp, ci, cf = init["row_ptr"], init["col_idx"], init["coef"]
    rows = oracle.csr_rows(rp)
    t0 = time.perf_counter()
    Wq = oracle.dequant(d["qweight"], d["scales"], d["zeros"], spec.bits, spec.group, spec.d_out, spec.d_in)
    oracle.adapter_fwd(rp, ci, cf, X[:tokens], spec.d_out, spec.had_block, 1.0, Wq)
    oracle.adapter_bwd_dx(rp, ci, cf, dY[:tokens], spec.d_in, spec.had_block, 1.0, Wq)
    oracle.adapter_bwd_dc(X[:tokens], dY[:tokens], rows, ci, spec.had_block, 1.0)
    dt = time.perf_counter() - t0
    return tokens / dt, dt, cores


def run_reference(args, spec):
    """The oracle as the reference arm: every step is one sampled token's full fwd+bwd."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    d = layer_inputs(spec, args.seed, WORKLOAD, parts=("W", "X", "dY"), rows=np.arange(64))
    probe, t_probe, cores = oracle_tokens_per_s(spec, d, d["X"], d["dY"], 1)
    budget_s = 150.0
    steps = int(max(1, min(args.steps, budget_s // max(t_probe, 1e-3) - min(args.warmup, 1))))
    for w in range(min(args.warmup, 1)):
        oracle_tokens_per_s(spec, d, d["X"][w + 1 :], d["dY"][w + 1 :], 1)
    total = 0.0
    for i in range(steps):
        r = (i + 2) % 64
        _, dt, _ = oracle_tokens_per_s(spec, d, d["X"][r:], d["dY"][r:], 1)
        total += dt
    value = steps / total
    sample = (f"1 token per step (Y and dX for that token, dc over all {spec.p} coefficients); {steps} of "
              f"{args.steps} requested steps timed, bounded to ~{int(budget_s)} s of host time")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": steps,
        "warmup": min(args.warmup, 1), "ms_per_step": 1e3 * total / steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(spec, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_block(spec, n):
    return {
        "workload": (f"{WORKLOAD}: d_in={spec.d_in} d_out={spec.d_out} T={spec.T} tokens per GPU (16 x 512), "
                     f"{spec.bits}-bit g{spec.group} RTN base weight, p={spec.p} (LoRA r=64 count), AdaAlloc E"),
        "global_batch": spec.T * n, "seq_len": 512, "parallelism": f"dp{n}",
        "l2": f"flushed before every timed step ({FLUSH_BYTES >> 20} MiB write)",
    }


# --------------------------------------------------------------------------- main


# --------------------------------------------------------------------------- the other workloads

# what the GPU needs of a layer's host-generated weights
W_KEYS = ("qweight", "scales", "zeros", "dWq")


def host_weights(spec, seed, workload, keys=W_KEYS):
    """The seeded weights of one layer (runs in a worker process): only the arrays the GPU needs."""
    d = layer_inputs(spec, seed, workload, parts=("W",))
    return {k: d[k] for k in keys}


class WeightPool:
    """Host generation of the other workloads' weights in spawned worker processes (started before the first GPU
    call), so that it overlaps the headline measurement instead of adding to the run."""

    def __init__(self, seed, workers):
        import concurrent.futures
        import multiprocessing

        self.ex = concurrent.futures.ProcessPoolExecutor(max_workers=workers,
                                                         mp_context=multiprocessing.get_context("spawn"))
        self.fut = {}
        for wl in ("mlp", "block"):
            for spec in CONFIGS[wl]:
                self.fut[(wl, spec.name)] = self.ex.submit(host_weights, spec, seed, wl)
        for spec in CONFIGS["init_sweep"]:
            key = ("init_sweep", spec.w_stream)
            if key not in self.fut:
                self.fut[key] = self.ex.submit(host_weights, spec, seed, "init_sweep", ("dWq",))

    def get(self, wl, name):
        return self.fut[(wl, name)].result()

    def close(self):
        self.ex.shutdown(wait=True, cancel_futures=True)


def run_stack(W, torch, dev, wl, weights, seed, K, warmup, peaks, compare_unshared=False):
    """Forward of every layer of workload `wl` in order, then the backward in reverse order (dense algorithm), as one
    step; the transform Z = X H is shared by the layers that read the same input (z_given). AdaAlloc on the GPU from
    the host-generated dW_Q; activations drawn on the GPU from a seeded generator with the workload's distribution
    (N(0, 1), 1% of input channels x20). Returns the timing record (and, with compare_unshared, the same step with
    every layer computing its own transform)."""
    from workloads.synth import _x_channels

    specs = CONFIGS[wl]
    T = specs[0].T
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    layers, X, Zb, dY, Y, dX, dc = [], {}, {}, {}, {}, {}, {}
    for spec in specs:
        d = weights(wl, spec.name)
        dWq = torch.from_numpy(d["dWq"]).to(dev)
        e = W.init_alloc(dWq, spec.p, spec.had_block, spec.min_per_row, spec.remainder)
        del dWq
        wq = W.QWeight(spec.bits, spec.group, torch.from_numpy(d["qweight"]).to(dev),
                       torch.from_numpy(d["scales"]).to(dev), torch.from_numpy(d["zeros"]).to(dev))
        a = W.Adapter(spec.d_in, spec.d_out, spec.had_block, spec.p, e["row_ptr"], e["col_idx"], e["coef"],
                      algo="dense")
        a.weff = torch.empty((spec.d_out, spec.d_in), dtype=torch.bfloat16, device=dev)
        layers.append((spec, a, wq))
        if spec.x_stream not in X:
            x = torch.randn((T, spec.d_in), generator=gen, device=dev)
            ch = torch.from_numpy(_x_channels(spec, seed, wl)).to(dev)
            x[:, ch] *= spec.x_outlier_scale
            X[spec.x_stream] = x.to(torch.bfloat16)
            Zb[spec.x_stream] = torch.empty_like(X[spec.x_stream])
            del x
        dY[spec.name] = torch.randn((T, spec.d_out), generator=gen, device=dev).to(torch.bfloat16)
        Y[spec.name] = torch.empty((T, spec.d_out), dtype=torch.bfloat16, device=dev)
        dX[spec.name] = torch.empty((T, spec.d_in), dtype=torch.bfloat16, device=dev)
        dc[spec.name] = torch.empty(spec.p, dtype=torch.float32, device=dev)
    ws = {}
    for spec, _, _ in layers:
        for op in (4, 5):
            n = W.workspace_size(op, spec.d_out, spec.d_in, spec.p, T, True)
            if n > ws.get(op, torch.empty(0)).numel():
                ws[op] = torch.empty(n, dtype=torch.uint8, device=dev)

    def step(shared):
        seen = set()
        for spec, a, wq in layers:
            given = shared and spec.x_stream in seen
            W.adapter_fwd(a, X[spec.x_stream], 1.0, wq, Z_out=Zb[spec.x_stream], Y=Y[spec.name], z_given=given,
                          ws=ws.get(4))
            seen.add(spec.x_stream)
        for spec, a, wq in reversed(layers):
            W.adapter_bwd(a, dY[spec.name], Zb[spec.x_stream], 1.0, wq, dc=dc[spec.name], dX=dX[spec.name],
                          ws=ws.get(5))

    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    res = {}
    for shared in ((True, False) if compare_unshared else (True,)):
        for _ in range(warmup):
            step(shared)
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        W.stage_report()
        W.stage_timing(shared)
        for i in range(K):
            flush.fill_(i & 0xFF)
            ev[i][0].record()
            step(shared)
            ev[i][1].record()
        torch.cuda.synchronize()
        W.stage_timing(False)
        rep = W.stage_report()
        ms = sum(s_.elapsed_time(e_) for s_, e_ in ev) / K
        res[shared] = (ms, rep, ev[0][0].elapsed_time(ev[-1][1]) / 1e3)
    ms, rep, region_s = res[True]
    # per-stage work of one step: every layer runs every stage once
    stages = {}
    for name, (calls, launches, tot_ms) in rep.items():
        if not calls:
            continue
        kinds = [stage_work(name, spec, T, spec.bits, "dense") for spec in specs]
        if any(k is None for k in kinds):
            stages[name] = {"ms_per_step": tot_ms / K}
            continue
        kind = kinds[0][0]
        work = sum(k[1] for k in kinds)
        peak, unit, note = peak_for(kind, peaks, region_s)
        ach = work / (tot_ms / K / 1e3) / (1e9 if unit == "GB/s" else 1e12)
        stages[name] = {"ms_per_step": tot_ms / K, "calls_per_step": calls / K, "bound": kind, "achieved": ach,
                        "unit": unit, "peak": peak, "frac": ach / peak, "peak_source": note}
    dom = max((n for n in stages if "frac" in stages[n]), key=lambda n: stages[n]["ms_per_step"])
    flops = sum(3 * 2.0 * T * sp.d_in * sp.d_out for sp in specs)
    out = {"ms_per_step": ms, "value": T / (ms / 1e3), "unit": UNIT, "steps": K, "tokens": T,
           "gemm_tflops": flops / (ms / 1e3) / 1e12, "stages": stages,
           "roofline": dict(kernel=dom, **{k: stages[dom][k] for k in ("bound", "achieved", "peak", "unit", "frac",
                                                                      "peak_source")})}
    if compare_unshared:
        out["without_sharing"] = {"ms_per_step": res[False][0], "value": T / (res[False][0] / 1e3)}
    del layers, X, Zb, dY, Y, dX, dc, ws, flush
    torch.cuda.empty_cache()
    return out


def run_init_sweep(W, torch, dev, weights, peaks):
    """AdaAlloc on the seven LLaMA-3-8B shapes at r = 16, 64, 128 (2-bit g64 error): the median of 3 timed calls
    per shape, each after a warm call; plus the Hill exponent and cumulative energy of |dW_Q H| at k = p (the
    selection diagnostics) for every shape and r."""
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    shapes, tot_ms, tot_bytes, cur = {}, 0.0, 0.0, {}
    for spec in CONFIGS["init_sweep"]:
        if spec.w_stream not in cur:
            cur.clear()
            cur[spec.w_stream] = torch.from_numpy(weights("init_sweep", spec.w_stream)["dWq"]).to(dev)
        dWq = cur[spec.w_stream]
        ws = torch.empty(W.workspace_size(2, spec.d_out, spec.d_in, spec.p, 0, False), dtype=torch.uint8, device=dev)
        W.init_alloc(dWq, spec.p, spec.had_block, spec.min_per_row, spec.remainder, ws=ws)
        ts = []
        for _ in range(3):
            ev[0].record()
            W.init_alloc(dWq, spec.p, spec.had_block, spec.min_per_row, spec.remainder, ws=ws)
            ev[1].record()
            torch.cuda.synchronize()
            ts.append(ev[0].elapsed_time(ev[1]))
        ms = statistics.median(ts)
        nbytes = 2 * 4.0 * spec.d_out * spec.d_in + 8.0 * spec.p
        es = W.energy_stats(dWq, spec.p, spec.had_block).cpu().numpy()
        shapes[spec.name] = {"ms": ms, "alg_GBps": nbytes / (ms / 1e3) / 1e9, "eta": float(es[0]),
                             "energy_top_p": float(es[1])}
        tot_ms += ms
        tot_bytes += nbytes
    return {"ms_total": tot_ms, "shapes": shapes, "alg_GBps": tot_bytes / (tot_ms / 1e3) / 1e9,
            "frac_hbm": tot_bytes / (tot_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
            "what": ("AdaAlloc (norms, budgets, fp64 transform, per-row top-k) on the 21 init-sweep shapes, 2-bit g64 "
                     "RTN error; eta / energy_top_p: Hill exponent and energy share of the p largest |dW_Q H|")}


def run_diagnostics(W, torch, spec, dWq, e, sel_e):
    """The selection diagnostics of the q_proj layer: Hill exponent and cumulative energy of |dW_Q H| at k = p, and
    the row/column counts (rank bound) of E under AdaAlloc, whole-matrix magnitude and random selection."""
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ws = torch.empty(W.workspace_size(8, spec.d_out, spec.d_in, 0, 0, False), dtype=torch.uint8, device=dWq.device)
    W.energy_stats(dWq, spec.p, spec.had_block, ws=ws)
    ts = []
    for _ in range(3):
        ev[0].record()
        es = W.energy_stats(dWq, spec.p, spec.had_block, ws=ws)
        ev[1].record()
        torch.cuda.synchronize()
        ts.append(ev[0].elapsed_time(ev[1]))
    es = es.cpu().numpy()
    names = W.api.PATTERN_STATS
    pats = {}
    for rule, ee in [("adaalloc", e)] + list(sel_e.items()):
        st, _ = W.pattern_stats(ee["row_ptr"], ee["col_idx"], spec.d_in)
        pats[rule] = dict(zip(names, st.cpu().numpy().tolist()))
    return {"eta": float(es[0]), "energy_top_p": float(es[1]), "energy_ms": statistics.median(ts),
            "pattern": pats,
            "what": ("eta: Hill exponent of the p largest |dW_Q H| (smaller = error energy more concentrated); "
                     "pattern: counts of E per rule, rank_bound = min(non-empty rows, non-empty columns) >= rank(F), "
                     "half_rows = fewest rows holding half of E")}


def run_block(args):
    """`--workload block`: the decoder-block workload alone (seven LLaMA-3-8B-shaped linears, 32768 tokens, 4-bit
    g128, r = 64), with and without the shared transform, printed as its own JSON line."""
    import torch

    import walsh_hadamard_sparse_b200 as W

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    r = run_stack(W, torch, dev, "block", lambda wl, name: host_weights(next(s for s in CONFIGS[wl] if s.name == name),
                                                                        args.seed, wl),
                  args.seed, max(3, min(args.steps, 10)), max(args.warmup, 3), load_peaks(), compare_unshared=True)
    line = {
        "metric": "decoder block (7 adapted linears) fwd+bwd tokens/s", "value": r["value"], "unit": "tokens/s",
        "n_gpus": 1, "steps": r["steps"], "ms_per_step": r["ms_per_step"], "higher_is_better": True, "dtype": "bf16",
        "data": "synthetic (seeded; weights host-generated, activations drawn on the GPU)",
        "config": {"workload": "block: LLaMA-3-8B q/k/v/o/gate/up/down, T=32768 (8 x 4096), 4-bit g128, r=64",
                   "l2": f"flushed before every timed step ({FLUSH_BYTES >> 20} MiB write)"},
        "algorithm": "dense; Z = X H shared by q/k/v and by gate/up (z_given)",
        "gemm_tflops": r["gemm_tflops"], "without_sharing": r["without_sharing"], "roofline": r["roofline"],
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--sparse-steps", type=int, default=40)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=["q_proj", "block"], default="q_proj",
                    help="block: time the decoder-block workload (seven linears) instead of the q_proj step")
    ap.add_argument("--no-init-extras", action="store_true",
                    help="skip timing the selection variants and Value Refinement (one-off setup, not the step)")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other workloads (MLP pair, decoder block, init sweep) and the diagnostics")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    spec = CONFIGS[WORKLOAD][0]
    if args.workload == "block" and args.impl == "ours":
        return run_block(args)
    if args.impl == "reference":
        return run_reference(args, spec)
    # the other workloads' weights are generated on the host while the GPU measures the headline (one GPU only;
    # the worker processes are spawned before the first CUDA call)
    pool = None
    if not args.no_workloads and int(os.environ.get("WORLD_SIZE", "1")) == 1:
        pool = WeightPool(args.seed, max(1, min(8, (os.cpu_count() or 2) - 1)))

    import torch
    import torch.distributed as dist

    import walsh_hadamard_sparse_b200 as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    T = spec.T
    d = layer_inputs(spec, args.seed, WORKLOAD, parts=("W",))
    act = layer_inputs(spec, args.seed, WORKLOAD, parts=("X", "dY"), rows=rank_rows(rank, T))

    def bf16(bits):
        return torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)

    X, dY = bf16(act["X_bits"]), bf16(act["dY_bits"])
    dWq = torch.from_numpy(d["dWq"]).to(dev)
    wq = W.QWeight(spec.bits, spec.group, torch.from_numpy(d["qweight"]).to(dev),
                   torch.from_numpy(d["scales"]).to(dev), torch.from_numpy(d["zeros"]).to(dev))
    peaks = load_peaks()

    # ---- AdaAlloc (one-off per layer), timed on its own
    for _ in range(2):
        e = W.init_alloc(dWq, spec.p, spec.had_block, spec.min_per_row, spec.remainder)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    init_ms = []
    for _ in range(5):
        ev[0].record()
        e = W.init_alloc(dWq, spec.p, spec.had_block, spec.min_per_row, spec.remainder)
        ev[1].record()
        torch.cuda.synchronize()
        init_ms.append(ev[0].elapsed_time(ev[1]))
    # the pages' alternatives to AdaAlloc (whole-matrix magnitude top-p, seeded random E), timed the same way
    sel_ms, sel_e = {}, {}
    for sel in (() if args.no_init_extras else ("magnitude", "random")):
        sws = torch.empty(W.workspace_size(6, spec.d_out, spec.d_in, spec.p, 0, False), dtype=torch.uint8, device=dev)
        sel_e[sel] = W.init_select_global(dWq, spec.p, spec.had_block, sel, 1, ws=sws)
        torch.cuda.synchronize()
        ts = []
        for _ in range(3):
            ev[0].record()
            W.init_select_global(dWq, spec.p, spec.had_block, sel, 1, ws=sws)
            ev[1].record()
            torch.cuda.synchronize()
            ts.append(ev[0].elapsed_time(ev[1]))
        sel_ms[sel] = statistics.median(ts)
        del sws
    # Value Refinement of the AdaAlloc values with this GPU's tokens as calibration rows
    rws = torch.empty(W.workspace_size(7, spec.d_out, spec.d_in, spec.p, 0, False), dtype=torch.uint8, device=dev)
    S_cal = torch.empty((spec.d_in, spec.d_in), dtype=torch.float32, device=dev)
    c_ref = torch.empty(spec.p, dtype=torch.float32, device=dev)
    refine_ms = []
    for it in range(0 if args.no_init_extras else 4):
        ev[0].record()
        W.calib_hessian(X, S_cal)
        W.refine_values(dWq, S_cal, e["row_ptr"], e["col_idx"], spec.had_block, 0.01, coef=c_ref, ws=rws)
        ev[1].record()
        torch.cuda.synchronize()
        if it:
            refine_ms.append(ev[0].elapsed_time(ev[1]))
    del rws, S_cal, c_ref
    a = W.Adapter(spec.d_in, spec.d_out, spec.had_block, spec.p, e["row_ptr"], e["col_idx"], e["coef"])
    W.plan_build(a)  # the views the sparse backward needs

    alpha = 1.0
    Z = torch.empty_like(X)
    Y = torch.empty((T, spec.d_out), dtype=torch.bfloat16, device=dev)
    dX = torch.empty_like(X)
    dc = torch.empty(spec.p, dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    adapters = {
        algo: W.Adapter(spec.d_in, spec.d_out, spec.had_block, spec.p, a.row_ptr, a.col_idx, a.coef, a.col_ptr,
                        a.row_idx, a.perm, a.tile_ptr, a.tile_pos, a.tile_rk, algo=algo)
        for algo in ("dense", "sparse")
    }
    # the dense forward keeps W_eff = W_Q + alpha F H for its backward (like Z)
    adapters["dense"].weff = torch.empty((spec.d_out, spec.d_in), dtype=torch.bfloat16, device=dev)
    ws = {}
    for algo, ops in (("dense", (4, 5)), ("sparse", (0, 1))):
        ws[algo] = [torch.empty(max(1, W.workspace_size(op, spec.d_out, spec.d_in, spec.p, T, True)),
                                dtype=torch.uint8, device=dev) for op in ops]

    def make_step(algo):
        ad, (wf, wb) = adapters[algo], ws[algo]

        def step():
            if world > 1:
                # dc first; its all-reduce (the path's one exchange) overlaps the dX computation
                W.dp_step(ad, X, dY, alpha, wq, Z=Z, Y=Y, dc=dc, dX=dX, ws_fwd=wf, ws_bwd=wb)
            else:
                W.adapter_fwd(ad, X, alpha, wq, Z_out=Z, Y=Y, ws=wf)
                W.adapter_bwd(ad, dY, Z, alpha, wq, dc=dc, dX=dX, ws=wb)

        return step

    def timed(step, K, sample_clocks):
        """K steps, each bracketed by events on the current stream after an L2 flush; (ms, stage report, clocks)."""
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        W.stage_report()
        W.stage_timing(True)
        clocks = ClockSampler() if (rank == 0 and sample_clocks) else None
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        if clocks:
            clocks.start()
            time.sleep(0.3)
        for i in range(K):
            flush.fill_(i & 0xFF)
            starts[i].record()
            step()
            ends[i].record()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        clk = clocks.stop() if clocks else None
        W.stage_timing(False)
        rep = W.stage_report()
        t_ms = sum(s_.elapsed_time(e_) for s_, e_ in zip(starts, ends))
        span_ms = starts[0].elapsed_time(ends[-1])  # the whole timed region, L2 flushes included
        if world > 1:
            tt = torch.tensor([t_ms, span_ms], device=dev)
            dist.all_reduce(tt, op=dist.ReduceOp.MAX)
            t_ms, span_ms = float(tt[0].item()), float(tt[1].item())
        return t_ms, rep, clk, span_ms

    def kernel_table(rep, K, algo, region_s):
        kernels = {}
        for name, (calls, launches, ms) in rep.items():
            if calls == 0:
                continue
            per = ms / calls
            k = {"calls": calls, "launches": launches, "ms_per_call": per}
            wk = stage_work(name, spec, T, spec.bits, algo)
            if wk:
                kind, amount, nbytes = wk
                peak, unit, note = peak_for(kind, peaks, region_s)
                ach = amount / (per / 1e3) / (1e9 if unit == "GB/s" else 1e12)
                k.update(bound=kind, work=amount, achieved=ach, peak=peak, unit=unit, frac=ach / peak,
                         peak_source=note, alg_GBps=nbytes / (per / 1e3) / 1e9, alg_bytes=nbytes,
                         traffic=ncu_traffic(algo, name))
                if name in METHOD_WORK:
                    mkind, mwork = METHOD_WORK[name](spec, T)
                    mpeak, munit, mnote = peak_for(mkind, peaks, region_s)
                    mach = mwork / (per / 1e3) / 1e12
                    k["method"] = {"bound": mkind, "work": mwork, "achieved": mach, "peak": mpeak, "unit": munit,
                                   "frac": mach / mpeak, "peak_source": mnote,
                                   "what": "2 p T FLOP of the coefficient gradient, against the FP32 FMA roofline"}
            kernels[name] = k
        tot = sum(v["ms_per_call"] * v["calls"] for v in kernels.values())
        for v in kernels.values():
            v["share"] = v["ms_per_call"] * v["calls"] / tot
        return kernels

    def roofline_of(kernels, algo):
        dom = max((n for n in kernels if "bound" in kernels[n]), key=lambda n: kernels[n]["share"])
        kd = kernels[dom]
        r = {"kernel": dom, "bound": kd["bound"], "achieved": kd["achieved"], "peak": kd["peak"],
             "unit": kd["unit"], "frac": kd["frac"], "traffic": ncu_traffic(algo, dom), "peak_source": kd["peak_source"],
             "work_per_launch": kd["work"], "ms_per_call": kd["ms_per_call"]}
        if "method" in kd:
            r["method"] = kd["method"]
        return r

    results = {}
    for algo in ("dense", "sparse"):
        step = make_step(algo)
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        if not (torch.isfinite(Y.float()).all() and torch.isfinite(dc).all() and torch.isfinite(dX.float()).all()):
            raise RuntimeError(f"non-finite output ({algo})")
        K = args.steps if algo == "dense" else max(3, min(args.steps, args.sparse_steps))
        t_ms, rep, clk, span_ms = timed(step, K, algo == "dense")
        kernels = kernel_table(rep, K, algo, span_ms / 1e3)
        results[algo] = dict(K=K, t_ms=t_ms, value=world * T * K / (t_ms / 1e3), kernels=kernels,
                             roofline=roofline_of(kernels, algo), launches=sum(v[1] for v in rep.values()), clocks=clk)
    head = results["dense"]
    K, t_ms, value, kernels, clk = head["K"], head["t_ms"], head["value"], head["kernels"], head["clocks"]
    roofline, launches = head["roofline"], head["launches"]
    step = make_step("dense")

    # the host generation of the other workloads' weights is over before the host-link and host-core legs
    weights = {}
    if pool is not None:
        for key, f in pool.fut.items():
            weights[key] = f.result()
        pool.close()

    # ---- end to end through host buffers: every step copies its X and dY in from pinned host memory and reads
    # its dc back; the copy of step i+1's inputs (on a copy stream, into the other of two device buffers) runs
    # while step i computes, as an input pipeline would.
    e2e = None
    if args.e2e_steps > 0:
        Xh = torch.empty_like(X, device="cpu").pin_memory()
        dYh = torch.empty_like(dY, device="cpu").pin_memory()
        Xh.copy_(X)
        dYh.copy_(dY)
        dch = torch.empty_like(dc, device="cpu").pin_memory()
        bufs = [(X, dY), (torch.empty_like(X), torch.empty_like(dY))]
        ad, (wf, wb) = adapters["dense"], ws["dense"]
        comp, cs = torch.cuda.current_stream(), torch.cuda.Stream()
        ready = [torch.cuda.Event() for _ in bufs]
        free = [torch.cuda.Event() for _ in bufs]

        def e2e_steps(n, start_ev=None):
            if start_ev is not None:
                cs.wait_event(start_ev)
            for i in range(n):
                b = i % 2
                Xb, dYb = bufs[b]
                with torch.cuda.stream(cs):
                    if i >= 2:
                        cs.wait_event(free[b])  # step i-2 has finished reading this buffer
                    Xb.copy_(Xh, non_blocking=True)
                    dYb.copy_(dYh, non_blocking=True)
                    ready[b].record(cs)
                comp.wait_event(ready[b])
                if world > 1:
                    W.dp_step(ad, Xb, dYb, alpha, wq, Z=Z, Y=Y, dc=dc, dX=dX, ws_fwd=wf, ws_bwd=wb)
                else:
                    W.adapter_fwd(ad, Xb, alpha, wq, Z_out=Z, Y=Y, ws=wf)
                    W.adapter_bwd(ad, dYb, Z, alpha, wq, dc=dc, dX=dX, ws=wb)
                free[b].record(comp)
                dch.copy_(dc, non_blocking=True)

        Ke = args.e2e_steps
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2e_steps(3)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        s0.record(comp)
        e2e_steps(Ke, s0)
        s1.record(comp)
        torch.cuda.synchronize()
        te = s0.elapsed_time(s1)
        if world > 1:
            tt = torch.tensor([te], device=dev)
            dist.all_reduce(tt, op=dist.ReduceOp.MAX)
            te = float(tt.item())
        e2e = {"value": world * T * Ke / (te / 1e3), "unit": UNIT, "steps": Ke,
               "h2d_bytes_per_step": X.numel() * 2 + dY.numel() * 2, "d2h_bytes_per_step": dc.numel() * 4,
               "note": ("pinned host X and dY copied in and dc read back every step (the next step's inputs are "
                        "copied on a second stream while the current step computes); Y, Z and dX stay on the GPU")}

    # ---- CPU oracle baseline (rank 0, one GPU only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        host_act = {"X": act["X"][:512].astype(np.float64), "dY": act["dY"][:512].astype(np.float64)}
        # size the sample for ~15 s of host work: a call costs a fixed part (dequantizing W_Q) plus a part per token
        _, t1, cores = oracle_tokens_per_s(spec, d, host_act["X"], host_act["dY"], 1)
        _, t4, cores = oracle_tokens_per_s(spec, d, host_act["X"], host_act["dY"], 4)
        per_tok = max((t4 - t1) / 3.0, 1e-3)
        toks = int(max(1, min(512, (15.0 - max(t1 - per_tok, 0.0)) / per_tok)))
        rate, dt, cores = oracle_tokens_per_s(spec, d, host_act["X"], host_act["dY"], toks)
        cpu = {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{toks} tokens of the same layer (Y, dX for them; dc over all {spec.p} coefficients), "
                         f"{dt:.1f} s of host time"}

    # ---- the other workloads (one GPU): the LLaMA-3-8B MLP pair, the decoder block, the init sweep; and the
    # selection diagnostics of the q_proj layer
    extra = {}
    if weights:
        del Z, Y, dX, ws, adapters, flush
        torch.cuda.empty_cache()
        get = lambda wl, name: weights[(wl, name)]  # noqa: E731
        extra["mlp"] = run_stack(W, torch, dev, "mlp", get, args.seed, 10, 3, peaks)
        extra["mlp"]["what"] = ("LLaMA-3-8B MLP: gate and up 4096 -> 14336 (one shared Z), down 14336 -> 4096 "
                                "(seven 2048-point blocks), 16384 tokens, 3-bit g128, r = 64, dense, fwd + bwd")
        extra["block"] = run_stack(W, torch, dev, "block", get, args.seed, 5, 3, peaks, compare_unshared=True)
        extra["block"]["what"] = ("LLaMA-3-8B decoder block, 7 adapted linears (q, k, v share Z; gate, up share Z), "
                                  "32768 tokens, 4-bit g128, r = 64, dense, fwd + bwd")
        extra["init_sweep"] = run_init_sweep(W, torch, dev, get, peaks)
        diagnostics = run_diagnostics(W, torch, spec, dWq, e, sel_e) if sel_e else None
    else:
        diagnostics = None

    init_bytes = 2 * 4.0 * spec.d_in * spec.d_out + 8.0 * spec.p
    init_med = statistics.median(init_ms)
    sp = results["sparse"]

    def adapter_only(res, algo):
        """The adapter's share of a step (tokens/s over its stages alone): the sparse path's transforms, SpMM, SDDMM
        and gather; the dense path's W_eff and coefficient-gradient GEMM (its forward and dX ride in the GEMMs the
        frozen layer runs anyway; the transform inside the forward GEMM's launch is counted there, not here)."""
        names = ADAPTER_STAGES[algo]
        ms = sum(res["kernels"][n]["ms_per_call"] * res["kernels"][n]["calls"] for n in names if n in res["kernels"])
        ms /= res["K"]
        return {"ms_per_step": ms, "value": world * T / (ms / 1e3), "unit": UNIT, "stages": names}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": t_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; stands in for LLaMA-7B q_proj weights and activations)",
        "config": config_block(spec, world),
        "algorithm": ("dense: adapter folded into the tcgen05 GEMMs (W_eff = W_Q + alpha F H, kept from the forward "
                      "for the backward); dc from dY^T Z sampled at E in the GEMM epilogue"),
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clk,
        "kernels": kernels,
        "adapter_only": adapter_only(head, "dense"),
        "paths": {
            "sparse": {"value": sp["value"], "unit": UNIT, "steps": sp["K"], "ms_per_step": sp["t_ms"] / sp["K"],
                       "adapter_only": adapter_only(sp, "sparse"),
                       "roofline": sp["roofline"], "gpu_launches": sp["launches"], "kernels": sp["kernels"],
                       "what": "segment SpMM over CSR, tiled SDDMM, CSC gather on the FMA units; base GEMMs on tcgen05"},
        },
        "workloads": extra or None,
        "diagnostics": diagnostics,
        "init": {"ms": init_med, "alg_GBps": init_bytes / (init_med / 1e3) / 1e9,
                 "frac_hbm": init_bytes / (init_med / 1e3) / 1e9 / peaks["hbm_gbs"],
                 "what": "AdaAlloc on dW_Q (4096 x 4096 fp32): norms, budgets, fp64 transform, top-k; one-off per layer",
                 "select_global_ms": sel_ms,
                 "refine_ms": statistics.median(refine_ms) if refine_ms else None,
                 "refine_what": ("Value Refinement at E: calibration Hessian X^T X over the 8192 tokens, G = H S H, "
                                 "dW_Q S H, per-channel fp64 Cholesky solves"),
                 "select_global_what": ("whole-matrix selection (magnitude top-p; seeded random E): fp64 transform of "
                                        "all rows kept in HBM, 8-bit radix passes over the 16.8 M keys until the "
                                        "candidates fit a 64 K list, one CTA finishes on the list, per-row "
                                        "compaction")},
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
