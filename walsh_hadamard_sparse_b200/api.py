"""torch-facing wrappers of the C ABI (argument marshalling only).

Tensors must be CUDA tensors, contiguous, of the documented dtypes; work is
enqueued on torch's current stream. Scratch space comes from torch's
allocator and is passed to the library as the `ws` argument.
"""

from __future__ import annotations

import ctypes
from dataclasses import dataclass, fields

import torch

from ._lib import QwhaAdapter, QwhaQweight, check, lib

F32, BF16 = 0, 1
OP_FWD, OP_BWD, OP_INIT, OP_PLAN, OP_FWD_DENSE, OP_BWD_DENSE, OP_SELECT_GLOBAL, OP_REFINE = 0, 1, 2, 3, 4, 5, 6, 7
OP_ENERGY, OP_PATTERN = 8, 9
PATTERN_STATS = ("empty_rows", "empty_cols", "min_row", "max_row", "min_col", "max_col", "rank_bound", "half_rows")
SELECTION = {"magnitude": 0, "random": 1}
ALGO = {"sparse": 0, "dense": 1}
REMAINDER = {"fewest": 0, "largest": 1}


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t) -> ctypes.c_void_p | None:
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("expected a contiguous CUDA tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ws(nbytes: int, device) -> torch.Tensor | None:
    if nbytes == 0:
        return None
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


@dataclass
class Adapter:
    """F = Scatter(c, E) on the device: CSR arrays plus the views from plan_build."""

    d_in: int
    d_out: int
    had_block: int
    p: int
    row_ptr: torch.Tensor
    col_idx: torch.Tensor
    coef: torch.Tensor
    col_ptr: torch.Tensor | None = None
    row_idx: torch.Tensor | None = None
    perm: torch.Tensor | None = None
    tile_ptr: torch.Tensor | None = None
    tile_pos: torch.Tensor | None = None
    tile_rk: torch.Tensor | None = None
    algo: str = "sparse"
    weff: torch.Tensor | None = None  # dense: W_eff kept from the forward for the backward

    def c_struct(self) -> QwhaAdapter:
        s = QwhaAdapter()
        s.d_in, s.d_out, s.had_block, s.p = self.d_in, self.d_out, self.had_block, self.p
        s.algo = ALGO[self.algo]
        for f in fields(self):
            if f.name in ("d_in", "d_out", "had_block", "p", "algo"):
                continue
            v = getattr(self, f.name)
            setattr(s, f.name, None if v is None else v.data_ptr())
        return s


@dataclass
class QWeight:
    """Packed b-bit codes [d_out, d_in*bits/8] u8, scales f32 and zeros u8 [d_out, d_in/group]."""

    bits: int
    group: int
    qweight: torch.Tensor
    scales: torch.Tensor
    zeros: torch.Tensor

    def c_struct(self) -> QwhaQweight:
        s = QwhaQweight()
        s.bits, s.group = self.bits, self.group
        s.qweight, s.scales, s.zeros = self.qweight.data_ptr(), self.scales.data_ptr(), self.zeros.data_ptr()
        return s


def workspace_size(op: int, d_out: int, d_in: int, p: int, T: int, with_base: bool) -> int:
    return int(lib().qwha_workspace_size(op, d_out, d_in, p, T, int(bool(with_base))))


def plan_tiles(d_out: int, d_in: int) -> int:
    return int(lib().qwha_plan_tiles(d_out, d_in))


def fwht(x: torch.Tensor, had_block: int | None = None, out: torch.Tensor | None = None) -> torch.Tensor:
    """Z = X H over the last dimension (block-diagonal with blocks of had_block)."""
    n = x.shape[-1]
    had_block = had_block or n
    out = torch.empty_like(x) if out is None else out
    rows = x.numel() // n if n else 0
    check(lib().qwha_fwht(_dt(x), _ptr(x), _ptr(out), rows, n, had_block, _stream()), "qwha_fwht")
    return out


def adapter_fwd(a: Adapter, X: torch.Tensor, alpha: float = 1.0, wq: QWeight | None = None,
                Z_out: torch.Tensor | None = None, Y: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                z_given: bool = False):
    """(Z, Y) with Z = X H and Y = X W_Q^T + alpha Z F^T (W_Q term only with wq).
    z_given: Z_out already holds X H (from the forward of another layer reading the same X with the same
    had_block) and is read instead of computed."""
    T = X.shape[0]
    if z_given and Z_out is None:
        raise ValueError("z_given needs Z_out")
    Z_out = torch.empty_like(X) if Z_out is None else Z_out
    Y = torch.empty((T, a.d_out), dtype=X.dtype, device=X.device) if Y is None else Y
    need = workspace_size(OP_FWD_DENSE if a.algo == "dense" else OP_FWD, a.d_out, a.d_in, a.p, T, wq is not None)
    ws = _ws(need, X.device) if ws is None else ws
    cs = a.c_struct()
    cs.z_given = 1 if z_given else 0
    cw = wq.c_struct() if wq is not None else None
    rc = lib().qwha_adapter_fwd(ctypes.byref(cs), ctypes.byref(cw) if cw is not None else None, _dt(X), _ptr(X), T,
                                float(alpha), _ptr(Z_out), _ptr(Y), _ptr(ws), 0 if ws is None else ws.numel(), _stream())
    check(rc, "qwha_adapter_fwd")
    return Z_out, Y


def adapter_bwd(a: Adapter, dY: torch.Tensor, Z: torch.Tensor, alpha: float = 1.0, wq: QWeight | None = None,
                dc: torch.Tensor | None = None, dX: torch.Tensor | None = None, want_dx: bool = True,
                ws: torch.Tensor | None = None, want_dc: bool = True):
    """(dc, dX): dc_j = alpha sum_t dY[t,r_j] Z[t,k_j]; dX = dY W_Q + alpha (dY F) H.
    want_dc / want_dx False skip that output (returned as None): a data-parallel step computes dc, starts its
    all-reduce, then computes dX while the all-reduce runs."""
    T = dY.shape[0]
    if want_dc and dc is None:
        dc = torch.empty(a.p, dtype=torch.float32, device=dY.device)
    if want_dx and dX is None:
        dX = torch.empty((T, a.d_in), dtype=dY.dtype, device=dY.device)
    need = workspace_size(OP_BWD_DENSE if a.algo == "dense" else OP_BWD, a.d_out, a.d_in, a.p, T, wq is not None)
    ws = _ws(need, dY.device) if ws is None else ws
    cs = a.c_struct()
    cw = wq.c_struct() if wq is not None else None
    rc = lib().qwha_adapter_bwd(ctypes.byref(cs), ctypes.byref(cw) if cw is not None else None, _dt(dY), _ptr(dY),
                                _ptr(Z), T, float(alpha), _ptr(dc) if want_dc else None,
                                _ptr(dX) if want_dx else None, _ptr(ws), 0 if ws is None else ws.numel(), _stream())
    check(rc, "qwha_adapter_bwd")
    return (dc if want_dc else None), (dX if want_dx else None)


def dp_backward(a: Adapter, dY: torch.Tensor, Z: torch.Tensor, alpha: float = 1.0, wq: QWeight | None = None,
                dc: torch.Tensor | None = None, dX: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                group=None, bwd=None):
    """Backward of one adapted layer under token data parallelism: every rank holds its own token rows of dY and Z.

    dc is a sum over tokens, so it is the one quantity the ranks exchange (only c trains: papernotes.org "QWHA",
    整体框架 and 训练策略); dX of a token needs only that token. The call computes this rank's dc first
    (qwha_adapter_bwd with dX NULL), starts an asynchronous all-reduce (sum) of it over `group`, computes this
    rank's dX (dc NULL) while the all-reduce runs, and waits for it. Returns (dc summed over the ranks, dX of this
    rank's tokens); without an initialised process group it is the single-process backward.

    `bwd` replaces adapter_bwd (same signature); the collective runs on whatever device the tensors live on."""
    import torch.distributed as dist

    bwd = bwd or adapter_bwd
    dc, _ = bwd(a, dY, Z, alpha, wq, dc=dc, want_dx=False, ws=ws)
    work = None
    if dist.is_available() and dist.is_initialized():
        work = dist.all_reduce(dc, group=group, async_op=True)
    _, dX = bwd(a, dY, Z, alpha, wq, dX=dX, want_dc=False, ws=ws)
    if work is not None:
        work.wait()
    return dc, dX


def dp_step(a: Adapter, X: torch.Tensor, dY: torch.Tensor, alpha: float = 1.0, wq: QWeight | None = None,
            Z: torch.Tensor | None = None, Y: torch.Tensor | None = None, dc: torch.Tensor | None = None,
            dX: torch.Tensor | None = None, ws_fwd: torch.Tensor | None = None, ws_bwd: torch.Tensor | None = None,
            group=None, fwd=None, bwd=None):
    """One data-parallel training step of the layer on this rank's tokens: the forward (Z, Y), then dp_backward.
    Returns (Z, Y, dc summed over the ranks, dX). `fwd` / `bwd` replace adapter_fwd / adapter_bwd."""
    fwd = fwd or adapter_fwd
    Z, Y = fwd(a, X, alpha, wq, Z_out=Z, Y=Y, ws=ws_fwd)
    dc, dX = dp_backward(a, dY, Z, alpha, wq, dc=dc, dX=dX, ws=ws_bwd, group=group, bwd=bwd)
    return Z, Y, dc, dX


def init_alloc(dWq: torch.Tensor, p: int, had_block: int, min_per_row: int = 2, mode: str = "fewest",
               ws: torch.Tensor | None = None) -> dict:
    """AdaAlloc on the device: dict(budgets, row_ptr, col_idx, coef)."""
    d_out, d_in = dWq.shape
    dev = dWq.device
    out = dict(
        budgets=torch.empty(d_out, dtype=torch.int32, device=dev),
        row_ptr=torch.empty(d_out + 1, dtype=torch.int32, device=dev),
        col_idx=torch.empty(max(p, 1), dtype=torch.int32, device=dev),
        coef=torch.empty(max(p, 1), dtype=torch.float32, device=dev),
    )
    need = workspace_size(OP_INIT, d_out, d_in, p, 0, False)
    ws = _ws(need, dev) if ws is None else ws
    rc = lib().qwha_init_alloc(_ptr(dWq), d_out, d_in, had_block, p, min_per_row, REMAINDER[mode],
                               _ptr(out["budgets"]), _ptr(out["row_ptr"]), _ptr(out["col_idx"]), _ptr(out["coef"]),
                               _ptr(ws), 0 if ws is None else ws.numel(), _stream())
    check(rc, "qwha_init_alloc")
    out["col_idx"], out["coef"] = out["col_idx"][:p], out["coef"][:p]
    return out


def init_select_global(dWq: torch.Tensor, p: int, had_block: int, sel: str = "magnitude", seed: int = 0,
                       ws: torch.Tensor | None = None) -> dict:
    """E and c by a whole-matrix rule ("magnitude": the p largest |V|; "random": p seeded uniform positions):
    dict(budgets, row_ptr, col_idx, coef)."""
    d_out, d_in = dWq.shape
    dev = dWq.device
    out = dict(
        budgets=torch.empty(d_out, dtype=torch.int32, device=dev),
        row_ptr=torch.empty(d_out + 1, dtype=torch.int32, device=dev),
        col_idx=torch.empty(max(p, 1), dtype=torch.int32, device=dev),
        coef=torch.empty(max(p, 1), dtype=torch.float32, device=dev),
    )
    need = workspace_size(OP_SELECT_GLOBAL, d_out, d_in, p, 0, False)
    ws = _ws(need, dev) if ws is None else ws
    rc = lib().qwha_init_select_global(_ptr(dWq), d_out, d_in, had_block, p, SELECTION[sel], seed & (2**64 - 1),
                                       _ptr(out["budgets"]), _ptr(out["row_ptr"]), _ptr(out["col_idx"]),
                                       _ptr(out["coef"]), _ptr(ws), 0 if ws is None else ws.numel(), _stream())
    check(rc, "qwha_init_select_global")
    out["col_idx"], out["coef"] = out["col_idx"][:p], out["coef"][:p]
    return out


def energy_stats(dWq: torch.Tensor, k: int, had_block: int, ws: torch.Tensor | None = None) -> torch.Tensor:
    """Hill exponent eta and cumulative energy of the k largest |dW_Q H| (qwha_energy_stats): fp64 device tensor
    [eta, energy fraction of the k largest, a_(k+1), sum of all a^2]."""
    d_out, d_in = dWq.shape
    out = torch.empty(4, dtype=torch.float64, device=dWq.device)
    need = workspace_size(OP_ENERGY, d_out, d_in, 0, 0, False)
    ws = _ws(need, dWq.device) if ws is None else ws
    check(lib().qwha_energy_stats(_ptr(dWq), d_out, d_in, had_block, int(k), _ptr(out), _ptr(ws),
                                  0 if ws is None else ws.numel(), _stream()), "qwha_energy_stats")
    return out


def pattern_stats(row_ptr: torch.Tensor, col_idx: torch.Tensor, d_in: int,
                  ws: torch.Tensor | None = None) -> tuple[torch.Tensor, torch.Tensor]:
    """(stats int64 [8] in the order of PATTERN_STATS, col_counts int32 [d_in]) of E (qwha_pattern_stats)."""
    d_out = row_ptr.numel() - 1
    p = col_idx.numel()
    dev = row_ptr.device
    stats = torch.empty(8, dtype=torch.int64, device=dev)
    cc = torch.empty(d_in, dtype=torch.int32, device=dev)
    need = workspace_size(OP_PATTERN, d_out, d_in, p, 0, False)
    ws = _ws(need, dev) if ws is None else ws
    check(lib().qwha_pattern_stats(d_out, d_in, p, _ptr(row_ptr), _ptr(col_idx) if p else None, _ptr(cc),
                                   _ptr(stats), _ptr(ws), 0 if ws is None else ws.numel(), _stream()),
          "qwha_pattern_stats")
    return stats, cc


def calib_hessian(X: torch.Tensor, S: torch.Tensor | None = None) -> torch.Tensor:
    """S = X^T X (fp32 [d_in, d_in]) from bf16 calibration rows X [T, d_in]."""
    T, d_in = X.shape
    S = torch.empty((d_in, d_in), dtype=torch.float32, device=X.device) if S is None else S
    check(lib().qwha_calib_hessian(_ptr(X), T, d_in, _ptr(S), _stream()), "qwha_calib_hessian")
    return S


def refine_values(dWq: torch.Tensor, S: torch.Tensor, row_ptr: torch.Tensor, col_idx: torch.Tensor, had_block: int,
                  damp: float = 0.01, coef: torch.Tensor | None = None, ws: torch.Tensor | None = None) -> torch.Tensor:
    """Value Refinement: least-squares coefficients at E (row_ptr, col_idx) for the calibration Hessian S."""
    d_out, d_in = dWq.shape
    p = col_idx.numel()
    coef = torch.empty(max(p, 1), dtype=torch.float32, device=dWq.device) if coef is None else coef
    need = workspace_size(OP_REFINE, d_out, d_in, p, 0, False)
    ws = _ws(need, dWq.device) if ws is None else ws
    rc = lib().qwha_refine_values(_ptr(dWq), d_out, d_in, had_block, _ptr(S), float(damp), _ptr(row_ptr),
                                  _ptr(col_idx) if p else None, p, _ptr(coef), _ptr(ws), 0 if ws is None else ws.numel(),
                                  _stream())
    check(rc, "qwha_refine_values")
    return coef[:p]


def init_norms(dWq_rows: torch.Tensor) -> torch.Tensor:
    """e[i] = ||dWq_rows[i, :]||_2 in fp64 (the first step of AdaAlloc) for a block of rows."""
    rows, d_in = dWq_rows.shape
    e = torch.empty(rows, dtype=torch.float64, device=dWq_rows.device)
    check(lib().qwha_init_norms(_ptr(dWq_rows), rows, d_in, _ptr(e), _stream()), "qwha_init_norms")
    return e


def init_budgets(e: torch.Tensor, d_in: int, p: int, min_per_row: int = 2, mode: str = "fewest",
                 ws: torch.Tensor | None = None) -> tuple[torch.Tensor, torch.Tensor]:
    """(budgets [d_out], row_ptr [d_out+1]) from all d_out row norms (fp64)."""
    d_out = e.shape[0]
    dev = e.device
    budgets = torch.empty(d_out, dtype=torch.int32, device=dev)
    row_ptr = torch.empty(d_out + 1, dtype=torch.int32, device=dev)
    need = workspace_size(OP_INIT, d_out, d_in, p, 0, False)
    ws = _ws(need, dev) if ws is None else ws
    rc = lib().qwha_init_budgets(_ptr(e), d_out, d_in, p, min_per_row, REMAINDER[mode], _ptr(budgets), _ptr(row_ptr),
                                 _ptr(ws), 0 if ws is None else ws.numel(), _stream())
    check(rc, "qwha_init_budgets")
    return budgets, row_ptr


def init_select(dWq_rows: torch.Tensor, had_block: int, budgets: torch.Tensor,
                row_ptr: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor]:
    """(col_idx, coef) of a block of rows: budgets [rows] and row_ptr [rows+1] are the block's slices of the global
    budgets and row_ptr (row_ptr need not start at 0)."""
    rows, d_in = dWq_rows.shape
    p_local = int(row_ptr[-1].item() - row_ptr[0].item()) if rows else 0
    dev = dWq_rows.device
    # the ABI takes 16-byte aligned pointers: a slice that starts elsewhere is copied
    dWq_rows, budgets, row_ptr = (t if t.data_ptr() % 16 == 0 else t.clone() for t in (dWq_rows, budgets, row_ptr))
    col_idx = torch.empty(max(p_local, 1), dtype=torch.int32, device=dev)
    coef = torch.empty(max(p_local, 1), dtype=torch.float32, device=dev)
    rc = lib().qwha_init_select(_ptr(dWq_rows), rows, d_in, had_block, _ptr(budgets), _ptr(row_ptr), p_local,
                                _ptr(col_idx), _ptr(coef), _stream())
    check(rc, "qwha_init_select")
    return col_idx[:p_local], coef[:p_local]


def shard_rows(d_out: int, rank: int, world: int) -> tuple[int, int]:
    """Rows [r0, r1) of output channels held by `rank` of `world` in sharded AdaAlloc."""
    return rank * d_out // world, (rank + 1) * d_out // world


def init_alloc_sharded(dWq_rows: torch.Tensor, d_out: int, p: int, had_block: int, min_per_row: int = 2,
                       mode: str = "fewest", group=None, steps=None) -> dict:
    """AdaAlloc with the rows of dW_Q sharded over the ranks of `group` (rank r holds rows shard_rows(d_out, r,
    world)): the ranks exchange their row norms (fp64), compute the same budgets from all of them, select E and c
    for their own rows and exchange the CSR slices. Every rank returns the full result of init_alloc on the whole
    dW_Q: dict(budgets, row_ptr, col_idx, coef).

    `steps` = (norms, budgets, select) replaces the three device steps (defaults: init_norms, init_budgets,
    init_select); the collectives run on whatever device the tensors live on."""
    import torch.distributed as dist

    norms_fn, budgets_fn, select_fn = steps or (init_norms, init_budgets, init_select)
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    r0, r1 = shard_rows(d_out, rank, world)
    d_in = dWq_rows.shape[1]
    if dWq_rows.shape[0] != r1 - r0:
        raise ValueError(f"rank {rank} holds {dWq_rows.shape[0]} rows, expected {r1 - r0}")
    e_local = norms_fn(dWq_rows)
    bounds = [shard_rows(d_out, r, world) for r in range(world)]
    most = max(b1 - b0 for b0, b1 in bounds)
    pad = torch.zeros(most, dtype=torch.float64, device=e_local.device)
    pad[: r1 - r0] = e_local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    e_all = torch.cat([parts[r][: b1 - b0] for r, (b0, b1) in enumerate(bounds)])
    budgets, row_ptr = budgets_fn(e_all, d_in, p, min_per_row, mode)
    col_local, coef_local = select_fn(dWq_rows, had_block, budgets[r0:r1], row_ptr[r0:r1 + 1])
    rp_host = row_ptr.cpu()
    sizes = [int(rp_host[b1] - rp_host[b0]) for b0, b1 in bounds]
    cap = max(max(sizes), 1)
    out = {}
    for name, t in (("col_idx", col_local), ("coef", coef_local)):
        buf = torch.zeros(cap, dtype=t.dtype, device=t.device)
        buf[: t.numel()] = t
        gathered = [torch.empty_like(buf) for _ in range(world)]
        dist.all_gather(gathered, buf, group=group)
        out[name] = torch.cat([gathered[r][: sizes[r]] for r in range(world)])
    out["budgets"], out["row_ptr"] = budgets, row_ptr
    return out


def plan_build(a: Adapter, ws: torch.Tensor | None = None) -> Adapter:
    """Fill the CSC and tile views of `a` (new tensors) and return it."""
    dev = a.row_ptr.device
    n_tiles = plan_tiles(a.d_out, a.d_in)
    pp = max(a.p, 1)
    a.col_ptr = torch.empty(a.d_in + 1, dtype=torch.int32, device=dev)
    a.row_idx = torch.empty(pp, dtype=torch.int32, device=dev)
    a.perm = torch.empty(pp, dtype=torch.int32, device=dev)
    a.tile_ptr = torch.empty(n_tiles + 1, dtype=torch.int32, device=dev)
    a.tile_pos = torch.empty(pp, dtype=torch.int32, device=dev)
    a.tile_rk = torch.empty(pp, dtype=torch.int32, device=dev)
    need = workspace_size(OP_PLAN, a.d_out, a.d_in, a.p, 0, False)
    ws = _ws(need, dev) if ws is None else ws
    rc = lib().qwha_plan_build(a.d_out, a.d_in, a.p, _ptr(a.row_ptr), _ptr(a.col_idx), _ptr(a.col_ptr),
                               _ptr(a.row_idx), _ptr(a.perm), _ptr(a.tile_ptr), _ptr(a.tile_pos), _ptr(a.tile_rk),
                               _ptr(ws), 0 if ws is None else ws.numel(), _stream())
    check(rc, "qwha_plan_build")
    return a


def validate_plan(a: Adapter) -> None:
    cs = a.c_struct()
    check(lib().qwha_validate_plan(ctypes.byref(cs), _stream()), "qwha_validate_plan")


def stage_timing(enable: bool) -> None:
    """Turn the library's per-stage event timing on or off."""
    lib().qwha_stage_timing(int(bool(enable)))


def stage_report() -> dict:
    """{stage: (calls, kernel launches, total ms)} since the previous report (synchronises)."""
    import numpy as np

    h = lib()
    n = h.qwha_stage_count()
    calls = np.zeros(n, dtype=np.int64)
    launches = np.zeros(n, dtype=np.int64)
    ms = np.zeros(n, dtype=np.float64)
    check(h.qwha_stage_report(calls.ctypes.data_as(ctypes.c_void_p), launches.ctypes.data_as(ctypes.c_void_p),
                              ms.ctypes.data_as(ctypes.c_void_p)), "qwha_stage_report")
    return {h.qwha_stage_name(i).decode(): (int(calls[i]), int(launches[i]), float(ms[i])) for i in range(n)}
