"""B200 (sm_100a) Walsh-Hadamard adapter layer: Python binding of libqwha.

The arithmetic runs in the CUDA kernels of libqwha.so; this package only
marshals torch tensors (device memory and the current stream) into the C ABI
of include/qwha.h. Import fails if the library is not built.
"""

from ._lib import QwhaError, lib  # noqa: F401
from .api import (  # noqa: F401
    Adapter,
    QWeight,
    adapter_bwd,
    adapter_fwd,
    calib_hessian,
    dp_backward,
    dp_step,
    energy_stats,
    fwht,
    init_alloc,
    init_alloc_sharded,
    init_budgets,
    init_norms,
    init_select,
    init_select_global,
    pattern_stats,
    plan_build,
    plan_tiles,
    refine_values,
    shard_rows,
    stage_report,
    stage_timing,
    validate_plan,
    workspace_size,
)

lib()  # fail loudly at import when libqwha.so is missing
