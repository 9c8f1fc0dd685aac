"""Shared helpers of the test suite (no method arithmetic here)."""

import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qwha.h")

# Tolerances on the relative Frobenius error against the fp64 oracle.
TOL_F32 = 1e-5
TOL_BF16 = 2e-2


def rel_fro(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def header_functions() -> list[str]:
    """Names of the functions declared in include/qwha.h."""
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(qwha_[a-z_]+)\s*\(", src)))


def to_dev(a, dtype=None):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def bf16_dev(bits):
    """uint16 bf16 bit patterns (numpy) -> CUDA bfloat16 tensor with the same bits."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16))
    return t.cuda().view(torch.bfloat16)


def host(t) -> np.ndarray:
    """CUDA tensor -> float64 numpy (bf16 widened exactly)."""
    import torch

    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy().astype(np.float64)
