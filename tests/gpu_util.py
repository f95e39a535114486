"""Helpers shared by the GPU tests: NumPy bf16 bit patterns <-> torch tensors
and the output tolerance checks (derived in the design notes: the GPU's int32
accumulator is exact, the fp32 epilogue adds a few ulp and the bf16 store half
an ulp of bf16, so elementwise |Y - ref| <= 2^-8 |ref| holds with margin; the
gate is max|Y - ref| / max|ref| <= 1e-2, or 2e-2 with the bf16 low-rank
branch)."""
from __future__ import annotations

import numpy as np


def dev_bf16(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def host_bits(t) -> np.ndarray:
    import torch
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def host_f64(t) -> np.ndarray:
    import torch
    return t.detach().float().cpu().numpy().astype(np.float64)


def max_rel(got: np.ndarray, ref: np.ndarray) -> float:
    denom = float(np.max(np.abs(ref)))
    return float(np.max(np.abs(got - ref))) / (denom if denom > 0 else 1.0)


def check_output(got: np.ndarray, ref: np.ndarray, lowrank: bool):
    gate = 2e-2 if lowrank else 1e-2
    mr = max_rel(got, ref)
    assert mr <= gate, f"max-rel {mr:.3e} > {gate}"
    if not lowrank:
        bound = 2.0 ** -8 * np.abs(ref) + 1e-6 * np.max(np.abs(ref))
        bad = np.count_nonzero(np.abs(got - ref) > bound)
        assert bad == 0, f"{bad} outputs outside 2^-8 relative"
    return mr
