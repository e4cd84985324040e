"""Shared helpers of the GPU tests: upload seeded inputs, normwise errors."""

from __future__ import annotations

import numpy as np
import torch

TOL = {"bf16": 5e-3, "f32": 1e-5}


def to_device(inp, dtype: str, device="cuda"):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    return {k: torch.from_numpy(v).to(device=device, dtype=tdt).contiguous() for k, v in inp.items()}


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def host(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)
