"""Shared helpers for the GPU parity tests (device transfer, error metrics)."""
from __future__ import annotations

import numpy as np
import torch

TOL = {"f32": 1e-4, "bf16": 2e-2}   # normalised max-abs tolerances for o and S


def dev_inputs(inp: dict, dtype: str, device="cuda") -> dict:
    """numpy inputs (float32 arrays holding bf16-exact values) -> CUDA tensors."""
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = {}
    for key in ("q", "k", "v"):
        out[key] = torch.from_numpy(np.ascontiguousarray(inp[key])).to(device=device).to(tdt)
    out["log_alpha"] = torch.from_numpy(np.ascontiguousarray(inp["log_alpha"])).to(device)
    out["beta"] = torch.from_numpy(np.ascontiguousarray(inp["beta"])).to(device)
    if "cu_seqlens" in inp:
        out["cu_seqlens"] = torch.from_numpy(np.ascontiguousarray(inp["cu_seqlens"])).to(device)
    if inp.get("pad_mask") is not None:
        out["pad_mask"] = torch.from_numpy(np.ascontiguousarray(inp["pad_mask"])).to(device)
    if inp.get("init_state") is not None:
        out["init_state"] = torch.from_numpy(np.ascontiguousarray(inp["init_state"])).to(device)
    return out


def norm_err(got, ref) -> float:
    """max|got - ref| / max|ref| (the tolerance metric of the parity tests)."""
    g = np.asarray(got, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    den = np.abs(r).max()
    num = np.abs(g - r).max() if g.size else 0.0
    return float(num / den) if den > 0 else float(num)


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()
