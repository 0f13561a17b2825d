"""Helpers shared by the GPU parity tests: host<->device transfer of storage
arrays and the element-wise comparison rule.

Comparison rule (fp32 accumulation, tolerance stated per storage dtype):
    |gpu - oracle| <= rtol * max(|oracle|, rms(oracle over the token's row))
with rtol = 1e-5 for fp32 storage and 2e-2 for bf16 storage. The rms floor
keeps near-zero outputs from dominating the relative error.
"""
from __future__ import annotations

import numpy as np
import torch

RTOL = {"f32": 1e-5, "bf16": 2e-2}
TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def to_dev(a: np.ndarray, dt: str, device="cuda") -> torch.Tensor:
    """Upload a storage array (bf16 as uint16 bit patterns) to the device."""
    a = np.ascontiguousarray(a)
    if dt == "bf16":
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(a.astype(np.float32, copy=False)).to(device)


def f32_dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def to_host(t: torch.Tensor, dt: str) -> np.ndarray:
    t = t.detach().contiguous().cpu()
    if dt == "bf16":
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    return t.numpy().astype(np.float32, copy=True)


def values(a: np.ndarray, dt: str) -> np.ndarray:
    """Storage array -> float64 values."""
    if dt == "bf16":
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def rel_err(gpu: np.ndarray, ref: np.ndarray, dt: str, token_axes: int = 1) -> float:
    """Max over elements of |g - o| / max(|o|, rms of o over the token's row)."""
    g, o = values(gpu, dt), values(ref, dt)
    lead = o.shape[:token_axes]
    o2 = o.reshape(*lead, -1)
    rms = np.sqrt(np.mean(o2 * o2, axis=-1, keepdims=True))
    den = np.maximum(np.abs(o2), rms)
    den = np.where(den == 0, 1.0, den)
    return float(np.max(np.abs(g.reshape(*lead, -1) - o2) / den)) if o.size else 0.0


def assert_close(gpu, ref, dt, what="", token_axes=1):
    e = rel_err(gpu, ref, dt, token_axes)
    assert e <= RTOL[dt], f"{what}: max rel err {e:.3e} > {RTOL[dt]:.0e}"
    return e


def assert_bitwise(gpu, ref, what=""):
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    if not np.array_equal(gpu, ref):
        bad = np.argwhere(gpu != ref)
        raise AssertionError(f"{what}: {len(bad)} of {gpu.size} elements differ; first at "
                             f"{tuple(bad[0])}: gpu={gpu[tuple(bad[0])]} oracle={ref[tuple(bad[0])]}")
