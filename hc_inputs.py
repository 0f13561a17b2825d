"""Seeded synthetic inputs for the Hyper-Connections residual step.

This module is the only code that the CUDA path's tests and the CPU oracle's
tests share. It holds no arithmetic of the method: it draws random numbers,
rounds them to the storage dtype with torch's own conversion, and lays them
out. Everything is synthetic (the pages measure on no dataset).

Layout: streams H[T][n][d] (token-major, a token's n rows contiguous), block
output y[T][d], fp32 parameters a[n] / A[n][n] / b[n] / g[d] (one set per
layer) or per token a[T][n] / A[T][n][n] / b[T][n], Sinkhorn logits
L[T][n][n] and read logits l[T][n].

Seeds: H = 1000 + cfg, y = 2000 + cfg, parameters = 3000 + cfg + layer,
logits = 4000 + cfg.

Storage "bf16" host arrays are np.uint16 bit patterns; "f32" are np.float32.
"""
from __future__ import annotations

import numpy as np
import torch

SEED_H, SEED_Y, SEED_P, SEED_L = 1000, 2000, 3000, 4000


def to_storage(x32: np.ndarray, dt: str) -> np.ndarray:
    """fp32 -> storage dtype through torch's conversion (round to nearest even)."""
    x32 = np.ascontiguousarray(x32, dtype=np.float32)
    if dt == "f32":
        return x32
    t = torch.from_numpy(x32).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def normal(seed: int, shape, std: float = 1.0, mean: float = 0.0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return (rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std)
            + np.float32(mean)).astype(np.float32)


def uniform(seed: int, shape, lo: float, hi: float) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return rng.uniform(lo, hi, size=shape).astype(np.float32)


def streams(cfg: int, T: int, n: int, d: int, dt: str) -> np.ndarray:
    """H ~ N(0,1), independent streams."""
    return to_storage(normal(SEED_H + cfg, (T, n, d)), dt)


def copied_streams(cfg: int, T: int, n: int, d: int, dt: str) -> np.ndarray:
    """n identical copies of one N(0,1) stream (the identity-init start state)."""
    one = to_storage(normal(SEED_H + cfg, (T, 1, d)), dt)
    return np.ascontiguousarray(np.repeat(one, n, axis=1))


def block_out(cfg: int, T: int, d: int, dt: str) -> np.ndarray:
    """y ~ N(0,1): a block output given as input."""
    return to_storage(normal(SEED_Y + cfg, (T, d)), dt)


def static_params(cfg: int, n: int, layer: int = 0, std: float = 0.02):
    """Per-layer a = e_0 + N(0,std), A = I + N(0,std), b = 1 + N(0,std)."""
    rng = np.random.default_rng(SEED_P + cfg + layer)
    a = np.zeros(n, np.float32)
    a[0] = 1.0
    a = (a + rng.standard_normal(n).astype(np.float32) * np.float32(std)).astype(np.float32)
    A = (np.eye(n, dtype=np.float32)
         + rng.standard_normal((n, n)).astype(np.float32) * np.float32(std)).astype(np.float32)
    b = (np.ones(n, np.float32)
         + rng.standard_normal(n).astype(np.float32) * np.float32(std)).astype(np.float32)
    return a, A, b


def identity_params(n: int):
    """a = e_0, A = I, b = 1 (the identity initialisation)."""
    a = np.zeros(n, np.float32)
    a[0] = 1.0
    return a, np.eye(n, dtype=np.float32), np.ones(n, np.float32)


def gain(cfg: int, d: int, layer: int = 0, lo: float = 0.5, hi: float = 1.5) -> np.ndarray:
    """Per-layer per-channel RMSNorm gain g ~ U(lo, hi)."""
    return uniform(SEED_P + 500 + cfg + layer, (d,), lo, hi)


def mix_logits(cfg: int, T: int, n: int) -> np.ndarray:
    """Per-token Sinkhorn logits L ~ N(0,1), [T, n, n]."""
    return normal(SEED_L + cfg, (T, n, n))


def read_logits(cfg: int, T: int, n: int) -> np.ndarray:
    """Per-token read-weight logits ~ N(0,1), [T, n]."""
    return normal(SEED_L + 100 + cfg, (T, n))


# ---- device-side generation for sizes the host should not materialise -------

def device_normal(seed: int, shape, dtype: torch.dtype, device, std: float = 1.0,
                  mean: float = 0.0) -> torch.Tensor:
    """N(mean, std) drawn with a seeded torch generator on `device`, then cast
    (torch's round-to-nearest-even) to the storage dtype."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    out = torch.empty(shape, dtype=torch.float32, device=device)
    out.normal_(mean=mean, std=std, generator=gen)
    return out.to(dtype)


TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def torch_to_storage_np(t: torch.Tensor, dt: str) -> np.ndarray:
    """Host numpy view of a storage tensor (bf16 -> uint16 bit patterns)."""
    t = t.detach().contiguous().cpu()
    if dt == "bf16":
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    return t.numpy().astype(np.float32, copy=True)
