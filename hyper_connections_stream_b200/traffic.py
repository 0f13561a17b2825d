"""Algorithmic HBM bytes of the Hyper-Connections step (the roofline numerator).

"Algorithmic" means each operand is read once and each result written once;
anything above that in a DRAM counter is re-reading. Storage element size s is
2 (bf16) or 4 (fp32); parameters are fp32.

The per-token residual state is n*d*s bytes, n times the one-stream state
("Tencent open-sources Hy4 Preview at 770B -- Identity Hyper-Connections",
section "What four streams cost per token": 16 KB -> 64 KB at d = 8192 bf16).
"""
from __future__ import annotations

DTYPE_BYTES = {"bf16": 2, "f32": 4}


def state_bytes_per_token(n: int, d: int, s: int) -> int:
    """Bytes of residual state one token carries across a layer boundary."""
    return n * d * s


def _param_bytes(n: int, per_token_mix: bool, per_token_b: bool, per_token_read: bool,
                 write: bool, read: bool):
    """(bytes per token, bytes per launch) of the fp32 mixing parameters."""
    tok = launch = 0
    if write:
        if per_token_mix:
            tok += 4 * n * n
        else:
            launch += 4 * n * n
        if per_token_b:
            tok += 4 * n
        else:
            launch += 4 * n
    if read:
        if per_token_read:
            tok += 4 * n
        else:
            launch += 4 * n
    return tok, launch


def step_bytes(kind: str, T: int, n: int, d: int, dtype: str, *, per_token_mix: bool = False,
               per_token_b: bool = False, per_token_read: bool = False,
               gain: bool = True) -> int:
    """Minimum HBM bytes of one launch.

    kind: "read"  (H -> x):            s*d*(n+1) per token
          "write" (H, y -> H'):        s*d*(2n+1) per token
          "fused" (H, y -> H', x):     s*d*(2n+2) per token
          "sinkhorn" (L -> A, fp32):   8*n*n per token
    plus the fp32 parameters (per token, or once per launch) and the gain g.
    """
    s = DTYPE_BYTES[dtype]
    if kind == "sinkhorn":
        return T * 8 * n * n
    write = kind in ("write", "fused")
    read = kind in ("read", "fused")
    per_tok = {"read": s * d * (n + 1), "write": s * d * (2 * n + 1),
               "fused": s * d * (2 * n + 2)}[kind]
    ptok, plaunch = _param_bytes(n, per_token_mix, per_token_b, per_token_read, write, read)
    g_bytes = 4 * d if (read and gain) else 0
    return T * (per_tok + ptok) + plaunch + g_bytes


def step_flops_per_token(kind: str, n: int, d: int) -> int:
    """fp32 multiply-adds x2 of the mixes (Sinkhorn and the statistic excluded)."""
    write = 2 * (n * n + n) * d
    read = 2 * n * d + 3 * d
    return {"write": write, "read": read, "fused": write + read}[kind]
