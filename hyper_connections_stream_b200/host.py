"""Running the HC step on stream state that lives in host memory.

`write_then_read_from_host` takes pinned host tensors, splits the tokens into
chunks and runs each chunk's host->device copies, the fused step and the
device->host copies on one of several CUDA streams, so the copies of one chunk
overlap the kernel of another and both PCIe directions stay busy. The step
itself is the library's kernel (`_lib.write_then_read`); this module only
moves data and orders streams. Device staging buffers are allocated here
through torch (the C library itself never allocates).
"""
from __future__ import annotations

import torch

from . import _lib


class HostStepper:
    """Reusable staging buffers and streams for `write_then_read_from_host`."""

    def __init__(self, max_chunk_tokens: int, n: int, d: int, dtype: torch.dtype, device,
                 per_token_mix: bool, per_token_read: bool, streams: int = 3):
        self.device = torch.device(device)
        self.chunk = int(max_chunk_tokens)
        self.streams = [torch.cuda.Stream(device=self.device) for _ in range(streams)]
        mk = lambda *shape, dt=dtype: torch.empty(shape, dtype=dt, device=self.device)
        self.H = [mk(self.chunk, n, d) for _ in range(streams)]
        self.y = [mk(self.chunk, d) for _ in range(streams)]
        self.x = [mk(self.chunk, d) for _ in range(streams)]
        self.A = [mk(self.chunk, n, n, dt=torch.float32) if per_token_mix else None
                  for _ in range(streams)]
        self.a = [mk(self.chunk, n, dt=torch.float32) if per_token_read else None
                  for _ in range(streams)]


def write_then_read_from_host(H, y, A, b, a_next, g_next, *, out_H, out_x, eps: float = 1e-6,
                              mix: int = _lib.MIX_MATRIX, K: int = 0,
                              read: int = _lib.READ_WEIGHTS, stepper: HostStepper | None = None,
                              chunks: int = 8):
    """Fused step on host-resident state.

    H [T,n,d], y [T,d] and the per-token parameters A [T,n,n] / a_next [T,n]
    (if per token) are pinned host tensors; b, g_next and shared A / a_next are
    device tensors. Results land in the pinned host tensors out_H and out_x.
    Work is enqueued behind the current stream and the current stream waits
    for all of it, so callers order and time it like any other launch.
    """
    T, n, d = H.shape
    per_mix = A.dim() == 3
    per_read = a_next.dim() == 2
    chunk = (T + chunks - 1) // chunks
    if stepper is None:
        stepper = HostStepper(chunk, n, d, H.dtype, b.device, per_mix, per_read)
    if stepper.chunk < chunk:
        raise ValueError("stepper staging buffers are smaller than one chunk")
    cur = torch.cuda.current_stream(stepper.device)
    start = torch.cuda.Event()
    start.record(cur)
    done = []
    for c, t0 in enumerate(range(0, T, chunk)):
        t1 = min(T, t0 + chunk)
        m = t1 - t0
        s = c % len(stepper.streams)
        st = stepper.streams[s]
        st.wait_event(start)
        with torch.cuda.stream(st):
            dH, dy, dx = stepper.H[s][:m], stepper.y[s][:m], stepper.x[s][:m]
            dH.copy_(H[t0:t1], non_blocking=True)
            dy.copy_(y[t0:t1], non_blocking=True)
            dA = A
            if per_mix:
                dA = stepper.A[s][:m]
                dA.copy_(A[t0:t1], non_blocking=True)
            da = a_next
            if per_read:
                da = stepper.a[s][:m]
                da.copy_(a_next[t0:t1], non_blocking=True)
            _lib.write_then_read(dH, dy, dA, b, da, g_next, eps=eps, mix=mix, K=K, read=read,
                                 out=dH, x_next=dx)
            out_H[t0:t1].copy_(dH, non_blocking=True)
            out_x[t0:t1].copy_(dx, non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(st)
            done.append(ev)
    for ev in done:
        cur.wait_event(ev)
    return out_H, out_x
