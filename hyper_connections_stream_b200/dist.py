"""Multi-process plumbing for running the HC step on several GPUs of a node.

The step shards with no collective: every token is independent (the mixes act
within a token's n streams and RMSNorm within one token), so N ranks each run
their own tokens. torch.distributed carries only the barrier and the
max-over-ranks timing. Works with NCCL (tensors on the rank's GPU) and gloo
(CPU tensors, used by the CPU tests).
"""
from __future__ import annotations

import os

import torch


def env():
    """(world_size, rank, local_rank) from the torchrun environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def seed_offset(rank: int) -> int:
    """Seed shift that gives every rank its own synthetic batch."""
    return 7919 * rank


def token_shard(T: int, rank: int, world: int):
    """(start, count) of rank's contiguous share of T tokens (strong scaling):
    the first T % world ranks take one extra token."""
    base, extra = divmod(T, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The maximum of `value` over all ranks (the slowest rank's time)."""
    if world == 1:
        return float(value)
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---- tensor-parallel all-reduce of y fused with the write ---------------------
#
# Under tensor parallelism every rank of a group ends a block with a partial y
# and holds a replica of the streams H. hc_reduce_write_then_read reads all
# ranks' partials over peer memory and sums them in rank order inside the
# fused write + read, so y never goes through a separate all-reduce. The
# kernel waits on no other rank; the host orders the partials' writes before
# the call and their next overwrite after every rank's call (reduce_step).

class PeerPartials:
    """Every rank's partial-y buffer, mapped into this process.

    `local` is this rank's [T, d] partial buffer (kept and rewritten in place
    every layer). The ranks exchange CUDA IPC handles over `group` (any
    torch.distributed backend) and open each other's; `pointers` lists the R
    device addresses in rank order, this rank's own buffer at its index.
    export / open_ / close default to the library's hc_ipc_* calls and are
    parameters so the exchange can be exercised without GPUs."""

    def __init__(self, local, group=None, *, export=None, open_=None, close=None):
        import torch.distributed as dist
        if export is None or open_ is None or close is None:
            from . import _lib as hc
            export = export or hc.ipc_export
            open_ = open_ or hc.ipc_open
            close = close or hc.ipc_close
        self._close = close
        self.local = local
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        handle, offset = export(local)
        gathered = [None] * self.world
        dist.all_gather_object(gathered, (self.rank, bytes(handle), int(offset)), group=group)
        self._bases = []
        self.pointers = []
        try:
            for r, (who, h, off) in enumerate(gathered):
                if who != r:
                    raise RuntimeError(f"rank {r} reported itself as rank {who}")
                if r == self.rank:
                    self.pointers.append(int(local.data_ptr()))
                else:
                    base = int(open_(h))
                    self._bases.append(base)
                    self.pointers.append(base + off)
        except BaseException:
            self.close()  # unmap what was opened before the failure
            raise

    def close(self):
        while self._bases:
            self._close(self._bases.pop())


def reduce_step(peers: PeerPartials, H, A, b, a_next, g_next=None, group=None, *,
                call=None, sync=None, **kw):
    """One fused step on the all-reduced y: waits until every rank's partial
    is written (stream sync + barrier), runs hc_reduce_write_then_read on the
    peers' pointers, then waits until every rank has read them (stream sync +
    barrier) so each may overwrite its partial for the next layer. Returns
    (H', x_next). `call` and `sync` default to the library call and
    torch.cuda.current_stream().synchronize."""
    import torch.distributed as dist
    if call is None:
        from . import _lib as hc
        call = hc.reduce_write_then_read
    if sync is None:
        sync = lambda: torch.cuda.current_stream().synchronize()  # noqa: E731
    sync()
    dist.barrier(group)
    out = call(peers.pointers, H, A, b, a_next, g_next, **kw)
    sync()
    dist.barrier(group)
    return out


def reduce_scatter_step(peers_y: PeerPartials, peers_x: PeerPartials, H_shard, A, b, a_next,
                        g_next=None, group=None, *, call=None, sync=None, **kw):
    """The reduce-scatter form of reduce_step: the streams are sharded by
    token over the group (this rank holds H_shard, token_shard(T, rank, R)),
    peers_y maps the ranks' partials and peers_x the ranks' x_next buffers.
    The call reduces this rank's rows, writes its shard of H' and stores its
    rows of x_next into every rank's x buffer; the second barrier makes all of
    x_next complete on every rank before anyone reads it. Returns H'_shard."""
    import torch.distributed as dist
    if peers_y.rank != peers_x.rank or peers_y.world != peers_x.world:
        raise ValueError("peers_y and peers_x must come from the same group")
    if call is None:
        from . import _lib as hc
        call = hc.reduce_scatter_write_then_read
    if sync is None:
        sync = lambda: torch.cuda.current_stream().synchronize()  # noqa: E731
    # the pointer lists are plain addresses: the group's token count comes
    # from this rank's own partial buffer
    shape = getattr(peers_y.local, "shape", None)
    if shape is not None:
        kw.setdefault("T_total", int(shape[0]))
    sync()
    dist.barrier(group)
    out = call(peers_y.pointers, peers_x.pointers, peers_y.rank, H_shard, A, b, a_next, g_next, **kw)
    sync()
    dist.barrier(group)
    return out
