"""Multi-rank path on CPU: two gloo ranks run the bench's sharding and timing
helpers. Each rank steps its own batch of tokens through the oracle; the
shards, concatenated, must equal one oracle call over all tokens (the step
has no cross-token coupling, so sharding needs no collective), and the timing
reduction must return the slowest rank's value."""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_inputs(rank, T, n, d):
    import hc_inputs as gen
    from hyper_connections_stream_b200 import dist as hd
    off = hd.seed_offset(rank)
    H = gen.to_storage(gen.normal(gen.SEED_H + off, (T, n, d)), "bf16")
    y = gen.to_storage(gen.normal(gen.SEED_Y + off, (T, d)), "bf16")
    L = gen.normal(gen.SEED_L + off, (T, n, n))
    rl = gen.normal(gen.SEED_L + 100 + off, (T, n))
    return H, y, L, rl


def _worker(rank, world, port, T, n, d, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import oracle
    from hyper_connections_stream_b200 import dist as hd
    oracle.set_threads(1)
    ws, r, _ = hd.env()
    assert (ws, r) == (world, rank)
    H, y, L, rl = _rank_inputs(rank, T, n, d)
    b = np.ones(n, np.float32)
    hd.barrier(ws)
    H2, x2 = oracle.write_then_read(H, y, L, b, rl, None, 1e-6, "bf16", K=20,
                                    mix_logits=True, read_logits=True)
    slowest = hd.max_over_ranks(float(rank + 1) * 0.25, ws)
    outs = [torch.zeros(T * n * d, dtype=torch.int32) for _ in range(ws)]
    dist.all_gather(outs, torch.from_numpy(H2.astype(np.int32).reshape(-1)))
    xs = [torch.zeros(T * d, dtype=torch.int32) for _ in range(ws)]
    dist.all_gather(xs, torch.from_numpy(x2.astype(np.int32).reshape(-1)))
    if rank == 0:
        np.save(os.path.join(out_dir, "H.npy"), torch.cat(outs).numpy())
        np.save(os.path.join(out_dir, "x.npy"), torch.cat(xs).numpy())
        np.save(os.path.join(out_dir, "slowest.npy"), np.array([slowest]))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_shard_tokens_without_a_collective(tmp_path):
    world, T, n, d = 2, 6, 4, 64
    mp.spawn(_worker, args=(world, _free_port(), T, n, d, str(tmp_path)), nprocs=world, join=True)
    import oracle
    parts = [_rank_inputs(r, T, n, d) for r in range(world)]
    H = np.concatenate([p[0] for p in parts])
    y = np.concatenate([p[1] for p in parts])
    L = np.concatenate([p[2] for p in parts])
    rl = np.concatenate([p[3] for p in parts])
    H2, x2 = oracle.write_then_read(H, y, L, np.ones(n, np.float32), rl, None, 1e-6, "bf16",
                                    K=20, mix_logits=True, read_logits=True)
    got_H = np.load(tmp_path / "H.npy").astype(np.uint16).reshape(world * T, n, d)
    got_x = np.load(tmp_path / "x.npy").astype(np.uint16).reshape(world * T, d)
    assert np.array_equal(got_H, H2) and np.array_equal(got_x, x2)
    assert float(np.load(tmp_path / "slowest.npy")[0]) == 0.5


def test_token_shard_partitions_exactly():
    from hyper_connections_stream_b200 import dist as hd
    for T in (0, 1, 7, 16384, 16387):
        for world in (1, 2, 3, 8):
            spans = [hd.token_shard(T, r, world) for r in range(world)]
            assert sum(c for _, c in spans) == T
            pos = 0
            for start, count in spans:
                assert start == pos
                pos += count
            assert max(c for _, c in spans) - min(c for _, c in spans) <= 1


class _FakeLocal:
    """Stands in for a rank's partial-y tensor: only its address is used."""

    def __init__(self, addr):
        self.addr = addr

    def data_ptr(self):
        return self.addr


def _peer_worker(rank, world, port, T, n, d, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import hc_inputs as gen
    import oracle
    from hyper_connections_stream_b200 import dist as hd
    oracle.set_threads(1)
    opened, closed, events = [], [], []
    # fake IPC: a handle names its exporter; an exporter's allocation starts
    # 16 * rank bytes before its partial; a peer's allocation maps at 1e6 * (r + 1)
    local = _FakeLocal(1000 * (rank + 1))

    def export(t):
        return f"rank{rank}".encode().ljust(64, b"\0"), 16 * rank

    def open_(h):
        r = int(h.rstrip(b"\0").decode()[4:])
        opened.append(r)
        return 10 ** 6 * (r + 1)

    peers = hd.PeerPartials(local, export=export, open_=open_, close=closed.append)
    want = [1000 * (rank + 1) if r == rank else 10 ** 6 * (r + 1) + 16 * r for r in range(world)]
    assert peers.pointers == want, (peers.pointers, want)
    assert sorted(opened) == [r for r in range(world) if r != rank]

    # every rank's partial, reachable "through its address" (the data moves
    # with gloo here, standing in for the peer loads of the GPU kernel)
    part = gen.to_storage(gen.normal(2600 + rank, (T, d)), "bf16")
    parts = [None] * world
    dist.all_gather_object(parts, part)
    by_addr = {want_r: parts[r] for r, want_r in enumerate(peers.pointers)}
    H = gen.to_storage(gen.normal(2700, (T, n, d)), "bf16")   # replicated stream state
    L = gen.normal(2701, (T, n, n))
    b = gen.normal(2702, (n,), mean=1.0, std=0.02)
    l = gen.normal(2703, (T, n))

    def call(ptrs, H_, A_, b_, a_, g_, **kw):
        events.append("call")
        Hp, x, _ = oracle.reduce_write_then_read([by_addr[p] for p in ptrs], H_, A_, b_, a_, g_,
                                                 1e-6, "bf16", K=20, mix_logits=True,
                                                 read_logits=True)
        return Hp, x

    Hp, x = hd.reduce_step(peers, H, L, b, l, None, call=call, sync=lambda: events.append("sync"))
    assert events == ["sync", "call", "sync"], events

    # the reduce-scatter form: x buffers mapped like the partials; the call
    # gets both pointer lists and this rank's shard
    xpeers = hd.PeerPartials(_FakeLocal(5000 + rank), export=export, open_=open_,
                             close=closed.append)
    t0, Tr = hd.token_shard(T, rank, world)
    seen = []

    def rs_call(yp, xp, r, H_, A_, b_, a_, g_, **kw):
        seen.append((list(yp), list(xp), r, H_.shape[0]))
        return H_

    hd.reduce_scatter_step(peers, xpeers, H[t0:t0 + Tr], L[t0:t0 + Tr], b, l[t0:t0 + Tr], None,
                           call=rs_call, sync=lambda: events.append("sync"))
    assert seen == [(peers.pointers, xpeers.pointers, rank, Tr)], seen
    assert xpeers.pointers[rank] == 5000 + rank
    xpeers.close()
    peers.close()
    assert sorted(closed) == sorted(2 * [10 ** 6 * (r + 1) for r in range(world) if r != rank])
    outs = [None] * world
    dist.all_gather_object(outs, (Hp, x))
    if rank == 0:
        np.save(os.path.join(out_dir, "Hp.npy"), np.stack([o[0] for o in outs]))
        np.save(os.path.join(out_dir, "x.npy"), np.stack([o[1] for o in outs]))
    dist.barrier()
    dist.destroy_process_group()


def test_peer_partials_and_reduce_step_on_gloo_ranks(tmp_path):
    """Three gloo ranks exchange (fake) IPC handles: each gets every rank's
    partial address in rank order (its own unopened, the others opened and
    offset), runs the step between two synchronisations, and closes what it
    opened. Every rank's H' and x_next equal the single-process oracle on all
    partials, so the replicas stay identical."""
    import hc_inputs as gen
    import oracle
    world, T, n, d = 3, 5, 4, 64
    mp.spawn(_peer_worker, args=(world, _free_port(), T, n, d, str(tmp_path)), nprocs=world,
             join=True)
    parts = [gen.to_storage(gen.normal(2600 + r, (T, d)), "bf16") for r in range(world)]
    H = gen.to_storage(gen.normal(2700, (T, n, d)), "bf16")
    L = gen.normal(2701, (T, n, n))
    b = gen.normal(2702, (n,), mean=1.0, std=0.02)
    l = gen.normal(2703, (T, n))
    Hp, x, _ = oracle.reduce_write_then_read(parts, H, L, b, l, None, 1e-6, "bf16", K=20,
                                             mix_logits=True, read_logits=True)
    got_H = np.load(tmp_path / "Hp.npy")
    got_x = np.load(tmp_path / "x.npy")
    for r in range(world):
        assert np.array_equal(got_H[r], Hp) and np.array_equal(got_x[r], x)


def _peer_fail_worker(rank, world, port):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    from hyper_connections_stream_b200 import dist as hd
    closed = []

    def open_(h):
        r = int(h.rstrip(b"\0").decode()[4:])
        if r == world - 1 and rank == 0:
            raise OSError("peer mapping refused")
        return 10 ** 6 * (r + 1)

    export = lambda t: (f"rank{rank}".encode().ljust(64, b"\0"), 0)  # noqa: E731
    if rank == 0:
        try:
            hd.PeerPartials(_FakeLocal(64), export=export, open_=open_, close=closed.append)
        except OSError:
            pass
        else:
            raise AssertionError("the refused mapping did not propagate")
        # the peer opened before the failure (rank 1) is unmapped again
        assert closed == [10 ** 6 * 2], closed
    else:
        peers = hd.PeerPartials(_FakeLocal(64), export=export, open_=open_, close=closed.append)
        peers.close()
    dist.barrier()
    dist.destroy_process_group()


def test_peer_partials_unmaps_on_a_failed_open():
    mp.spawn(_peer_fail_worker, args=(3, _free_port()), nprocs=3, join=True)
