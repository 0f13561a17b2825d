"""One rank of the two-process CUDA IPC test (tests/test_gpu_ipc.py).

Both ranks run on cuda:0 as separate processes, the way two tensor-parallel
ranks of one node share memory, except that here the "peer" allocation lives
on the same GPU. The ranks exchange real CUDA IPC handles (hc_ipc_export /
hc_ipc_open through dist.PeerPartials) over a gloo group, run the fused
all-reduce write in both forms (dist.reduce_step, dist.reduce_scatter_step),
and compare with the oracle. Waits are host-side only (gloo barriers with a
short timeout); the kernels read the peer's buffer with the loads the library
chooses for memory of this GPU and wait on nothing.

    python tests/_ipc_rank.py RANK WORLD INIT_FILE OUT_JSON
"""
from __future__ import annotations

import datetime
import json
import os
import sys
import traceback

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

EPS = 1e-6


def main(rank: int, world: int, init_file: str, out_json: str) -> int:
    import numpy as np
    import torch
    import torch.distributed as dist

    import hc_inputs as gen
    import oracle
    from hyper_connections_stream_b200 import _lib as hc
    from hyper_connections_stream_b200 import dist as hd

    result = {"rank": rank, "ok": False}
    dist.init_process_group("gloo", init_method=f"file://{init_file}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    peers = []
    try:
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        hc.lib()
        dt = "bf16"
        T, n, d = 96, 4, 2048

        def up(a):
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

        def down(t):
            return t.cpu().view(torch.int16).numpy().view(np.uint16)

        # every rank draws every partial on the host (same seeds), keeps its own on the GPU
        parts = [gen.to_storage(gen.normal(6100 + r, (T, d)), dt) for r in range(world)]
        H = gen.to_storage(gen.normal(6150, (T, n, d)), dt)
        A = (np.eye(n, dtype=np.float32) + gen.normal(6151, (T, n, n), std=0.05)).astype(np.float32)
        a = gen.normal(6152, (T, n), mean=1.0 / n, std=0.05)
        b = gen.normal(6153, (T, n), mean=1.0, std=0.05)
        g = gen.uniform(6154, (d,), 0.5, 1.5)
        L = gen.normal(6155, (T, n, n))
        rl = gen.normal(6156, (T, n))
        f32 = lambda v: torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).to(dev)  # noqa: E731

        y_local = up(parts[rank])
        py = hd.PeerPartials(y_local)
        peers.append(py)
        result["pointers_distinct"] = len(set(py.pointers)) == world

        # one-shot form, matrix and weights given: bit-exact
        Hp, x = hd.reduce_step(py, up(H), f32(A), f32(b), f32(a), f32(g), eps=EPS)
        Hr, xr, _ = oracle.reduce_write_then_read(parts, H, A, b, a, g, EPS, dt)
        result["oneshot_H"] = bool(np.array_equal(down(Hp), Hr))
        result["oneshot_x"] = bool(np.array_equal(down(x), xr))

        # one-shot form with Sinkhorn and softmax logits: within the bf16 bar
        Hp, x = hd.reduce_step(py, up(H), f32(L), f32(b), f32(rl), f32(g), eps=EPS,
                               mix=hc.MIX_SINKHORN_LOGITS, K=20, read=hc.READ_SOFTMAX_LOGITS)
        Hr, xr, _ = oracle.reduce_write_then_read(parts, H, L, b, rl, g, EPS, dt, K=20,
                                                  mix_logits=True, read_logits=True)

        def rel(got, ref):
            o = (ref.astype(np.uint32) << 16).view(np.float32).astype(np.float64).reshape(T, -1)
            v = (got.astype(np.uint32) << 16).view(np.float32).astype(np.float64).reshape(T, -1)
            rms = np.sqrt(np.mean(o * o, axis=1, keepdims=True))
            return float(np.max(np.abs(v - o) / np.maximum(np.abs(o), rms)))
        result["logits_H_err"] = rel(down(Hp), Hr)
        result["logits_x_err"] = rel(down(x), xr)

        # reduce-scatter form: this rank's shard of H', x_next pushed into both ranks' buffers
        x_local = torch.full((T, d), float("nan"), dtype=torch.bfloat16, device=dev)
        px = hd.PeerPartials(x_local)
        peers.append(px)
        t0, Tr = hd.token_shard(T, rank, world)
        sl = slice(t0, t0 + Tr)
        Hs = hd.reduce_scatter_step(py, px, up(H[sl]), f32(A[sl]), f32(b[sl]), f32(a[sl]), f32(g),
                                    eps=EPS)
        Hr, xr, _ = oracle.reduce_write_then_read(parts, H, A, b, a, g, EPS, dt)
        result["scatter_H"] = bool(np.array_equal(down(Hs), Hr[sl]))
        result["scatter_x"] = bool(np.array_equal(down(x_local), xr))
        result["device_fault"] = hc.device_fault()
        result["ok"] = True
    except BaseException:
        result["error"] = traceback.format_exc()[-3000:]
    finally:
        try:
            torch.cuda.synchronize()
            dist.barrier()  # nobody unmaps while the other may still read
        except BaseException:
            pass
        for p in peers:
            try:
                p.close()
            except BaseException:
                result["close_error"] = traceback.format_exc()[-1000:]
        dist.destroy_process_group()
        with open(out_json, "w") as f:
            json.dump(result, f)
    return 0 if result["ok"] else 1


if __name__ == "__main__":
    sys.exit(main(int(sys.argv[1]), int(sys.argv[2]), sys.argv[3], sys.argv[4]))
