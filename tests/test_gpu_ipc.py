"""The peer path through real CUDA IPC: two processes on cuda:0 (one GPU is
what a call here gets) act as two tensor-parallel ranks. Each exports its
partial y with hc_ipc_export, opens the other's with hc_ipc_open
(dist.PeerPartials over a gloo group), runs the fused all-reduce write in the
one-shot and the reduce-scatter form, compares with the oracle and unmaps
with hc_ipc_close. Barriers are host-side with a short timeout; no kernel
waits on the other process."""
from __future__ import annotations

import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_two_processes_exchange_ipc_handles_and_reduce(tmp_path):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hyper_connections_stream_b200 import build
    build.build()
    world = 2
    init = tmp_path / "init"
    env = dict(os.environ, PYTHONPATH=ROOT, CUDA_VISIBLE_DEVICES=os.environ.get("CUDA_VISIBLE_DEVICES", "0"))
    procs = [subprocess.Popen([sys.executable, os.path.join(ROOT, "tests", "_ipc_rank.py"), str(r),
                               str(world), str(init), str(tmp_path / f"r{r}.json")],
                              env=env, cwd=ROOT, stdout=subprocess.PIPE, stderr=subprocess.STDOUT,
                              start_new_session=True)
             for r in range(world)]
    outs = []
    try:
        for p in procs:
            outs.append(p.communicate(timeout=240)[0].decode(errors="replace"))
    finally:
        for p in procs:
            if p.poll() is None:
                os.killpg(p.pid, 9)
                p.wait()
    for r, p in enumerate(procs):
        res = json.loads((tmp_path / f"r{r}.json").read_text())
        assert p.returncode == 0 and res["ok"], (res.get("error"), outs[r][-2000:])
        assert res["pointers_distinct"]
        assert res["oneshot_H"] and res["oneshot_x"], res
        assert res["logits_H_err"] <= 2e-2 and res["logits_x_err"] <= 2e-2, res
        assert res["scatter_H"] and res["scatter_x"], res
        assert res["device_fault"] == 0 and "close_error" not in res, res
