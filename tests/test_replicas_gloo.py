"""World-size-2 gloo tests of the replica plumbing used by bench.py (CPU only)."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, ws, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    from llama_gqa_causal_b200 import replicas
    r, w, local = replicas.init("gloo", timeout_s=60)
    try:
        replicas.barrier(w)
        ms = 10.0 + 5.0 * r          # rank 1 is the slow one
        mx = replicas.max_over_ranks(ms, w)
        thr = replicas.job_throughput(100.0, 4, mx, w)
        q.put((r, w, local, mx, thr))
    finally:
        replicas.shutdown(w)


def test_max_over_ranks_and_job_throughput_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, (rank, ws, local, mx, thr) in enumerate(res):
        assert (rank, ws, local) == (r, 2, r)
        assert mx == 15.0                      # the slowest rank's time
        assert thr == pytest.approx(2 * 100.0 * 4 / 0.015)


def test_single_process_is_identity(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    from llama_gqa_causal_b200 import replicas
    assert replicas.init("gloo") == (0, 1, 0)
    assert replicas.max_over_ranks(3.5, 1) == 3.5
    assert replicas.job_throughput(10.0, 2, 1000.0, 1) == 20.0
