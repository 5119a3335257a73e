"""World-size-2 gloo tests of the multi-rank host logic (CPU only).

The decode path shards by sequence with no data exchange; the multi-GPU
benchmark's only collectives are a barrier and a max-reduction of the timed
region.  These tests run that logic on two CPU processes, including a rank
that fails before the collective (the peer must end with an error, not hang).
"""
from __future__ import annotations

import os
import socket

import pytest
import torch.multiprocessing as mp

from long_context_decode_nosa_b200 import multirank


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q, mode):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    info = multirank.rank_info()
    try:
        multirank.init(info, backend="gloo", timeout_s=10)
        if mode == "fail" and rank == 1:
            raise RuntimeError("rank 1 fails before the collective")
        multirank.barrier(info)
        elapsed = [3.0, 5.0][rank]
        m = multirank.max_over_ranks(elapsed, info)
        rate = multirank.aggregate_rate(8 * 100, info, m)
        q.put((rank, "ok", m, rate, multirank.rank_seed(7, info)))
        multirank.shutdown(info)
    except Exception as e:  # noqa: BLE001 -- reported to the parent
        q.put((rank, "error", type(e).__name__, str(e)[:200], None))


def _run(mode):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q, mode)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=90)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    out = {}
    while not q.empty():
        r = q.get()
        out[r[0]] = r
    return out, alive


def test_two_ranks_max_time_and_aggregate():
    out, alive = _run("ok")
    assert not alive
    assert out[0][1] == "ok" and out[1][1] == "ok"
    assert out[0][2] == out[1][2] == 5.0                 # max over ranks
    assert out[0][3] == pytest.approx(2 * 800 / 5.0)     # all ranks' units / slowest time
    assert out[0][4] != out[1][4]                        # distinct inputs per rank


def test_failed_rank_ends_peer_with_error_not_hang():
    out, alive = _run("fail")
    assert not alive, "a rank hung waiting for a failed peer"
    assert out[1][1] == "error"
    assert out[0][1] == "error"          # the barrier / collective ended with an error


def test_single_rank_is_a_no_op(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    info = multirank.rank_info()
    assert info.world == 1
    multirank.init(info)
    multirank.barrier(info)
    assert multirank.max_over_ranks(2.5, info) == 2.5
    assert multirank.aggregate_rate(100, info, 2.0) == 50.0
