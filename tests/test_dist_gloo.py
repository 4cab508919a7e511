"""The replica timing path with two gloo ranks on the CPU: the max-over-ranks
reduction and the aggregate time per call that bench.py reports for N > 1."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from block_sparse_linear_02_b200 import dist as sdist
    d = sdist.init("gloo", timeout_s=60)
    try:
        assert sdist.env_ranks() == (rank, world, rank)
        per_rank_ms = [3.0, 5.0][rank]
        m = sdist.max_over_ranks(per_rank_ms)
        out[rank] = (m, sdist.aggregate_ms_per_call(m, world))
        d.barrier()
    finally:
        d.destroy_process_group()


def test_two_gloo_ranks_max_and_aggregate():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0] == out[1] == (5.0, 2.5)


def test_single_process_defaults(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    from block_sparse_linear_02_b200 import dist as sdist
    assert sdist.env_ranks() == (0, 1, 0)
    assert sdist.init("gloo") is None
    assert sdist.max_over_ranks(7.5) == 7.5
    assert sdist.aggregate_ms_per_call(8.0, 1) == 8.0
