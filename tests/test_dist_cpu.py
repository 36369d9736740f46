"""The multi-process plumbing of bench.py on CPU: two gloo ranks, max-over-ranks timing and
the whole-job rate (replicas: every rank runs the same workload, no data-path collective)."""
from __future__ import annotations

import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [10.0 + rank, 20.0 - rank]  # rank 1 is slower on the first timer, faster on the second
        ms, ms2 = bench.max_over_ranks(local)
        rate = bench.whole_job_rate(17.367264e-3, 100, world, ms)
        q.put((rank, ms, ms2, rate))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_count_all_units():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, ms2, rate in res:
        assert ms == 11.0 and ms2 == 20.0
        assert abs(rate - 2 * 17.367264e-3 * 100 / 0.011) < 1e-9


def test_single_process_is_identity_and_config_matches_both_arms():
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    c1 = bench.workload_config("block_2b4t_decode_t1", 1, True)
    assert c1["packed_bytes_per_step"] == 17_367_264 and c1["T"] == 1
    packed, ops, tensors = bench.workload_units("ffn_32b_t4096")
    assert set(tensors) == {"gate", "up", "down"} and ops == 2 * 4096 * 3 * 27648 * 5120
