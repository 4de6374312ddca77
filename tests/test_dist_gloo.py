"""Multi-rank plumbing on CPU: two gloo ranks agree on the slowest rank's time
and the whole-job throughput (the bench's N>1 path, without GPUs)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from latentmoe_expert_routing_b200 import dist as D
    assert D.env_ranks() == (rank, world, rank)
    D.init("gloo", timeout_s=60)
    D.barrier()
    my_ms = [3.0, 5.0][rank]
    ms_max = D.max_over_ranks(my_ms)
    q.put((rank, ms_max, D.job_throughput(64, world, ms_max * 1e-3)))
    D.finish()


def test_two_gloo_ranks_agree_on_max_time_and_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms_max, tput in res:
        assert ms_max == 5.0
        assert abs(tput - 2 * 64 / 5e-3) < 1e-6


def test_single_rank_needs_no_process_group():
    from latentmoe_expert_routing_b200 import dist as D
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        os.environ.pop(k, None)
    assert D.init("gloo") == 1
    assert D.max_over_ranks(2.5) == 2.5
    assert D.job_throughput(64, 1, 0.002) == 32000.0
