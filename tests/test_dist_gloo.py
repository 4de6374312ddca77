"""Multi-rank plumbing on CPU: gloo ranks agree on the slowest rank's time
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


def _ep_worker(rank, world, port, q, T=37):
    """One expert-parallel rank on the CPU: the compute of each step is the
    oracle's arithmetic on this rank's experts; the exchange, the shard split
    and the rank-order sum are the library's multi-rank code."""
    import numpy as np
    import torch
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from latentmoe_expert_routing_b200 import dist as D
    from latentmoe_expert_routing_b200 import inputs as I
    from oracle import moe_oracle as O
    cfg = I.CONFIGS["tiny_fp32"].replace(T=T)
    x = I.hidden(cfg).numpy()
    W = {n: f(cfg).numpy() for n, f in (("g", I.w_gate), ("b", I.gate_bias), ("fc1", I.w_fc1),
                                        ("fc2", I.w_fc2), ("su", I.w_shared_up),
                                        ("sd", I.w_shared_down))}
    e0, e1 = D.ep_expert_range(rank, world, cfg.E)
    up = I.w_up(cfg, range(e0, e1)).numpy().astype(np.float64)
    dn = I.w_down(cfg, range(e0, e1)).numpy().astype(np.float64)

    class RankLayer:
        def ep_partial(self, xt):
            xs = xt.numpy().astype(np.float64)
            l = O.router_logits(xs, W["g"])
            _, _, idx, w = O.route(l, W["b"], cfg.k, cfg.rsf)
            z = xs @ W["fc1"].astype(np.float64).T
            zc = np.zeros_like(z)
            for t in range(xs.shape[0]):
                for j in range(cfg.k):
                    e = int(idx[t, j])
                    if e0 <= e < e1:
                        y = dn[e - e0] @ O.relu2(up[e - e0] @ z[t])
                        zc[t] += float(w[t, j]) * y
            self.xs = xs
            return torch.from_numpy(zc), torch.from_numpy(idx), torch.from_numpy(w)

        def ep_finish(self, parts, t0, ts):
            zc = parts[0].clone()
            for g in range(1, parts.shape[0]):
                zc += parts[g]
            xs = self.xs[t0:t0 + ts]
            sh = O.relu2(xs @ W["su"].astype(np.float64).T) @ W["sd"].astype(np.float64).T
            return torch.from_numpy(zc[t0:t0 + ts].numpy() @ W["fc2"].astype(np.float64).T + sh)

    D.init("gloo", timeout_s=60)
    t0, out, idx, w = D.ep_forward(RankLayer(), torch.from_numpy(x), rank, world)
    q.put((rank, t0, out.numpy(), idx.numpy()))
    D.finish()


@pytest.mark.parametrize("world,T,starts", [
    (2, 37, [0, 19]),                 # shards 0..18 and 19..36
    (4, 37, [0, 10, 19, 28]),         # 10, 9, 9, 9 rows
    (4, 3, [0, 1, 2, 3]),             # fewer rows than ranks: the last shard is empty
])
def test_expert_parallel_exchange_on_gloo_ranks(world, T, starts):
    """CPU ranks each hold E / world of the experts: gathered in rank order and
    finished on token shards, the outputs equal the whole oracle layer's."""
    import numpy as np
    from latentmoe_expert_routing_b200 import inputs as I
    from oracle import moe_oracle as O
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_ep_worker, args=(r, world, port, q, T)) for r in range(world)]
    for p in ps:
        p.start()
    res = sorted([q.get(timeout=120) for _ in range(world)], key=lambda r: r[0])
    for p in ps:
        p.join(120)
        assert p.exitcode == 0
    assert [r[1] for r in res] == starts
    out = np.concatenate([r[2] for r in res])
    assert out.shape[0] == T
    for r in res[1:]:
        assert np.array_equal(res[0][3], r[3])      # every rank routed alike
    cfg = I.CONFIGS["tiny_fp32"].replace(T=T)
    f = lambda g: g(cfg).numpy()
    ref = O.forward(I.hidden(cfg).numpy(), f(I.w_gate), f(I.gate_bias), f(I.w_fc1), f(I.w_fc2),
                    f(I.w_shared_up), f(I.w_shared_down),
                    lambda e: I.w_up(cfg, [e])[0].numpy().astype(np.float64),
                    lambda e: I.w_down(cfg, [e])[0].numpy().astype(np.float64),
                    k=cfg.k, rsf=cfg.rsf)
    assert np.array_equal(res[0][3], ref["topk_idx"])
    assert np.allclose(out, ref["out"], rtol=1e-9, atol=1e-9 * np.abs(ref["out"]).max())
