"""Helpers shared by the GPU parity tests: layer set-up, oracle runs, metrics."""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

from latentmoe_expert_routing_b200 import inputs as I
from oracle import moe_oracle as O

# bf16 tolerances (rel-L2 on the output, max-abs on rows normalised by the
# oracle row RMS); NVFP4 rel-L2 against the oracle's emulated NVFP4 path
REL_L2_BF16, MAX_ABS_BF16, REL_L2_NVFP4 = 1e-2, 2e-2, 5e-2


def np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64) if t.dtype == torch.bfloat16 \
        else t.detach().cpu().numpy().astype(np.float64)


def np32(t):
    return t.detach().float().cpu().numpy()


def oracle_rows(cfg, W, x_rows, rows=None):
    """Run the oracle on token rows (all rows when rows is None); the weights
    are the generator's tensors (copied from wherever they were generated)."""
    up, down = W["w_up"], W["w_down"]

    def get(t, e):             # one expert matrix at a time: Ultra experts are 21 MB
        return np64(t[e])

    x = x_rows if rows is None else x_rows[rows]
    return O.forward(np32(x), np32(W["w_gate"]), np32(W["gate_bias"]), np32(W["w_fc1"]),
                     np32(W["w_fc2"]), np32(W["w_shared_up"]), np32(W["w_shared_down"]),
                     lambda e: get(up, e), lambda e: get(down, e), k=cfg.k, rsf=cfg.rsf,
                     expert_fmt=cfg.expert_fmt, n_group=cfg.n_group,
                     topk_group=cfg.topk_group, act_scale=cfg.act_scale)


def out_metrics(gpu_out, ref):
    """(rel-L2, max-abs on rows normalised by the oracle row RMS, raw max-abs)."""
    g = np64(gpu_out)
    rel = np.linalg.norm(g - ref) / np.linalg.norm(ref)
    rms = np.sqrt(np.mean(ref ** 2, axis=1, keepdims=True))
    nmax = np.max(np.abs(g - ref) / np.maximum(rms, 1e-30))
    return rel, nmax, np.max(np.abs(g - ref))


def check_dispatch_properties(idx, counts, offsets, perm, pos, E):
    """perm / pos / counts / offsets must be the grouping of the GPU's own
    topk_idx by (expert asc, token asc): any size, plain numpy."""
    idx = np.asarray(idx)
    T, k = idx.shape
    flat = idx.reshape(-1).astype(np.int64)
    assert np.array_equal(np.asarray(counts), np.bincount(flat, minlength=E))
    assert offsets[0] == 0 and np.array_equal(np.diff(np.asarray(offsets)), np.asarray(counts))
    order = np.argsort(flat * (T * k) + np.arange(T * k), kind="stable")
    assert np.array_equal(np.asarray(perm), order)
    assert np.array_equal(np.asarray(perm)[np.asarray(pos)], np.arange(T * k))


def prepared_oracle_rows(cfg, W, x_rows, rows):
    """oracle_rows for sampled token rows of a full-size workload.  The oracle
    walks the selected experts in ascending order; their matrices (the oracle's
    own expert_weights_fp64, NVFP4 quantisation included) are made ahead of it
    on host threads, a bounded window at a time."""
    x = np32(x_rows[rows])
    l = O.router_logits(x, np32(W["w_gate"]))
    _, _, idx, _ = O.route(l, np32(W["gate_bias"]), cfg.k, cfg.rsf, cfg.n_group,
                           cfg.topk_group)
    need = sorted(set(idx.reshape(-1).tolist()))
    nw = max(1, min(32, os.cpu_count() or 1))
    jobs = [(name, e) for e in need for name in ("w_up", "w_down")]
    make = lambda j: O.expert_weights_fp64(np32(W[j[0]][j[1]]), cfg.expert_fmt)
    futs, nxt = {}, [0]
    with ThreadPoolExecutor(max_workers=nw) as ex:
        def get(name, e):
            while nxt[0] < len(jobs) and len(futs) < 2 * nw:
                futs[jobs[nxt[0]]] = ex.submit(make, jobs[nxt[0]])
                nxt[0] += 1
            return futs.pop((name, e)).result()
        return O.forward(x, np32(W["w_gate"]), np32(W["gate_bias"]), np32(W["w_fc1"]),
                         np32(W["w_fc2"]), np32(W["w_shared_up"]), np32(W["w_shared_down"]),
                         lambda e: get("w_up", e), lambda e: get("w_down", e), k=cfg.k,
                         rsf=cfg.rsf, expert_fmt=cfg.expert_fmt, n_group=cfg.n_group,
                         topk_group=cfg.topk_group, experts_prepared=True,
                         act_scale=cfg.act_scale)


def ragged_tile_tokens(counts, offsets, perm, k, nt, n=4):
    """Tokens of the last token tile (nt pairs per tile) of the most loaded
    expert: that tile is ragged unless the count is a multiple of nt."""
    counts, offsets, perm = (np.asarray(a) for a in (counts, offsets, perm))
    e = int(np.argmax(counts))
    c = int(counts[e])
    start = int(offsets[e]) + (c - 1) // nt * nt
    pairs = perm[start:int(offsets[e + 1])]
    toks = sorted(set((pairs // k).tolist()))
    return e, toks[:n // 2] + toks[-(n - n // 2):]


def spread_rows(T, n, extra=(), seed=0):
    """n distinct token rows: the first two and last two, `extra`, and evenly
    spread others (sorted)."""
    rows = {0, 1, T - 2, T - 1} | {int(r) for r in extra}
    for r in np.linspace(0, T - 1, n + 2).astype(int):
        if len(rows) >= n:
            break
        rows.add(int(r))
    rng = np.random.RandomState(seed)
    while len(rows) < n:
        rows.add(int(rng.randint(T)))
    return sorted(rows)
