"""Helpers shared by the GPU parity tests: layer set-up, oracle runs, metrics."""
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
                     topk_group=cfg.topk_group)


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
