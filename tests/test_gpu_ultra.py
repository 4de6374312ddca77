"""Ultra-shape parity at the full sizes and in the launch configuration the
benchmark times: routing of every token (decode) or of 512+ sampled tokens
(prefill, every outlier row among them) bit-exact against the oracle, the
grouping checked by its defining properties at full size, 16+ output rows
against the oracle (first and last token tiles, the ragged last tile of the
most loaded expert, outlier rows), and the tensor-core router logits against
the error bound the certified selection relies on."""
import warnings

import numpy as np
import pytest
import torch

from latentmoe_expert_routing_b200 import inputs as I
from oracle import moe_oracle as O
from tests.gpu_common import (check_dispatch_properties, np32, prepared_oracle_rows,
                              ragged_tile_tokens, spread_rows)
from tests.test_gpu_parity import _assert_out

pytestmark = pytest.mark.gpu

DEC = I.CONFIGS["ultra_decode_bf16"]
PRE = I.CONFIGS["ultra_prefill_bf16"]

# the certified router's model of the tensor-core logit error (section on the
# certified router in the library): the router GEMM writes S fp32 partial sums
# over D / S consecutive k each (S = 32 for batches of up to 256 tokens, else 8),
# added in fp64 and rounded to fp32, so
#   |l~ - l| <= (margin * gamma_{D/S} + 2^-23) * ||x|| ||w||,
# gamma_n = n u / (1 - n u), u = 2^-23, margin = 2
MARGIN, U = 2.0, 2.0 ** -23


def _splits(T):
    return 32 if T <= 256 else 8


@pytest.fixture(scope="module")
def ultra():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from latentmoe_expert_routing_b200 import build, layer
    build.build()
    W = layer.weights_for(DEC)            # decode and prefill share the weights
    yield layer, W
    del W
    torch.cuda.empty_cache()


def _routing_oracle(cfg, W, x):
    l = O.router_logits(np32(x), np32(W["w_gate"]))
    return O.route(l, np32(W["gate_bias"]), cfg.k, cfg.rsf)


def _check(cfg, ultra, route_rows, out_rows_fn, nt):
    L, W = ultra
    lay = L.layer_for(cfg, W, out_dtype="fp32")
    x = I.hidden(cfg, "cuda")
    out, idx, w = lay(x)
    counts, offsets, perm, pos = lay.routing(cfg.T)
    lay.sync()
    idx_h, w_h = idx.cpu().numpy(), np32(w)
    exact = lay.router_stats()           # certified router: every selected + band
    assert cfg.T * cfg.k <= exact <= cfg.T * cfg.E
    c_h, o_h, p_h = counts.cpu().numpy(), offsets.cpu().numpy(), perm.cpu().numpy()
    check_dispatch_properties(idx_h, c_h, o_h, p_h, pos.cpu().numpy(), cfg.E)
    _, _, ridx, rw = _routing_oracle(cfg, W, x[route_rows])
    assert np.array_equal(idx_h[route_rows], ridx)
    assert np.array_equal(w_h[route_rows].view(np.int32), rw.view(np.int32))
    _, ragged = ragged_tile_tokens(c_h, o_h, p_h, cfg.k, nt)
    rows = out_rows_fn(ragged)
    assert len(rows) >= 16
    r = prepared_oracle_rows(cfg, W, x, rows)
    assert np.array_equal(idx_h[rows], r["topk_idx"])
    _assert_out(out[rows], r["out"])
    lay.close()
    return c_h


def test_ultra_decode_bf16(ultra):
    counts = _check(DEC, ultra, list(range(DEC.T)),
                    lambda ragged: spread_rows(DEC.T, 16, extra=ragged), nt=16)
    assert counts.sum() == DEC.T * DEC.k


def test_ultra_prefill_bf16(ultra):
    outl = I.outlier_rows(PRE)
    rng = np.random.RandomState(5)
    route = sorted(set(outl) | set(range(32)) | set(range(PRE.T - 32, PRE.T)) |
                   set(rng.choice(PRE.T, 400, replace=False).tolist()))
    assert len(route) >= 512 and set(outl) <= set(route)
    _check(PRE, ultra, route,
           lambda ragged: spread_rows(PRE.T, 18, extra=list(ragged) + outl[:6]), nt=256)


def _logit_error_ratio(lt, x, W, K):
    """max over (t, e) of |l~ - l| / (Delta / margin): the tensor-core logits'
    error against the bound the certified router assumes, without its margin
    (K = the length of one fp32 accumulation)."""
    xs, wg = np32(x).astype(np.float64), np32(W["w_gate"]).astype(np.float64)
    l = O.router_logits(xs, wg).astype(np.float64)
    gamma = K * U / (1 - K * U) + U / MARGIN
    bound = gamma * np.linalg.norm(xs, axis=1)[:, None] * np.linalg.norm(wg, axis=1)[None, :]
    return float(np.max(np.abs(lt.cpu().numpy().astype(np.float64) - l) / bound))


def test_tensor_core_logits_within_the_certified_bound(ultra):
    """The certified router assumes |l~ - l| <= margin * gamma_K ||x|| ||w||; the
    observed error of the tensor-core logits must sit inside the bound even
    without the margin, for the 64 decode tokens (split-K logits) and for 128
    prefill tokens (one K pass per 256-token tile), outlier rows among them."""
    L, W = ultra
    ratios = {}
    for cfg, rows in ((DEC, list(range(DEC.T))),
                      (PRE, I.outlier_rows(PRE)[:64] + list(range(64)))):
        lay = L.layer_for(cfg, W, out_dtype="fp32")
        x = I.hidden(cfg, "cuda")
        lay(x)
        lay.sync()
        ratios[cfg.name] = _logit_error_ratio(lay.router_logits(cfg.T)[rows], x[rows], W,
                                              cfg.D // _splits(cfg.T))
        lay.close()
    # reported in the run's warnings summary, which pytest prints even with -q
    warnings.warn(f"tensor-core logit error / bound without the margin: {ratios}")
    assert all(v <= 1.0 for v in ratios.values()), ratios
