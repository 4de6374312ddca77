"""Ultra-shape parity at the full sizes and in the launch configuration the
benchmark times: routing of every token (decode) or of sampled tokens
(prefill) bit-exact against the oracle, the grouping checked by its defining
properties at full size, and sampled output rows against the oracle."""
import numpy as np
import pytest
import torch

from latentmoe_expert_routing_b200 import inputs as I
from oracle import moe_oracle as O
from tests.gpu_common import check_dispatch_properties, np32, oracle_rows, out_metrics
from tests.test_gpu_parity import _assert_out

pytestmark = pytest.mark.gpu

DEC = I.CONFIGS["ultra_decode_bf16"]
PRE = I.CONFIGS["ultra_prefill_bf16"]


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


def _check(cfg, ultra, sample_route, sample_out):
    L, W = ultra
    lay = L.layer_for(cfg, W, out_dtype="fp32")
    x = I.hidden(cfg, "cuda")
    out, idx, w = lay(x)
    counts, offsets, perm, pos = lay.routing(cfg.T)
    lay.sync()
    idx_h, w_h = idx.cpu().numpy(), np32(w)
    exact = lay.router_stats()           # certified router: every selected + band
    assert cfg.T * cfg.k <= exact <= cfg.T * cfg.E
    check_dispatch_properties(idx_h, counts.cpu().numpy(), offsets.cpu().numpy(),
                              perm.cpu().numpy(), pos.cpu().numpy(), cfg.E)
    rows = sample_route
    _, _, ridx, rw = _routing_oracle(cfg, W, x[rows])
    assert np.array_equal(idx_h[rows], ridx)
    assert np.array_equal(w_h[rows].view(np.int32), rw.view(np.int32))
    r = oracle_rows(cfg, W, x, rows=sample_out)
    _assert_out(out[sample_out], r["out"])
    lay.close()
    return counts.cpu().numpy()


def test_ultra_decode_bf16(ultra):
    counts = _check(DEC, ultra, list(range(DEC.T)), [0, 31, 63])
    assert counts.sum() == DEC.T * DEC.k


def test_ultra_prefill_bf16(ultra):
    outl = I.outlier_rows(PRE)
    rows = sorted(set([0, 1, 4095, 8191] + outl[:4] + list(range(3000, 3024))))
    _check(PRE, ultra, rows, [0, outl[0], 8191])
