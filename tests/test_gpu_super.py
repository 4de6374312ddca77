"""The Super shape of the family (report section 1.2: 128 routed experts, 8 per
token, expert and shared intermediate size 7688 -- not a multiple of the 64-wide
K step, nor of the 16-element NVFP4 block -- latent 2048), at full size, with
bf16 experts and with NVFP4 experts (W4A16 decode, W4A4 prefill): routing of
every decode token and of 512+ prefill tokens bit-exact against the oracle,
16+ output rows of each within the bf16 or the NVFP4 tolerance."""
import numpy as np
import pytest
import torch

from latentmoe_expert_routing_b200 import inputs as I
from oracle import moe_oracle as O
from tests.gpu_common import (REL_L2_NVFP4, check_dispatch_properties, np32, out_metrics,
                              prepared_oracle_rows, ragged_tile_tokens, spread_rows)
from tests.test_gpu_parity import _assert_out

pytestmark = pytest.mark.gpu

DEC = I.CONFIGS["super_decode_bf16"]
PRE = I.CONFIGS["super_prefill_bf16"]
DEC_W4A16 = DEC.replace(name="super_decode_w4a16", expert_fmt="w4a16")
PRE_W4A4 = PRE.replace(name="super_prefill_w4a4", expert_fmt="w4a4")


@pytest.fixture(scope="module")
def sup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from latentmoe_expert_routing_b200 import build, layer
    build.build()
    W = layer.weights_for(DEC)
    yield layer, W
    del W
    torch.cuda.empty_cache()


@pytest.mark.parametrize("cfg,nt", [(DEC, 16), (PRE, 256), (DEC_W4A16, 16), (PRE_W4A4, 128)])
def test_super_shape(sup, cfg, nt):
    L, W = sup
    lay = L.layer_for(cfg, W, out_dtype="fp32")
    x = I.hidden(cfg, "cuda")
    out, idx, w = lay(x)
    counts, offsets, perm, pos = lay.routing(cfg.T)
    lay.sync()
    idx_h, w_h = idx.cpu().numpy(), np32(w)
    c_h, o_h, p_h = counts.cpu().numpy(), offsets.cpu().numpy(), perm.cpu().numpy()
    check_dispatch_properties(idx_h, c_h, o_h, p_h, pos.cpu().numpy(), cfg.E)
    rng = np.random.RandomState(7)
    route = list(range(cfg.T)) if cfg.T <= 512 else sorted(
        set(I.outlier_rows(cfg)) | set(range(32)) | set(range(cfg.T - 32, cfg.T)) |
        set(rng.choice(cfg.T, 420, replace=False).tolist()))
    l = O.router_logits(np32(x[route]), np32(W["w_gate"]))
    _, _, ridx, rw = O.route(l, np32(W["gate_bias"]), cfg.k, cfg.rsf)
    assert np.array_equal(idx_h[route], ridx)
    assert np.array_equal(w_h[route].view(np.int32), rw.view(np.int32))
    _, ragged = ragged_tile_tokens(c_h, o_h, p_h, cfg.k, nt)
    rows = spread_rows(cfg.T, 16, extra=list(ragged) + I.outlier_rows(cfg)[:3])
    r = prepared_oracle_rows(cfg, W, x, rows)
    if cfg.expert_fmt == "dense":
        _assert_out(out[rows], r["out"])
    else:
        rel, nmax, raw = out_metrics(out[rows], r["out"])
        assert rel <= REL_L2_NVFP4, (rel, nmax)
        if cfg.expert_fmt == "w4a16":      # the oracle's own weights: bf16-level error
            assert rel <= 1e-2, rel
    lay.close()
