"""The block around the layer on the GPU against the oracle (report
"Nemotron-3-Ultra architecture", layer stack: pre-norm RMSNorm, mixer,
residual add): out = x + layer(RMSNorm(x)).

The normalised rows must equal the oracle's bits (the norm has a defined fp64
order and one rounding to the layer dtype), the routing of them is bit-exact,
and the layer's contribution out - x meets the bf16 tolerances."""
import numpy as np
import pytest
import torch

from latentmoe_expert_routing_b200 import inputs as I
from oracle import moe_oracle as O
from tests.gpu_common import MAX_ABS_BF16, REL_L2_BF16, np32, np64, out_metrics

pytestmark = pytest.mark.gpu

EPS = 1e-5
TINY = I.CONFIGS["tiny_fp32"]
MID = TINY.replace(dtype="bf16", E=16, k=4, D=512, L=256, F=512, Fs=512)


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from latentmoe_expert_routing_b200 import build
    build.build()
    from latentmoe_expert_routing_b200 import layer
    return layer


def _gpu_rmsnorm(x, g, eps):
    from latentmoe_expert_routing_b200 import binding as B
    y = torch.empty_like(x)
    dt = B.MOE_BF16 if x.dtype == torch.bfloat16 else B.MOE_FP32
    B.moe_rmsnorm(x.data_ptr(), g.data_ptr(), x.shape[0], x.shape[1], eps, dt, y.data_ptr(),
                  torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return y


def _oracle_block(cfg, W, x, g, rows=None):
    up, down = W["w_up"], W["w_down"]
    xs = x if rows is None else x[rows]
    return O.block_forward(np32(xs), np32(g), EPS, np32(W["w_gate"]), np32(W["gate_bias"]),
                           np32(W["w_fc1"]), np32(W["w_fc2"]), np32(W["w_shared_up"]),
                           np32(W["w_shared_down"]), lambda e: np64(up[e]),
                           lambda e: np64(down[e]), dtype=cfg.dtype, k=cfg.k, rsf=cfg.rsf,
                           expert_fmt=cfg.expert_fmt, n_group=cfg.n_group,
                           topk_group=cfg.topk_group)


@pytest.mark.parametrize("cfg", [TINY, MID, I.CONFIGS["ultra_decode_bf16"]], ids=["fp32", "bf16", "ultra"])
def test_rmsnorm_bits(L, cfg):
    """The normalised rows are the oracle's, bit for bit (several row counts,
    and one row of zeros)."""
    x = I.hidden(cfg, "cuda", T=37)
    x[5].zero_()
    g = I.norm_weight(cfg, "cuda")
    y = _gpu_rmsnorm(x, g, EPS)
    yo = O.rmsnorm_spec(np32(x), np32(g), EPS)
    want = O.round_fp64_to_bf16(yo) if cfg.dtype == "bf16" else yo.astype(np.float32)
    assert np.array_equal(np32(y).view(np.int32), want.view(np.int32))


@pytest.mark.parametrize("cfg,T", [(TINY, 64), (TINY, 3), (MID, 1), (MID, 200)],
                         ids=["fp32-64", "fp32-3", "bf16-1", "bf16-200"])
def test_block_parity(L, cfg, T):
    W = L.weights_for(cfg)
    lay = L.layer_for(cfg, W, max_tokens=T, out_dtype="fp32")
    x = I.hidden(cfg, "cuda", T=T)
    g = I.norm_weight(cfg, "cuda")
    out, idx, w = lay.block(x, g, EPS)
    lay.sync()
    r = _oracle_block(cfg, W, x, g)
    assert np.array_equal(idx.cpu().numpy(), r["topk_idx"])
    assert np.array_equal(np32(w).view(np.int32), r["topk_w"].view(np.int32))
    rel, nmax, raw = out_metrics(out.double() - x.double(), r["layer_out"])
    assert rel <= REL_L2_BF16 and nmax <= MAX_ABS_BF16, (rel, nmax, raw)
    rel, nmax, raw = out_metrics(out, r["out"])
    assert rel <= REL_L2_BF16 and nmax <= MAX_ABS_BF16, (rel, nmax, raw)
    lay.close()


def test_block_ultra_decode(L):
    """Ultra decode shape: routing of every row exact, the layer's contribution
    checked on sampled rows."""
    cfg = I.CONFIGS["ultra_decode_bf16"]
    W = L.weights_for(cfg)
    lay = L.layer_for(cfg, W, out_dtype="fp32")
    x = I.hidden(cfg, "cuda")
    g = I.norm_weight(cfg, "cuda")
    out, idx, w = lay.block(x, g, EPS)
    lay.sync()
    y = O.round_fp64_to_bf16(O.rmsnorm_spec(np32(x), np32(g), EPS))
    l = O.router_logits(y, np32(W["w_gate"]))
    _, _, ridx, rw = O.route(l, np32(W["gate_bias"]), cfg.k, cfg.rsf)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert np.array_equal(np32(w).view(np.int32), rw.view(np.int32))
    rows = [0, 17, 63]
    r = _oracle_block(cfg, W, x, g, rows=rows)
    rel, nmax, raw = out_metrics((out.double() - x.double())[rows], r["layer_out"])
    assert rel <= REL_L2_BF16 and nmax <= MAX_ABS_BF16, (rel, nmax, raw)
    lay.close()
    del W
    torch.cuda.empty_cache()


def test_block_rejects_bad_arguments(L):
    from latentmoe_expert_routing_b200 import binding as B
    cfg = TINY
    W = L.weights_for(cfg)
    lay = L.layer_for(cfg, W, max_tokens=8, out_dtype="fp32")
    x = I.hidden(cfg, "cuda", T=8)
    g = I.norm_weight(cfg, "cuda")
    for eps in (0.0, -1.0, float("inf"), float("nan")):
        with pytest.raises(B.MoeError):
            lay.block(x, g, eps)
    lay.sync()
    lay.close()
