"""NVFP4 on the GPU against the oracle (report section 8.1; NVFP4 format details).

The quantiser's codes, block scales and global scales must equal the oracle's
bit for bit on the same inputs; NVFP4 layers must route bit-exactly and match
the oracle's emulated NVFP4 layer within rel-L2 5e-2."""
import numpy as np
import pytest
import torch

from latentmoe_expert_routing_b200 import inputs as I
from oracle import moe_oracle as O
from tests.gpu_common import (REL_L2_NVFP4, check_dispatch_properties, np32, out_metrics,
                              prepared_oracle_rows, ragged_tile_tokens, spread_rows)
from tests.test_gpu_parity import _assert_routing_exact, _run_full

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from latentmoe_expert_routing_b200 import build
    build.build()
    from latentmoe_expert_routing_b200 import layer
    return layer


def _gpu_quantize(w):
    from latentmoe_expert_routing_b200 import binding as B
    n, rows, K = w.shape
    codes = torch.empty(n, rows, K // 2, dtype=torch.uint8, device="cuda")
    scales = torch.empty(n, rows, (K + 15) // 16, dtype=torch.uint8, device="cuda")
    gs = torch.empty(n, dtype=torch.float32, device="cuda")
    dt = B.MOE_BF16 if w.dtype == torch.bfloat16 else B.MOE_FP32
    B.moe_quantize_nvfp4(w.data_ptr(), dt, n, rows, K, codes.data_ptr(), scales.data_ptr(),
                         gs.data_ptr(), torch.cuda.current_stream().cuda_stream)
    return codes.cpu().numpy(), scales.cpu().numpy(), gs.cpu().numpy()


def test_hardware_conversions_match_format(L):
    """The W4A4 path rounds activations with the hardware E2M1 conversion and
    expands codes and scales with the hardware fp16 conversions; over every
    finite fp32 input, all 256 E2M1 bytes and all E4M3 scale pairs they must
    agree with the encoders written from the format definition (which the
    quantiser test pins to the oracle bit for bit)."""
    from latentmoe_expert_routing_b200 import binding as B
    assert B.moe_selftest_nvfp4_convert(torch.cuda.current_stream().cuda_stream) == 0


@pytest.mark.parametrize("K", [320, 328])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quantizer_bit_exact(L, dtype, K):
    """K = 328 ends every row in a block of 8 elements."""
    g = torch.Generator().manual_seed(3)
    w = (torch.randn(4, 192, K, generator=g) * 0.05)
    w[0, 7, -8:] = 0.0                                   # an all-zero partial block
    w[1, 9, -8:] = torch.tensor([6.0, -3.0, 1.5, 0.5, 0.0, 2.0, -4.0, 1.0]) * 0.01
    w[0, 0, :16] = 0.0                                   # all-zero block
    w[1, 3, :16] = torch.tensor([6.0, 3.0, 2.5, 1.75, 1.25, 0.75, 0.25, -5.0,
                                 -3.5, 0.5, 1.0, 1.5, 2.0, 4.0, -6.0, 0.0]) * 0.01
    w[2] *= 100.0                                        # another global scale
    w[3, 5, 16:32] = 1e-6                                # subnormal block scale region
    w = w.to(dtype).cuda()
    codes, scales, gs = _gpu_quantize(w)
    wn = w.float().cpu().numpy()
    for m in range(4):
        sg = O.nvfp4_global_scale(wn[m])
        q, sb = O.nvfp4_quantize(wn[m], sg)
        assert gs[m].view(np.int32) == np.float32(sg).view(np.int32)
        assert np.array_equal(scales[m], sb)
        assert np.array_equal(codes[m], O.pack_e2m1(q))


@pytest.mark.parametrize("fmt", ["w4a16", "w4a4"])
@pytest.mark.parametrize("T", [3, 64, 200])
def test_tiny_nvfp4_layer(L, fmt, T):
    cfg = I.CONFIGS["tiny_fp32"].replace(dtype="bf16", expert_fmt=fmt)
    lay, g, r = _run_full(L, cfg, T)
    _assert_routing_exact(g, r)
    rel, nmax, raw = out_metrics(g[0], r["out"])
    assert rel <= REL_L2_NVFP4, (rel, nmax)
    if fmt == "w4a16":
        # same weights as the oracle's emulated path: only accumulation order and
        # bf16 activation rounding differ, so the error stays at the bf16 level
        assert rel <= 1e-2, rel


@pytest.mark.parametrize("fmt", ["w4a16", "w4a4"])
@pytest.mark.parametrize("T", [3, 64, 200, 600, 1200])
def test_nvfp4_mid_layer(L, fmt, T):
    """Mid-size NVFP4 layer (several 128-row weight blocks per expert, K of
    256 and 512 = whole 4-slice pipeline steps): T spans the 16-, 64- and
    128-token tiles and ragged tails, and every output row is checked.  For
    W4A4, T = 600 (~150 pairs per expert) runs the one-SM block-scaled FP4
    GEMMs and T = 1200 (~300) the SM-pair ones, whose last token tile of an
    expert leaves the second CTA without valid rows."""
    cfg = I.CONFIGS["tiny_fp32"].replace(dtype="bf16", expert_fmt=fmt, E=16, k=4, D=512,
                                         L=256, F=512, Fs=512)
    lay, g, r = _run_full(L, cfg, T)
    _assert_routing_exact(g, r)
    rel, nmax, raw = out_metrics(g[0], r["out"])
    assert rel <= REL_L2_NVFP4, (rel, nmax)
    if fmt == "w4a16":
        assert rel <= 1e-2, rel


@pytest.mark.parametrize("fmt", ["w4a16", "w4a4"])
@pytest.mark.parametrize("T", [3, 64, 200, 600])
def test_nvfp4_ragged_expert_width(L, fmt, T):
    """Expert width F = 328: not a multiple of 16, so each down-projection row
    ends in an NVFP4 block of 8 (and W4A4's ReLU^2 activations too), the last
    128-row block of the up projection holds 72 rows, and the down
    projection's records end in a partial slice followed by zero slices."""
    cfg = I.CONFIGS["tiny_fp32"].replace(dtype="bf16", expert_fmt=fmt, E=16, k=4, D=512,
                                         L=256, F=328, Fs=328)
    lay, g, r = _run_full(L, cfg, T)
    _assert_routing_exact(g, r)
    rel, nmax, raw = out_metrics(g[0], r["out"])
    assert rel <= REL_L2_NVFP4, (rel, nmax)
    if fmt == "w4a16":
        assert rel <= 1e-2, rel


@pytest.mark.parametrize("T", [3, 64, 600, 1200])
def test_w4a4_latent_tensor_scale(L, T):
    """W4A4 with the latent's own per-tensor global scale (amax(z) / 2688,
    computed on the device every forward): the fp16-operand path (16- and
    64-token tiles), the block-scaled FP4 GEMMs on one SM (~150 pairs per
    expert) and on SM pairs (~300), against the oracle's tensor-scale layer."""
    cfg = I.CONFIGS["tiny_fp32"].replace(dtype="bf16", expert_fmt="w4a4", E=16, k=4, D=512,
                                         L=256, F=512, Fs=512, act_scale="tensor")
    lay, g, r = _run_full(L, cfg, T)
    _assert_routing_exact(g, r)
    rel, nmax, raw = out_metrics(g[0], r["out"])
    assert rel <= REL_L2_NVFP4, (rel, nmax)


@pytest.fixture(scope="module")
def ultra_bf16_weights(L):
    W = L.weights_for(I.CONFIGS["ultra_decode_bf16"])
    yield W
    del W
    torch.cuda.empty_cache()


def _ultra_check(L, W, cfg, route_rows, out_rows_fn, nt):
    lay = L.layer_for(cfg, W, out_dtype="fp32")
    x = I.hidden(cfg, "cuda")
    out, idx, w = lay(x)
    counts, offsets, perm, pos = lay.routing(cfg.T)
    lay.sync()
    idx_h = idx.cpu().numpy()
    c_h, o_h, p_h = counts.cpu().numpy(), offsets.cpu().numpy(), perm.cpu().numpy()
    check_dispatch_properties(idx_h, c_h, o_h, p_h, pos.cpu().numpy(), cfg.E)
    l = O.router_logits(np32(x[route_rows]), np32(W["w_gate"]))
    _, _, ridx, rw = O.route(l, np32(W["gate_bias"]), cfg.k, cfg.rsf)
    assert np.array_equal(idx_h[route_rows], ridx)
    assert np.array_equal(np32(w)[route_rows].view(np.int32), rw.view(np.int32))
    _, ragged = ragged_tile_tokens(c_h, o_h, p_h, cfg.k, nt)
    rows = out_rows_fn(ragged)
    assert len(rows) >= 16
    r = prepared_oracle_rows(cfg, W, x, rows)
    rel, nmax, raw = out_metrics(out[rows], r["out"])
    assert rel <= REL_L2_NVFP4, (rel, nmax)
    if cfg.expert_fmt == "w4a16":          # the oracle's own weights: bf16-level error
        assert rel <= 1e-2, rel
    lay.close()
    return c_h


def test_ultra_decode_w4a16(L, ultra_bf16_weights):
    cfg = I.CONFIGS["ultra_decode_w4a16"]
    _ultra_check(L, ultra_bf16_weights, cfg, list(range(cfg.T)),
                 lambda ragged: spread_rows(cfg.T, 16, extra=ragged), nt=16)


def test_skewed_prefill_w4a4(L, ultra_bf16_weights):
    cfg = I.CONFIGS["skewed_prefill_w4a4"]
    W = dict(ultra_bf16_weights)
    W["gate_bias"] = I.gate_bias(cfg, "cuda")          # Zipf profile
    rng = np.random.RandomState(6)
    route = sorted(set(range(64)) | set(range(cfg.T - 64, cfg.T)) |
                   set(rng.choice(cfg.T, 400, replace=False).tolist()))
    assert len(route) >= 512
    counts = _ultra_check(L, W, cfg, route,
                          lambda ragged: spread_rows(cfg.T, 16, extra=ragged), nt=256)
    assert O.max_violation(counts) > 20
