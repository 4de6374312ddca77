"""moe_route_noalloc: the router for callers that cannot allocate device memory.

Some callers may not call cudaMalloc or let a library call it (a serving loop
that owns a fixed HBM budget, a framework whose allocator must account for every
byte, a latency path that cannot take cudaMalloc's implicit synchronisation).
For them the library's router runs with its scratch in a fixed device array.
These checks call it through the C ABI and compare its routing with what the
existing moe_forward entry point returns for the same tokens, on two calls in a
row (the array keeps the previous call's contents), plus its size limit.
This file is collected last on purpose."""
import ctypes

import pytest
import torch

from latentmoe_expert_routing_b200 import inputs as I

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mods():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from latentmoe_expert_routing_b200 import build
    build.build()
    from latentmoe_expert_routing_b200 import binding, layer
    return binding, layer


def _noalloc(B, x, W, cfg, T):
    idx = torch.full((T, cfg.k), -1, dtype=torch.int32, device="cuda")
    w = torch.full((T, cfg.k), -1.0, dtype=torch.float32, device="cuda")
    B.moe_route_noalloc(x.data_ptr(), W["w_gate"].data_ptr(), W["gate_bias"].data_ptr(),
                        T, cfg.D, cfg.E, cfg.k, cfg.rsf, B.DTYPE[cfg.dtype],
                        idx.data_ptr(), w.data_ptr(), torch.cuda.current_stream().cuda_stream)
    return idx, w


@pytest.mark.parametrize("name,T", [("tiny_fp32", 64), ("tiny_fp32", 37),
                                     ("tiny_bf16", 129)])
def test_noalloc_router_matches_forward(mods, name, T):
    B, LY = mods
    cfg = I.CONFIGS["tiny_fp32"]
    if name == "tiny_bf16":
        cfg = cfg.replace(dtype="bf16", T=T)
    W = LY.weights_for(cfg, "cuda")
    lay = LY.layer_for(cfg, W, max_tokens=T, out_dtype="fp32")
    x = I.hidden(cfg, "cuda", T=T)
    _, ref_idx, ref_w = lay(x)
    torch.cuda.synchronize()
    for _ in range(2):                      # two calls in a row share the array
        idx, w = _noalloc(B, x, W, cfg, T)
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx)
        assert torch.equal(w.view(torch.int32), ref_w.view(torch.int32))
    lay.close()


def test_noalloc_router_ultra_decode_rows(mods):
    B, LY = mods
    cfg = I.CONFIGS["ultra_decode_bf16"].replace(E=64)   # 64 experts keep the test small
    W = LY.weights_for(cfg, "cuda")
    lay = LY.layer_for(cfg, W, out_dtype="fp32")
    x = I.hidden(cfg, "cuda")
    _, ref_idx, ref_w = lay(x)
    torch.cuda.synchronize()
    for _ in range(2):
        idx, w = _noalloc(B, x, W, cfg, cfg.T)
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx)
        assert torch.equal(w.view(torch.int32), ref_w.view(torch.int32))
    lay.close()


def test_noalloc_rejects_more_tokens_than_the_scratch_holds(mods):
    B, _ = mods
    lib = B.lib
    # 3812 tokens fit at E=512, k=22; 3813 do not (checked before any launch)
    dummy = torch.zeros(16, dtype=torch.float32, device="cuda")
    p = dummy.data_ptr()
    st = lib.moe_route_noalloc(p, p, p, 3813, 8192, 512, 22, ctypes.c_float(5.0),
                               B.MOE_BF16, p, p, None)
    assert st == B.MOE_ERR_INVALID_ARG
    assert lib.moe_route_noalloc(p, p, p, 4, 8192, 512, 600, ctypes.c_float(5.0),
                                 B.MOE_BF16, p, p, None) == B.MOE_ERR_INVALID_ARG


def test_noalloc_reports_device_errors_through_moe_sync(mods):
    """The no-alloc router cannot own an error flag in caller memory, so the
    problems its kernels see are kept in the fixed array's error word:
    moe_sync(NULL, stream) drains the stream and reports, then clears, it."""
    B, LY = mods
    cfg = I.CONFIGS["tiny_fp32"]
    W = LY.weights_for(cfg, "cuda")
    st = torch.cuda.current_stream().cuda_stream
    x = I.hidden(cfg, "cuda")
    _noalloc(B, x, W, cfg, cfg.T)
    assert B.lib.moe_sync(None, st) == B.MOE_OK            # a clean call
    # NaN rows give NaN logits
    xn = x.clone()
    xn[3] = float("nan")
    _noalloc(B, xn, W, cfg, cfg.T)
    assert B.lib.moe_sync(None, st) == B.MOE_ERR_DEVICE_CHECK
    assert B.lib.moe_sync(None, st) == B.MOE_OK            # read and cleared
    # only k - 1 experts have a choice score above -inf: the last slot of
    # every token cannot be filled
    bias = W["gate_bias"].clone()
    bias[cfg.k - 1:] = float("-inf")
    idx, w = _noalloc(B, x, dict(W, gate_bias=bias), cfg, cfg.T)
    assert B.lib.moe_sync(None, st) == B.MOE_ERR_DEVICE_CHECK
    assert torch.all(idx[:, cfg.k - 1] == 0x7FFFFFFF)
    assert torch.all((idx[:, :cfg.k - 1] >= 0) & (idx[:, :cfg.k - 1] < cfg.k - 1))
    # the array works on after the errors
    idx, w = _noalloc(B, x, W, cfg, cfg.T)
    assert B.lib.moe_sync(None, st) == B.MOE_OK
    _, ref_idx, ref_w = LY.layer_for(cfg, W, out_dtype="fp32")(x)
    torch.cuda.synchronize()
    assert torch.equal(idx, ref_idx)
