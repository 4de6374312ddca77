"""The C-ABI library: it builds, loads and exports every declared entry point,
and host-side validation answers without touching a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", "latentmoe.h")]


def _declared():
    names = set()
    for h in HEADERS:
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


@pytest.fixture(scope="module")
def B():
    from latentmoe_expert_routing_b200 import build
    build.build()
    from latentmoe_expert_routing_b200 import binding
    return binding


def test_every_declared_symbol_is_exported(B):
    names = _declared()
    assert "moe_forward" in names and "moe_init" in names
    for n in names:
        assert hasattr(B.lib, n), n
    bound = {s[0] for s in B.SIGNATURES}
    assert set(names) <= bound, set(names) - bound


def test_status_strings_and_version(B):
    assert B.status_string(0) == "ok"
    assert "unsupported" in B.status_string(B.MOE_ERR_UNSUPPORTED)
    assert B.moe_version() >= 100


def _cfg(B, **kw):
    d = dict(d_model=256, d_latent=64, n_experts=16, top_k=4, d_ff=128,
             d_ff_shared=256, n_group=1, topk_group=1, max_tokens=64,
             routed_scaling_factor=5.0, dtype=B.MOE_FP32,
             expert_fmt=B.MOE_EXPERT_DENSE, out_dtype=B.MOE_FP32)
    d.update(kw)
    return B.moe_config(**d)


def _w(B, ptr=4096):
    return B.moe_weights(*([ptr] * 8), 1, *([None] * 6), 1)


@pytest.mark.parametrize("kw,status", [
    (dict(top_k=17), 1), (dict(d_model=0), 1), (dict(d_latent=60), 1),
    (dict(max_tokens=0), 1), (dict(dtype=7), 1),
    (dict(n_group=3), 1), (dict(topk_group=2), 1), (dict(n_group=16), 1),
    (dict(n_group=0), 1), (dict(n_group=4, top_k=5), 1),
    (dict(n_group=128, topk_group=8, n_experts=256), 2), (dict(n_experts=2048), 2),
    (dict(top_k=80, n_experts=100), 2),
])
def test_init_rejects_bad_config_before_any_launch(B, kw, status):
    h = ctypes.c_void_p()
    cfg = _cfg(B, **kw)
    assert B.lib.moe_init(ctypes.byref(h), ctypes.byref(cfg), ctypes.byref(_w(B)), None) == status
    assert not h.value


def test_init_rejects_null_and_misaligned_weights(B):
    h = ctypes.c_void_p()
    cfg = _cfg(B)
    assert B.lib.moe_init(ctypes.byref(h), ctypes.byref(cfg), ctypes.byref(_w(B, 0)), None) == 1
    assert B.lib.moe_init(ctypes.byref(h), ctypes.byref(cfg), ctypes.byref(_w(B, 4100)), None) == 1
    assert B.lib.moe_init(None, ctypes.byref(cfg), ctypes.byref(_w(B)), None) == 1


def test_calls_on_null_handle(B):
    assert B.lib.moe_forward(None, None, 1, None, None, None, None) == 1
    assert B.lib.moe_forward_host(None, None, 1, None, None, None, None) == 1
    assert B.lib.moe_get_routing(None, None, None, None, None, None) == 1
    import torch
    # NULL handle: drains the stream and reports the no-alloc router's error word
    assert B.lib.moe_sync(None, None) == (0 if torch.cuda.is_available() else B.MOE_ERR_CUDA)
    assert B.lib.moe_get_expert_counts(None, None, None) == 1
    B.lib.moe_destroy(None)


def test_block_entry_points_validate_before_any_launch(B):
    """moe_block_forward and moe_rmsnorm reject bad arguments with
    MOE_ERR_INVALID_ARG before touching the device."""
    assert B.lib.moe_block_forward(None, None, 1, None, 1e-5, None, None, None, None) == 1
    p = ctypes.c_void_p(256)                   # never dereferenced: validation fails first
    for eps in (0.0, -1.0, float("inf"), float("nan")):
        assert B.lib.moe_rmsnorm(p, p, 4, 64, eps, B.MOE_BF16, p, None) == 1
    assert B.lib.moe_rmsnorm(None, p, 4, 64, 1e-5, B.MOE_BF16, p, None) == 1
    assert B.lib.moe_rmsnorm(p, None, 4, 64, 1e-5, B.MOE_BF16, p, None) == 1
    assert B.lib.moe_rmsnorm(p, p, 4, 64, 1e-5, B.MOE_BF16, None, None) == 1
    assert B.lib.moe_rmsnorm(p, p, -1, 64, 1e-5, B.MOE_BF16, p, None) == 1
    assert B.lib.moe_rmsnorm(p, p, 4, 0, 1e-5, B.MOE_BF16, p, None) == 1
    assert B.lib.moe_rmsnorm(p, p, 4, 64, 1e-5, 7, p, None) == 1


def test_init_rejects_mixed_or_partial_expert_sources(B):
    """Dense experts and pre-quantised NVFP4 tensors exclude each other, the
    pre-quantised set must be complete and needs an NVFP4 format, and borrowed
    weights must be device pointers: all answered before any device work."""
    h = ctypes.c_void_p()
    q = [4096] * 6
    nv = _cfg(B, dtype=B.MOE_BF16, expert_fmt=B.MOE_EXPERT_NVFP4_W4A16)
    cases = [
        (nv, B.moe_weights(*([4096] * 8), 1, *q, 1)),                 # both sources
        (nv, B.moe_weights(*([4096] * 6), None, None, 1, *q[:5], None, 1)),   # partial
        (_cfg(B), B.moe_weights(*([4096] * 6), None, None, 1, *q, 1)),  # dense format
        (nv, B.moe_weights(*([4096] * 6), None, None, 1, *q[:5], 4100, 1)),   # misaligned
        (_cfg(B), B.moe_weights(*([4096] * 8), 1, *([None] * 6), 0)),   # borrow of host
        (_cfg(B), B.moe_weights(*([4096] * 6), None, 4096, 1, *([None] * 6), 1)),
    ]
    for cfg, w in cases:
        assert B.lib.moe_init(ctypes.byref(h), ctypes.byref(cfg), ctypes.byref(w), None) == 1
        assert not h.value
