"""Thin ctypes binding of include/latentmoe.h (argument marshalling only).

Every function keeps the C name; `LatentMoE` wraps a handle for torch tensors
(device memory and the current stream come from torch, all compute runs in
liblatentmoe.so).  Importing this module loads the library and fails loudly when
it is missing: there is no other implementation of the layer behind it.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("LMOE_LIBRARY", os.path.join(PKG, "liblatentmoe.so"))

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_OOM = 0, 1, 2, 3
MOE_ERR_CUDA, MOE_ERR_TIMEOUT, MOE_ERR_DEVICE_CHECK = 4, 5, 6
MOE_FP32, MOE_BF16 = 0, 1
MOE_EXPERT_DENSE, MOE_EXPERT_NVFP4_W4A16, MOE_EXPERT_NVFP4_W4A4 = 0, 1, 2
EXPERT_FMT = {"dense": MOE_EXPERT_DENSE, "w4a16": MOE_EXPERT_NVFP4_W4A16,
              "w4a4": MOE_EXPERT_NVFP4_W4A4}
DTYPE = {"fp32": MOE_FP32, "bf16": MOE_BF16}
MOE_ACT_SCALE_UNIT, MOE_ACT_SCALE_TENSOR = 0, 1
ACT_SCALE = {"unit": MOE_ACT_SCALE_UNIT, "tensor": MOE_ACT_SCALE_TENSOR}


class moe_config(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int), ("d_latent", ctypes.c_int),
                ("n_experts", ctypes.c_int), ("top_k", ctypes.c_int),
                ("d_ff", ctypes.c_int), ("d_ff_shared", ctypes.c_int),
                ("n_group", ctypes.c_int), ("topk_group", ctypes.c_int),
                ("max_tokens", ctypes.c_int),
                ("routed_scaling_factor", ctypes.c_float),
                ("dtype", ctypes.c_int), ("expert_fmt", ctypes.c_int),
                ("out_dtype", ctypes.c_int), ("act_scale", ctypes.c_int)]


class moe_weights(ctypes.Structure):
    _fields_ = [("w_gate", ctypes.c_void_p), ("gate_bias", ctypes.c_void_p),
                ("w_fc1", ctypes.c_void_p), ("w_fc2", ctypes.c_void_p),
                ("w_shared_up", ctypes.c_void_p), ("w_shared_down", ctypes.c_void_p),
                ("w_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p),
                ("borrow", ctypes.c_int),
                ("up_codes", ctypes.c_void_p), ("up_scales", ctypes.c_void_p),
                ("up_gscale", ctypes.c_void_p), ("down_codes", ctypes.c_void_p),
                ("down_scales", ctypes.c_void_p), ("down_gscale", ctypes.c_void_p),
                ("weights_on_device", ctypes.c_int)]


class MoeError(RuntimeError):
    def __init__(self, status, what):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


_vp, _i, _p = ctypes.c_void_p, ctypes.c_int, ctypes.POINTER
# (name, restype, argtypes) of every entry point declared in include/latentmoe.h
SIGNATURES = [
    ("moe_init", _i, [_p(_vp), _p(moe_config), _p(moe_weights), _vp]),
    ("moe_init_ep", _i, [_p(_vp), _p(moe_config), _p(moe_weights), _i, _i, _vp]),
    ("moe_forward_ep_partial", _i, [_vp, _vp, _i, _vp, _vp, _vp, _vp]),
    ("moe_forward_ep_finish", _i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp]),
    ("moe_forward", _i, [_vp, _vp, _i, _vp, _vp, _vp, _vp]),
    ("moe_forward_host", _i, [_vp, _vp, _i, _vp, _vp, _vp, _vp]),
    ("moe_block_forward", _i, [_vp, _vp, _i, _vp, ctypes.c_float, _vp, _vp, _vp, _vp]),
    ("moe_rmsnorm", _i, [_vp, _vp, _i, _i, ctypes.c_float, _i, _vp, _vp]),
    ("moe_get_routing", _i, [_vp, _vp, _vp, _vp, _vp, _vp]),
    ("moe_get_expert_counts", _i, [_vp, _vp, _vp]),
    ("moe_get_router_logits", _i, [_vp, _vp, _vp]),
    ("moe_profile_enable", _i, [_vp, _i]),
    ("moe_profile_read", _i, [_vp, _p(ctypes.c_float), _i]),
    ("moe_route_noalloc", _i, [_vp, _vp, _vp, _i, _i, _i, _i, ctypes.c_float, _i,
                               _vp, _vp, _vp]),
    ("moe_quantize_nvfp4", _i, [_vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp]),
    ("moe_get_router_stats", _i, [_vp, _p(ctypes.c_ulonglong), _vp]),
    ("moe_selftest_wait_timeout", _i, [_vp, _i, _vp]),
    ("moe_selftest_nvfp4_convert", _i, [_vp, _vp]),
    ("moe_sync", _i, [_vp, _vp]),
    ("moe_destroy", None, [_vp]),
    ("moe_status_string", ctypes.c_char_p, [_i]),
    ("moe_version", _i, []),
]


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m latentmoe_expert_routing_b200.build`")
    lib = ctypes.CDLL(path)
    for name, res, args in SIGNATURES:
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = load_library()
lib = _lib


def status_string(s: int) -> str:
    return _lib.moe_status_string(int(s)).decode()


def _check(status, what):
    if status != MOE_OK:
        raise MoeError(status, what)


def moe_init(cfg: moe_config, w: moe_weights, stream: int):
    h = ctypes.c_void_p()
    _check(_lib.moe_init(ctypes.byref(h), ctypes.byref(cfg), ctypes.byref(w),
                         stream), "moe_init")
    return h


def moe_init_ep(cfg: moe_config, w: moe_weights, rank: int, n_ranks: int, stream: int):
    h = ctypes.c_void_p()
    _check(_lib.moe_init_ep(ctypes.byref(h), ctypes.byref(cfg), ctypes.byref(w), rank, n_ranks,
                            stream), "moe_init_ep")
    return h


def moe_forward_ep_partial(h, hidden_ptr, T, zc_part_ptr, topk_idx_ptr, topk_w_ptr, stream):
    _check(_lib.moe_forward_ep_partial(h, hidden_ptr, T, zc_part_ptr, topk_idx_ptr, topk_w_ptr,
                                       stream), "moe_forward_ep_partial")


def moe_forward_ep_finish(h, parts_ptr, n_parts, T, t0, Ts, out_ptr, stream):
    _check(_lib.moe_forward_ep_finish(h, parts_ptr, n_parts, T, t0, Ts, out_ptr, stream),
           "moe_forward_ep_finish")


def moe_forward(h, hidden_ptr, T, out_ptr, topk_idx_ptr, topk_w_ptr, stream):
    _check(_lib.moe_forward(h, hidden_ptr, T, out_ptr, topk_idx_ptr, topk_w_ptr,
                            stream), "moe_forward")


def moe_block_forward(h, hidden_ptr, T, norm_weight_ptr, eps, out_ptr, topk_idx_ptr, topk_w_ptr,
                      stream):
    _check(_lib.moe_block_forward(h, hidden_ptr, T, norm_weight_ptr, eps, out_ptr, topk_idx_ptr,
                                  topk_w_ptr, stream), "moe_block_forward")


def moe_rmsnorm(x_ptr, norm_weight_ptr, T, D, eps, dtype, y_ptr, stream):
    _check(_lib.moe_rmsnorm(x_ptr, norm_weight_ptr, T, D, eps, dtype, y_ptr, stream),
           "moe_rmsnorm")


def moe_forward_host(h, hidden_ptr, T, out_ptr, topk_idx_ptr, topk_w_ptr, stream):
    _check(_lib.moe_forward_host(h, hidden_ptr, T, out_ptr, topk_idx_ptr,
                                 topk_w_ptr, stream), "moe_forward_host")


def moe_get_routing(h, counts, offsets, perm, pos, stream):
    _check(_lib.moe_get_routing(h, counts, offsets, perm, pos, stream),
           "moe_get_routing")


MOE_NUM_STAGES = 7
STAGES = ["router_logits", "route", "dense_in", "expert_up", "expert_down",
          "combine", "dense_out"]


def moe_get_expert_counts(h, counts, stream):
    _check(_lib.moe_get_expert_counts(h, counts, stream), "moe_get_expert_counts")


def moe_get_router_logits(h, logits, stream):
    _check(_lib.moe_get_router_logits(h, logits, stream), "moe_get_router_logits")


def moe_profile_enable(h, on):
    _check(_lib.moe_profile_enable(h, int(on)), "moe_profile_enable")


def moe_profile_read(h):
    buf = (ctypes.c_float * MOE_NUM_STAGES)()
    _check(_lib.moe_profile_read(h, buf, MOE_NUM_STAGES), "moe_profile_read")
    return dict(zip(STAGES, list(buf)))


def moe_route_noalloc(hidden, w_gate, gate_bias, T, d_model, n_experts, top_k, rsf,
                      dtype, topk_idx, topk_w, stream):
    """Router with no device allocation (scratch in a fixed library array)."""
    _check(_lib.moe_route_noalloc(hidden, w_gate, gate_bias, T, d_model, n_experts,
                                  top_k, rsf, dtype, topk_idx, topk_w, stream),
           "moe_route_noalloc")


def moe_quantize_nvfp4(w, dtype, n_mat, rows, K, codes, scales, gscale, stream):
    _check(_lib.moe_quantize_nvfp4(w, dtype, n_mat, rows, K, codes, scales, gscale, stream),
           "moe_quantize_nvfp4")


def moe_get_router_stats(h, stream) -> int:
    v = ctypes.c_ulonglong(0)
    _check(_lib.moe_get_router_stats(h, ctypes.byref(v), stream), "moe_get_router_stats")
    return v.value


def moe_selftest_nvfp4_convert(stream) -> int:
    v = ctypes.c_ulonglong(0)
    _check(_lib.moe_selftest_nvfp4_convert(ctypes.byref(v), stream), "moe_selftest_nvfp4_convert")
    return v.value


def moe_sync(h, stream):
    _check(_lib.moe_sync(h, stream), "moe_sync")


def moe_destroy(h):
    _lib.moe_destroy(h)


def moe_version() -> int:
    return _lib.moe_version()
