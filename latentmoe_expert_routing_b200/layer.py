"""torch-facing wrapper of one liblatentmoe handle (marshalling only).

    layer = LatentMoE(dims, weights, max_tokens=T, out_dtype="fp32")
    out, topk_idx, topk_w = layer(x)          # x: [T, d_model] on cuda

torch provides the device buffers and the current stream; every step of the
layer runs in the CUDA library.
"""
from __future__ import annotations

import torch

from . import binding as B

_TORCH_DT = {"fp32": torch.float32, "bf16": torch.bfloat16}


_DENSE_NAMES = ("w_gate", "gate_bias", "w_fc1", "w_fc2", "w_shared_up", "w_shared_down")
_EXPERT_NAMES = ("w_up", "w_down")
_NVFP4_NAMES = ("up_codes", "up_scales", "up_gscale", "down_codes", "down_scales",
                "down_gscale")


class LatentMoE:
    """One LatentMoE layer.

    weights: dict with w_gate [E,D], gate_bias [E] fp32, w_fc1 [L,D],
    w_fc2 [D,L], w_shared_up [Fs,D], w_shared_down [D,Fs] and either dense
    experts w_up [E,F,L], w_down [E,L,F] or, for the NVFP4 formats, the
    pre-quantised up_codes [E,F,L/2] / up_scales [E,F,L/16] / up_gscale [E]
    and down_codes [E,L,F/2] / down_scales [E,L,F/16] / down_gscale [E]
    (uint8, uint8, fp32).  All tensors contiguous and on one side: cuda
    tensors are borrowed (the library keeps their pointers), cpu tensors are
    copied by moe_init."""

    def __init__(self, D, L, E, k, F, Fs, weights, *, max_tokens, rsf=5.0,
                 dtype="bf16", expert_fmt="dense", out_dtype=None,
                 n_group=1, topk_group=1, ep_rank=0, ep_ranks=1, act_scale="unit"):
        self.dims = dict(D=D, L=L, E=E, k=k, F=F, Fs=Fs)
        self.dtype = dtype
        self.out_dtype = out_dtype or dtype
        self.max_tokens = max_tokens
        self._w = {n: t.contiguous() for n, t in weights.items()}
        on_dev = {t.is_cuda for t in self._w.values()}
        if len(on_dev) != 1:
            raise ValueError("weights must all be cuda tensors or all cpu tensors")
        on_dev = on_dev.pop()
        cfg = B.moe_config(D, L, E, k, F, Fs, n_group, topk_group, max_tokens,
                           float(rsf), B.DTYPE[dtype], B.EXPERT_FMT[expert_fmt],
                           B.DTYPE[self.out_dtype], B.ACT_SCALE[act_scale])
        ptr = lambda n: self._w[n].data_ptr() if n in self._w else None
        w = B.moe_weights(*(ptr(n) for n in _DENSE_NAMES + _EXPERT_NAMES), int(on_dev),
                          *(ptr(n) for n in _NVFP4_NAMES), int(on_dev))
        self.cfg = cfg
        self.ep = (ep_rank, ep_ranks)
        st = torch.cuda.current_stream().cuda_stream
        self.handle = (B.moe_init(cfg, w, st) if ep_ranks == 1 else
                       B.moe_init_ep(cfg, w, ep_rank, ep_ranks, st))
        if not on_dev:
            self._w = {}                      # copied by moe_init

    @property
    def stream(self) -> int:
        return torch.cuda.current_stream().cuda_stream

    def __call__(self, x, out=None, topk_idx=None, topk_w=None):
        T = x.shape[0]
        D, k = self.dims["D"], self.dims["k"]
        if x.dtype != _TORCH_DT[self.dtype] or not x.is_cuda or x.shape[1] != D:
            raise ValueError("x must be a cuda [T, d_model] tensor in the layer dtype")
        x = x.contiguous()
        if out is None:
            out = torch.empty(T, D, dtype=_TORCH_DT[self.out_dtype], device=x.device)
        if topk_idx is None:
            topk_idx = torch.empty(T, k, dtype=torch.int32, device=x.device)
        if topk_w is None:
            topk_w = torch.empty(T, k, dtype=torch.float32, device=x.device)
        B.moe_forward(self.handle, x.data_ptr(), T, out.data_ptr(),
                      topk_idx.data_ptr(), topk_w.data_ptr(), self.stream)
        return out, topk_idx, topk_w

    def ep_partial(self, x, zc_part=None, topk_idx=None, topk_w=None):
        """Expert parallelism, steps 1-6: (zc_part [T, L] fp32, topk_idx, topk_w)
        with zc_part the slot-ordered combine of the experts this layer holds."""
        T = x.shape[0]
        L, k = self.dims["L"], self.dims["k"]
        if x.dtype != _TORCH_DT[self.dtype] or not x.is_cuda or x.shape[1] != self.dims["D"]:
            raise ValueError("x must be a cuda [T, d_model] tensor in the layer dtype")
        x = x.contiguous()
        if zc_part is None:
            zc_part = torch.empty(T, L, dtype=torch.float32, device=x.device)
        if topk_idx is None:
            topk_idx = torch.empty(T, k, dtype=torch.int32, device=x.device)
        if topk_w is None:
            topk_w = torch.empty(T, k, dtype=torch.float32, device=x.device)
        B.moe_forward_ep_partial(self.handle, x.data_ptr(), T, zc_part.data_ptr(),
                                 topk_idx.data_ptr(), topk_w.data_ptr(), self.stream)
        self._ep_T = T
        return zc_part, topk_idx, topk_w

    def ep_finish(self, parts, t0, Ts, out=None):
        """Expert parallelism, step 7 on token rows [t0, t0 + Ts): parts
        [n_ranks, T, L] fp32 (every rank's zc_part, rank order)."""
        parts = parts.contiguous()
        n, T = parts.shape[0], parts.shape[1]
        if out is None:
            out = torch.empty(Ts, self.dims["D"], dtype=_TORCH_DT[self.out_dtype],
                              device=parts.device)
        B.moe_forward_ep_finish(self.handle, parts.data_ptr(), n, T, t0, Ts,
                                out.data_ptr() if Ts else None, self.stream)
        return out

    def block(self, x, norm_weight, eps=1e-5, out=None, topk_idx=None, topk_w=None):
        """The block around the layer: out = x + layer(RMSNorm(x)); norm_weight [D]
        in the layer dtype (moe_block_forward)."""
        T = x.shape[0]
        D, k = self.dims["D"], self.dims["k"]
        if x.dtype != _TORCH_DT[self.dtype] or not x.is_cuda or x.shape[1] != D:
            raise ValueError("x must be a cuda [T, d_model] tensor in the layer dtype")
        if norm_weight.dtype != x.dtype or not norm_weight.is_cuda or norm_weight.numel() != D:
            raise ValueError("norm_weight must be a cuda [d_model] tensor in the layer dtype")
        x = x.contiguous()
        g = norm_weight.contiguous()
        if out is None:
            out = torch.empty(T, D, dtype=_TORCH_DT[self.out_dtype], device=x.device)
        if topk_idx is None:
            topk_idx = torch.empty(T, k, dtype=torch.int32, device=x.device)
        if topk_w is None:
            topk_w = torch.empty(T, k, dtype=torch.float32, device=x.device)
        B.moe_block_forward(self.handle, x.data_ptr(), T, g.data_ptr(), float(eps),
                            out.data_ptr(), topk_idx.data_ptr(), topk_w.data_ptr(), self.stream)
        return out, topk_idx, topk_w

    def forward_host(self, x_host, out_host, topk_idx_host=None, topk_w_host=None):
        """Host buffers in and out (pinned is fastest); synchronises."""
        B.moe_forward_host(self.handle, x_host.data_ptr(), x_host.shape[0],
                           out_host.data_ptr(),
                           None if topk_idx_host is None else topk_idx_host.data_ptr(),
                           None if topk_w_host is None else topk_w_host.data_ptr(),
                           self.stream)
        return out_host

    def routing(self, T):
        """(counts[E], offsets[E+1], perm[T*k], pos[T*k]) of the last forward."""
        E, k = self.dims["E"], self.dims["k"]
        dev = torch.device("cuda")
        counts = torch.empty(E, dtype=torch.int32, device=dev)
        offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(max(T * k, 1), dtype=torch.int32, device=dev)
        pos = torch.empty(max(T * k, 1), dtype=torch.int32, device=dev)
        B.moe_get_routing(self.handle, counts.data_ptr(), offsets.data_ptr(),
                          perm.data_ptr(), pos.data_ptr(), self.stream)
        return counts, offsets, perm[:T * k], pos[:T * k]

    def router_logits(self, T):
        """[T, E] fp32 router logits of the last forward (tensor-core logits for
        bf16 layers)."""
        lg = torch.empty(T, self.dims["E"], dtype=torch.float32, device="cuda")
        B.moe_get_router_logits(self.handle, lg.data_ptr(), self.stream)
        return lg

    def router_stats(self) -> int:
        """Exactly recomputed (token, expert) logits since the last call."""
        return B.moe_get_router_stats(self.handle, self.stream)

    def sync(self):
        B.moe_sync(self.handle, self.stream)

    def close(self):
        if getattr(self, "handle", None) is not None:
            B.moe_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def weights_for(cfg, device="cuda"):
    """Generate a config's synthetic weights on `device` (inputs module)."""
    from . import inputs as I
    dt = _TORCH_DT[cfg.dtype]
    up = torch.empty(cfg.E, cfg.F, cfg.L, dtype=dt, device=device)
    down = torch.empty(cfg.E, cfg.L, cfg.F, dtype=dt, device=device)
    I.w_up_into(cfg, up)
    I.w_down_into(cfg, down)
    return dict(w_gate=I.w_gate(cfg, device), gate_bias=I.gate_bias(cfg, device),
                w_fc1=I.w_fc1(cfg, device), w_fc2=I.w_fc2(cfg, device),
                w_shared_up=I.w_shared_up(cfg, device),
                w_shared_down=I.w_shared_down(cfg, device), w_up=up, w_down=down)


def layer_for(cfg, weights, max_tokens=None, out_dtype=None, ep_rank=0, ep_ranks=1):
    """A layer for config `cfg`; with ep_ranks > 1 the rank's slice of the
    experts is taken from the full expert tensors in `weights`."""
    if ep_ranks > 1:
        from .dist import ep_expert_range
        e0, e1 = ep_expert_range(ep_rank, ep_ranks, cfg.E)
        weights = dict(weights)
        for n in ("w_up", "w_down", "up_codes", "up_scales", "up_gscale", "down_codes",
                  "down_scales", "down_gscale"):
            if n in weights:
                weights[n] = weights[n][e0:e1]
    return LatentMoE(cfg.D, cfg.L, cfg.E, cfg.k, cfg.F, cfg.Fs, weights,
                     max_tokens=max_tokens or cfg.T, rsf=cfg.rsf, dtype=cfg.dtype,
                     expert_fmt=cfg.expert_fmt, out_dtype=out_dtype,
                     n_group=cfg.n_group, topk_group=cfg.topk_group,
                     ep_rank=ep_rank, ep_ranks=ep_ranks, act_scale=cfg.act_scale)
