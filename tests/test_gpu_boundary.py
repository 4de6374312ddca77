"""The C ABI's weight sources (report section 8.1; zhichai.net "NVFP4 format
details"): NVFP4 experts handed over pre-quantised, as a checkpoint ships them,
must give the same layer bit for bit as quantising dense experts at moe_init;
weights in host memory must give the same layer as weights on the device; and
moe_get_expert_counts returns the grouping's counts."""
import numpy as np
import pytest
import torch

from latentmoe_expert_routing_b200 import inputs as I
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu

MID = I.CONFIGS["tiny_fp32"].replace(dtype="bf16", E=16, k=4, D=512, L=256, F=512, Fs=512)


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from latentmoe_expert_routing_b200 import build
    build.build()
    from latentmoe_expert_routing_b200 import layer
    return layer


def _prequantised(w):
    """The oracle's NVFP4 quantisation of dense experts [E, rows, K], in the
    ABI's plain layout: codes [E, rows, K/2], scales [E, rows, ceil(K/16)],
    gscale [E]."""
    w = w.float().cpu().numpy()
    codes, scales, gs = [], [], []
    for m in w:
        sg = O.nvfp4_global_scale(m)
        q, sb = O.nvfp4_quantize(m, sg)
        codes.append(O.pack_e2m1(q))
        scales.append(sb)
        gs.append(sg)
    return (torch.from_numpy(np.stack(codes)), torch.from_numpy(np.stack(scales)),
            torch.from_numpy(np.array(gs, dtype=np.float32)))


def _run(L, cfg, W, T):
    lay = L.layer_for(cfg, W, max_tokens=T, out_dtype="fp32")
    x = I.hidden(cfg, "cuda", T=T)
    out, idx, w = lay(x)
    lay.sync()
    res = (out.clone(), idx.clone(), w.clone())
    lay.close()
    return res


def _same(a, b):
    for u, v in zip(a, b):
        assert torch.equal(u.view(torch.int32), v.view(torch.int32))


@pytest.mark.parametrize("fmt,T,F", [("w4a16", 3, 512), ("w4a16", 200, 512), ("w4a4", 64, 512),
                                     ("w4a4", 600, 512), ("w4a4", 1200, 512),
                                     ("w4a16", 64, 328), ("w4a4", 600, 328)])
def test_prequantised_nvfp4_equals_quantise_at_init(L, fmt, T, F):
    """F = 328 ends each down-projection row in a block of 8: its scales are
    [E, L, ceil(F/16)]."""
    cfg = MID.replace(expert_fmt=fmt, F=F)
    W = L.weights_for(cfg)
    ref = _run(L, cfg, W, T)
    uc, us, ug = _prequantised(W["w_up"])
    dc, ds, dg = _prequantised(W["w_down"])
    Wq = {n: t for n, t in W.items() if n not in ("w_up", "w_down")}
    Wq.update(up_codes=uc.cuda(), up_scales=us.cuda(), up_gscale=ug.cuda(),
              down_codes=dc.cuda(), down_scales=ds.cuda(), down_gscale=dg.cuda())
    _same(_run(L, cfg, Wq, T), ref)
    # the same tensors from host memory
    Wh = {n: t.cpu() for n, t in Wq.items()}
    _same(_run(L, cfg, Wh, T), ref)


@pytest.mark.parametrize("cfg", [I.CONFIGS["tiny_fp32"], MID, MID.replace(expert_fmt="w4a16")])
def test_host_weights_equal_device_weights(L, cfg):
    W = L.weights_for(cfg)
    ref = _run(L, cfg, W, 64)
    _same(_run(L, cfg, {n: t.cpu() for n, t in W.items()}, 64), ref)


def test_expert_counts(L):
    from latentmoe_expert_routing_b200 import binding as B
    W = L.weights_for(MID)
    lay = L.layer_for(MID, W, max_tokens=100, out_dtype="fp32")
    _, idx, _ = lay(I.hidden(MID, "cuda", T=100))
    counts = torch.full((MID.E,), -1, dtype=torch.int32, device="cuda")
    B.moe_get_expert_counts(lay.handle, counts.data_ptr(), lay.stream)
    lay.sync()
    ref = torch.bincount(idx.reshape(-1).long(), minlength=MID.E).int()
    assert torch.equal(counts, ref)
    assert torch.equal(counts, lay.routing(100)[0])
    lay.close()
