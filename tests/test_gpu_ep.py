"""Expert parallelism on one GPU: n_ranks layers, each holding E/n_ranks of the
experts, run one after another on the same device (no rank waits on another),
their partial latent combines stacked as an all-gather would, and each rank's
token shard finished (the pages' LatentMoE remark: the exchange is d_latent
wide).  Routing must equal the single layer's bit for bit, the output the
single layer's up to the fp32 combine order, and the oracle's within the bf16
(NVFP4) tolerance."""
import numpy as np
import pytest
import torch

from latentmoe_expert_routing_b200 import inputs as I
from tests.gpu_common import REL_L2_NVFP4, oracle_rows, out_metrics
from tests.test_gpu_parity import _assert_out

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


def _ep_run(L, cfg, W, x, G):
    from latentmoe_expert_routing_b200 import dist as D
    T = x.shape[0]
    lays = [L.layer_for(cfg, W, max_tokens=T, out_dtype="fp32", ep_rank=r, ep_ranks=G)
            for r in range(G)]
    res = [lay.ep_partial(x) for lay in lays]
    parts = torch.stack([zc for zc, _, _ in res])          # what the all-gather delivers
    outs = []
    for r, lay in enumerate(lays):
        t0, ts = D.ep_token_shard(r, G, T)
        outs.append(lay.ep_finish(parts, t0, ts))
    torch.cuda.synchronize()
    for lay in lays:
        lay.sync()
        lay.close()
    return torch.cat(outs), res, parts


@pytest.mark.parametrize("fmt,G,T", [("dense", 2, 64), ("dense", 4, 3), ("dense", 4, 200),
                                     ("dense", 16, 33), ("w4a16", 2, 64), ("w4a4", 4, 600)])
def test_expert_parallel_equals_single_layer(L, fmt, G, T):
    cfg = MID.replace(expert_fmt=fmt)
    W = L.weights_for(cfg)
    x = I.hidden(cfg, "cuda", T=T)
    ref_lay = L.layer_for(cfg, W, max_tokens=T, out_dtype="fp32")
    ref, ridx, rw = ref_lay(x)
    ref_lay.sync()
    out, res, parts = _ep_run(L, cfg, W, x, G)
    for zc, idx, w in res:                     # every rank routes identically
        assert torch.equal(idx, ridx)
        assert torch.equal(w.view(torch.int32), rw.view(torch.int32))
    # each token's slots split over the ranks by expert range: a rank's part is
    # zero exactly for the tokens with no held expert
    per = cfg.E // G
    held = torch.stack([((ridx >= r * per) & (ridx < (r + 1) * per)).any(1) for r in range(G)])
    assert torch.equal(parts.abs().amax(2) > 0, held)
    rel = (torch.linalg.norm(out.double() - ref.double()) / torch.linalg.norm(ref.double())).item()
    assert rel < 2e-3, rel                    # combine order only (zc rounds to bf16 for fc2)
    r = oracle_rows(cfg, W, x)
    if fmt == "dense":
        _assert_out(out, r["out"])
    else:
        assert out_metrics(out, r["out"])[0] <= REL_L2_NVFP4
    ref_lay.close()


def test_expert_parallel_handle_rejects_whole_layer_calls(L):
    from latentmoe_expert_routing_b200 import binding as B
    W = L.weights_for(MID)
    lay = L.layer_for(MID, W, max_tokens=8, ep_rank=1, ep_ranks=2)
    x = I.hidden(MID, "cuda", T=8)
    with pytest.raises(B.MoeError) as e:
        lay(x)
    assert e.value.status == B.MOE_ERR_UNSUPPORTED
    zc, _, _ = lay.ep_partial(x)
    with pytest.raises(B.MoeError):            # parts of the wrong rank count
        lay.ep_finish(torch.stack([zc] * 3), 0, 8)
    lay.close()
