"""Device-side failure reporting without a GPU fault: a bounded device wait on
a flag that nothing sets gives up, the error word carries the timeout to the
host through moe_sync, and the context stays usable for the next forward."""
import numpy as np
import pytest
import torch

from latentmoe_expert_routing_b200 import inputs as I

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mods():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from latentmoe_expert_routing_b200 import binding, build, layer
    build.build()
    return binding, layer


def test_bounded_wait_reports_timeout_and_context_survives(mods):
    B, LY = mods
    cfg = I.CONFIGS["tiny_fp32"].replace(dtype="bf16")
    W = LY.weights_for(cfg)
    lay = LY.layer_for(cfg, W, out_dtype="fp32")
    x = I.hidden(cfg, "cuda")
    out0, idx0, _ = lay(x)
    lay.sync()
    st = torch.cuda.current_stream().cuda_stream
    assert B.lib.moe_selftest_wait_timeout(lay.handle, 2000, st) == B.MOE_OK
    assert B.lib.moe_sync(lay.handle, st) == B.MOE_ERR_TIMEOUT
    assert B.lib.moe_sync(lay.handle, st) == B.MOE_OK        # the word was cleared
    out1, idx1, _ = lay(x)                                   # the context still works
    lay.sync()
    assert torch.equal(idx0, idx1) and torch.equal(out0, out1)


def test_selftest_rejects_bad_arguments(mods):
    B, LY = mods
    assert B.lib.moe_selftest_wait_timeout(None, 10, None) == B.MOE_ERR_INVALID_ARG
