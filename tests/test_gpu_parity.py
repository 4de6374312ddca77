"""CUDA path vs the CPU oracle, element by element (run on a B200).

Routing indices, weights, counts, offsets and the permutation must match bit for
bit; the layer output within rel-L2 1e-2 and max-abs 2e-2 (rows normalised by
the oracle's row RMS; parity runs write fp32 output)."""
import numpy as np
import pytest
import torch

from latentmoe_expert_routing_b200 import inputs as I
from oracle import moe_oracle as O
from tests.gpu_common import (MAX_ABS_BF16, REL_L2_BF16, check_dispatch_properties,
                              np32, oracle_rows, out_metrics)

pytestmark = pytest.mark.gpu

TINY = I.CONFIGS["tiny_fp32"]


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from latentmoe_expert_routing_b200 import build
    build.build()
    from latentmoe_expert_routing_b200 import layer
    return layer


def _run_full(L, cfg, T=None, W=None):
    T = cfg.T if T is None else T
    W = W or L.weights_for(cfg)
    lay = L.layer_for(cfg, W, max_tokens=max(T, 1), out_dtype="fp32")
    x = I.hidden(cfg, "cuda", T=T)
    out, idx, w = lay(x)
    counts, offsets, perm, pos = lay.routing(T)
    lay.sync()
    r = oracle_rows(cfg, W, x)
    return lay, (out, idx, w, counts, offsets, perm, pos), r


def _assert_routing_exact(g, r):
    out, idx, w, counts, offsets, perm, pos = g
    assert np.array_equal(idx.cpu().numpy(), r["topk_idx"])
    assert np.array_equal(np32(w).view(np.int32), r["topk_w"].view(np.int32))
    assert np.array_equal(counts.cpu().numpy(), r["counts"])
    assert np.array_equal(offsets.cpu().numpy(), r["offsets"])
    assert np.array_equal(perm.cpu().numpy(), r["perm"])
    assert np.array_equal(pos.cpu().numpy(), r["pos"].reshape(-1))


def _assert_out(gout, ref, rel_tol=REL_L2_BF16, abs_tol=MAX_ABS_BF16):
    rel, nmax, raw = out_metrics(gout, ref)
    assert rel <= rel_tol and nmax <= abs_tol, (rel, nmax, raw)


@pytest.mark.parametrize("T", [64, 1, 3, 33, 65, 129])
def test_tiny_fp32_full_parity(L, T):
    lay, g, r = _run_full(L, TINY, T)
    _assert_routing_exact(g, r)
    _assert_out(g[0], r["out"])


@pytest.mark.parametrize("k", [1, 16])
def test_tiny_degenerate_k(L, k):
    lay, g, r = _run_full(L, TINY.replace(k=k))
    _assert_routing_exact(g, r)
    _assert_out(g[0], r["out"])


def test_tiny_bf16_zero_bias(L):
    cfg = TINY.replace(dtype="bf16", bias_kind="zero")
    lay, g, r = _run_full(L, cfg)
    _assert_routing_exact(g, r)
    _assert_out(g[0], r["out"])


def test_tiny_skewed_bias_load(L):
    cfg = TINY.replace(dtype="bf16", bias_kind="zipf", E=64, T=256)
    lay, g, r = _run_full(L, cfg)
    _assert_routing_exact(g, r)
    _assert_out(g[0], r["out"])


def test_zero_tokens_is_a_no_op(L):
    W = L.weights_for(TINY)
    lay = L.layer_for(TINY, W, max_tokens=8, out_dtype="fp32")
    x = torch.empty(0, TINY.D, device="cuda")
    out, idx, w = lay(x)
    lay.sync()
    assert out.shape == (0, TINY.D)


def test_too_many_tokens_rejected(L):
    from latentmoe_expert_routing_b200 import binding as B
    W = L.weights_for(TINY)
    lay = L.layer_for(TINY, W, max_tokens=8, out_dtype="fp32")
    with pytest.raises(B.MoeError) as ei:
        lay(I.hidden(TINY, "cuda", T=9))
    assert ei.value.status == B.MOE_ERR_INVALID_ARG


def test_generator_identical_on_gpu_and_cpu(L):
    cfg = I.CONFIGS["ultra_prefill_bf16"]
    for name, fn in [("x", lambda d: I.hidden(cfg, d, T=40, start_row=100)),
                     ("fc1", lambda d: I.normal_tensor(0, 4, (300000,), 0.01, "bf16", d)),
                     ("up7", lambda d: I.normal_tensor(0, 8, (4096,), 0.02, "bf16", d,
                                                       start=7 * 5120 * 2048))]:
        assert torch.equal(fn("cuda").cpu(), fn("cpu")), name


def test_host_entry_point_matches_device_entry_point(L):
    W = L.weights_for(TINY)
    lay = L.layer_for(TINY, W, out_dtype="fp32")
    x = I.hidden(TINY, "cuda")
    out, idx, w = lay(x)
    torch.cuda.synchronize()
    xh = x.cpu().pin_memory()
    oh = torch.empty(TINY.T, TINY.D, dtype=torch.float32).pin_memory()
    ih = torch.empty(TINY.T, TINY.k, dtype=torch.int32).pin_memory()
    lay.forward_host(xh, oh, ih)
    assert torch.equal(oh, out.cpu()) and torch.equal(ih, idx.cpu())


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_host_entry_point_repeated_calls(L, dtype):
    """Repeated host calls with one T replay a captured graph of the forward;
    every call, with new inputs and a change of T in between, must equal the
    device entry point on the same inputs."""
    cfg = TINY.replace(dtype=dtype, T=129)
    W = L.weights_for(cfg)
    lay = L.layer_for(cfg, W, out_dtype="fp32")
    for i, T in enumerate([129, 129, 129, 64, 64, 129, 129]):
        x = I.hidden(cfg.replace(seed=i), "cuda", T=T)
        out, idx, w = lay(x)
        torch.cuda.synchronize()
        xh = x.cpu().pin_memory()
        oh = torch.empty(T, cfg.D, dtype=torch.float32).pin_memory()
        ih = torch.empty(T, cfg.k, dtype=torch.int32).pin_memory()
        lay.forward_host(xh, oh, ih)
        assert torch.equal(oh, out.cpu()) and torch.equal(ih, idx.cpu()), (i, T)


@pytest.mark.parametrize("T", [1, 3, 64, 129, 300])
def test_tiny_bf16_tensor_core_path(L, T):
    """bf16 layers run on the tcgen05 GEMMs; T spans 16-, 64- and 256-row
    token tiles and ragged tails."""
    cfg = TINY.replace(dtype="bf16")
    lay, g, r = _run_full(L, cfg, T)
    _assert_routing_exact(g, r)
    _assert_out(g[0], r["out"])


def test_bf16_wide_tiles_and_many_experts(L):
    cfg = TINY.replace(dtype="bf16", E=64, k=8, D=512, L=128, F=256, Fs=384, T=700)
    lay, g, r = _run_full(L, cfg)
    _assert_routing_exact(g, r)
    _assert_out(g[0], r["out"])


@pytest.mark.parametrize("bias_kind,T", [("normal", 1200), ("zipf", 1200), ("normal", 64),
                                         ("normal", 200), ("zipf", 256)])
def test_bf16_sm_pair_tiles(L, bias_kind, T):
    """256-token tiles whose weight matrices have rows in multiples of 256 run
    on SM pairs (two-CTA MMA): grouped up/down and the dense fc1, shared-up and
    fc2 GEMMs here.  Zipf bias gives experts with many full tiles and experts
    with a handful of tokens (ragged tiles down to one 16-row MMA step).
    T = 200 and 256 (one token tile) run the dense GEMMs on SM pairs with a
    K split (fp32 partials, fixed-order reduce); T = 64 runs fc1 and the
    shared up projection as one launch (rows split between two weights and
    two outputs)."""
    cfg = TINY.replace(dtype="bf16", E=16, k=4, D=512, L=256, F=512, Fs=512, T=T,
                       bias_kind=bias_kind)
    lay, g, r = _run_full(L, cfg)
    _assert_routing_exact(g, r)
    _assert_out(g[0], r["out"])


@pytest.mark.parametrize("dtype,E,k,n_group,topk_group,T", [
    ("fp32", 16, 4, 4, 2, 64),       # exact-logit router
    ("bf16", 16, 4, 4, 2, 129),      # certified router, tensor-core GEMMs
    ("bf16", 64, 8, 8, 3, 300),
    ("bf16", 64, 6, 32, 4, 65),      # groups of two experts
    ("bf16", 32, 4, 4, 4, 33),       # every group kept
])
def test_group_routing(L, dtype, E, k, n_group, topk_group, T):
    """Group routing (section 5.5): only experts of the topk_group groups with
    the largest top-2 sums compete; indices, weights and grouping must equal
    the oracle's bit for bit, the output within tolerance."""
    cfg = TINY.replace(dtype=dtype, E=E, k=k, n_group=n_group, topk_group=topk_group, T=T)
    lay, g, r = _run_full(L, cfg)
    _assert_routing_exact(g, r)
    _assert_out(g[0], r["out"])
    G = E // n_group
    assert all(len(set((row // G).tolist())) <= topk_group for row in g[1].cpu().numpy())


@pytest.mark.parametrize("T", [3, 64, 300])
def test_ragged_expert_and_shared_widths(L, T):
    """Expert and shared intermediate widths that are not multiples of 64 (the
    Super shape's 7688 is one): the expert up / shared up GEMMs end in a partial
    block of output columns, the expert down / fc2 + shared down GEMMs in a
    partial K step.  T spans the 16-, 64- and 256-token tiles."""
    cfg = TINY.replace(dtype="bf16", E=16, k=4, D=256, L=64, F=200, Fs=136)
    lay, g, r = _run_full(L, cfg, T)
    _assert_routing_exact(g, r)
    _assert_out(g[0], r["out"])
