"""Closed-form pins of the oracle's whole layer (report section 5.6 steps 1-7).

Each case reduces the layer to a formula written here with plain dense algebra
(einsum over all experts, no routing bookkeeping), so a dropped term, a wrong
operand or a mis-ordered normalisation in the oracle fails one of them.
"""
import numpy as np
import pytest

from latentmoe_expert_routing_b200 import inputs as I
from oracle import moe_oracle as O


def _layer(cfg, **over):
    x = I.hidden(cfg).numpy()
    W = dict(w_gate=I.w_gate(cfg).numpy(), bias=I.gate_bias(cfg).numpy(),
             w_fc1=I.w_fc1(cfg).numpy(), w_fc2=I.w_fc2(cfg).numpy(),
             w_su=I.w_shared_up(cfg).numpy(), w_sd=I.w_shared_down(cfg).numpy())
    up = I.w_up(cfg).numpy().astype(np.float64)
    down = I.w_down(cfg).numpy().astype(np.float64)
    W.update(over.pop("W", {}))
    up = over.pop("up", up)
    down = over.pop("down", down)
    r = O.forward(x, W["w_gate"], W["bias"], W["w_fc1"], W["w_fc2"], W["w_su"],
                  W["w_sd"], lambda e: up[e], lambda e: down[e], k=cfg.k,
                  rsf=cfg.rsf, **over)
    return x.astype(np.float64), W, up, down, r


def _shared(x, W):
    h = np.maximum(x @ W["w_su"].astype(np.float64).T, 0) ** 2
    return h @ W["w_sd"].astype(np.float64).T


def _expert_out(z, up, down):
    """y[t, e, :] = down_e relu(up_e z_t)^2 for every expert."""
    h = np.maximum(np.einsum("tl,efl->tef", z, up), 0) ** 2
    return np.einsum("tef,elf->tel", h, down)


TINY = I.CONFIGS["tiny_fp32"]


def test_k_equals_E_is_dense_weighted_sum():
    cfg = TINY.replace(k=TINY.E)
    x, W, up, down, r = _layer(cfg)
    s = r["s"].astype(np.float64)
    z = x @ W["w_fc1"].astype(np.float64).T
    y = _expert_out(z, up, down)
    g = s / s.sum(1, keepdims=True) * cfg.rsf
    ref = np.einsum("te,tel->tl", g, y) @ W["w_fc2"].astype(np.float64).T + _shared(x, W)
    assert np.allclose(r["out"], ref, rtol=1e-6, atol=1e-6 * np.abs(ref).max())
    assert sorted(r["topk_idx"][0].tolist()) == list(range(cfg.E))


def test_k1_is_single_mlp_with_weight_rsf():
    cfg = TINY.replace(k=1)
    x, W, up, down, r = _layer(cfg)
    e = r["topk_idx"][:, 0]
    ref_e = np.argmax(r["s"] + W["bias"], axis=1)
    assert np.array_equal(e, ref_e)
    z = x @ W["w_fc1"].astype(np.float64).T
    y = _expert_out(z, up, down)[np.arange(cfg.T), e]
    ref = 5.0 * y @ W["w_fc2"].astype(np.float64).T + _shared(x, W)
    assert np.allclose(r["out"], ref, rtol=1e-12, atol=1e-12)


def test_zero_experts_and_fc2_leave_only_shared_mlp():
    x, W, up, down, r = _layer(TINY, up=np.zeros((TINY.E, TINY.F, TINY.L)),
                               down=np.zeros((TINY.E, TINY.L, TINY.F)),
                               W={"w_fc2": np.zeros((TINY.D, TINY.L), np.float32)})
    assert np.array_equal(r["out"], _shared(x, W))


def test_routed_part_uses_latent_and_shared_uses_input():
    # with zero shared weights the output lies in the span of fc2's columns
    x, W, up, down, r = _layer(TINY, W={"w_sd": np.zeros((TINY.D, TINY.Fs), np.float32)})
    fc2 = W["w_fc2"].astype(np.float64)
    coef, *_ = np.linalg.lstsq(fc2, r["out"].T, rcond=None)
    assert np.allclose(fc2 @ coef, r["out"].T, atol=1e-9 * np.abs(r["out"]).max())
    z = x @ W["w_fc1"].astype(np.float64).T
    y = _expert_out(z, up, down)
    zc = np.zeros_like(z)
    for t in range(TINY.T):
        for j in range(TINY.k):
            zc[t] += r["topk_w"][t, j] * y[t, r["topk_idx"][t, j]]
    assert np.allclose(coef.T, zc, rtol=1e-8, atol=1e-8 * np.abs(zc).max())


def test_routing_matches_direct_definition_on_tiny():
    x, W, up, down, r = _layer(TINY)
    l64 = x @ W["w_gate"].astype(np.float64).T
    assert np.all(np.abs(r["logits"] - l64) <= 1e-6 * (1 + np.abs(l64)))
    s = 1 / (1 + np.exp(-l64))
    c = s + W["bias"]
    for t in range(TINY.T):
        ref = sorted(range(TINY.E), key=lambda e: (-c[t, e], e))[:TINY.k]
        assert r["topk_idx"][t].tolist() == ref


@pytest.mark.parametrize("fmt", ["w4a16", "w4a4"])
def test_nvfp4_layer_close_to_dense(fmt):
    cfg = TINY.replace(expert_fmt=fmt)
    x, W, up, down, rq = _layer(cfg, expert_fmt=fmt)
    _, _, _, _, rd = _layer(cfg)
    assert np.array_equal(rq["topk_idx"], rd["topk_idx"])
    rel = np.linalg.norm(rq["out"] - rd["out"]) / np.linalg.norm(rd["out"])
    assert 1e-3 < rel < 0.35     # two fp4 matrices in series, squared ReLU between


def test_skewed_bias_concentrates_load():
    cfg = I.CONFIGS["skewed_prefill_w4a4"].replace(T=256, D=256, L=64, F=64, Fs=64)
    x = I.hidden(cfg).float().numpy()
    l = O.router_logits(x, I.w_gate(cfg).float().numpy())
    _, _, idx, _ = O.route(l, I.gate_bias(cfg).numpy(), cfg.k, cfg.rsf)
    counts, _, _, _ = O.dispatch(idx, cfg.E)
    assert O.max_violation(counts) > 20


# ---------------------------------------------------------------------------
# Planted mistakes: each plausible slip in the oracle's layer (report section
# 5.6 steps 1-7, sections 5.1 and 5.3-5.4) breaks at least one pin above.
# The mistakes are planted in the oracle, on the CPU, and undone afterwards.
# ---------------------------------------------------------------------------

def _holds(pin):
    try:
        pin()
    except AssertionError:
        return False
    return True


_LAYER_PINS = {
    "k_equals_E": test_k_equals_E_is_dense_weighted_sum,
    "k1": test_k1_is_single_mlp_with_weight_rsf,
    "shared_only": test_zero_experts_and_fc2_leave_only_shared_mlp,
    "routing": test_routing_matches_direct_definition_on_tiny,
}


def test_layer_pins_hold_for_the_oracle():
    assert all(_holds(p) for p in _LAYER_PINS.values())


def _plant(monkeypatch, mistake):
    route, relu2, logits = O.route, O.relu2, O.router_logits

    def reroute(fix):
        def wrapped(l, bias, k, rsf, *a, **kw):
            s, choice, idx, w = route(l, bias, k, rsf, *a, **kw)
            return s, choice, idx, fix(s, choice, idx, w, rsf)
        monkeypatch.setattr(O, "route", wrapped)

    def gathered(v, idx):
        return np.take_along_axis(v, idx, axis=1).astype(np.float32)

    if mistake == "relu_not_squared":             # section 5.1: the square dropped
        monkeypatch.setattr(O, "relu2", lambda v: np.maximum(v, 0.0))
    elif mistake == "no_scaling_factor":          # the routed scaling factor left out
        reroute(lambda s, c, idx, w, rsf: (w / np.float32(rsf)).astype(np.float32))
    elif mistake == "unnormalised_weights":       # raw scores, not divided by their sum
        reroute(lambda s, c, idx, w, rsf: gathered(s, idx) * np.float32(rsf))
    elif mistake == "weights_from_biased_score":  # the bias leaking into the weights
        def fix(s, c, idx, w, rsf):
            r = gathered(c, idx)
            return (r / r.sum(1, keepdims=True) * np.float32(rsf)).astype(np.float32)
        reroute(fix)
    elif mistake == "weights_in_wrong_slots":     # slot j weighted by slot j+1's weight
        reroute(lambda s, c, idx, w, rsf: np.roll(w, 1, axis=1))
    elif mistake == "bias_ignored_in_selection":  # plain top-k of the scores
        monkeypatch.setattr(O, "route", lambda l, bias, *a, **kw:
                            route(l, np.zeros_like(bias), *a, **kw))
    elif mistake == "gate_rows_misindexed":       # expert e scored with row E-1-e
        monkeypatch.setattr(O, "router_logits", lambda x, w: logits(x, w[::-1]))
    elif mistake == "shared_expert_dropped":      # the shared MLP's activation lost
        monkeypatch.setattr(O, "relu2", lambda v: relu2(v) * (v.shape[-1] != TINY.Fs))
    elif mistake == "shared_relu_not_squared":    # the shared MLP's square dropped
        monkeypatch.setattr(O, "relu2", lambda v: relu2(v) if v.shape[-1] != TINY.Fs else
                            np.maximum(v, 0.0))
    else:
        raise ValueError(mistake)


@pytest.mark.parametrize("mistake,caught_by", [
    ("relu_not_squared", "k1"), ("no_scaling_factor", "k1"),
    ("unnormalised_weights", "k_equals_E"), ("weights_from_biased_score", "k_equals_E"),
    ("weights_in_wrong_slots", "k_equals_E"), ("bias_ignored_in_selection", "k1"),
    ("gate_rows_misindexed", "routing"), ("shared_expert_dropped", "shared_only"),
    ("shared_relu_not_squared", "shared_only")])
def test_planted_mistakes_break_a_layer_pin(monkeypatch, mistake, caught_by):
    _plant(monkeypatch, mistake)
    assert not _holds(_LAYER_PINS[caught_by])
