"""Planted mistakes in the oracle's router, codec and norm functions: each
plausible slip breaks at least one pin of tests/test_oracle_pins.py, so the
pins would have caught it.  Mistakes are planted in the oracle, on the CPU,
with monkeypatch (undone after each test); the pins run unchanged.

Sources of the behaviour each pin fixes: the Nemotron-3-Ultra architecture
report, section 5.3 (sigmoid gating), 5.4-5.5 (correction bias, top-k, group
routing), 5.6 step 6 (token / expert grouping), 8.1 and the "NVFP4 format
details" commentary (E2M1 / E4M3 codecs), and the block's pre-norm RMSNorm.
"""
import numpy as np
import pytest

from oracle import moe_oracle as O
from tests import test_oracle_pins as P


def _holds(pin, *args):
    try:
        pin(*args)
    except AssertionError:
        return False
    return True


PINS = {
    "dot_order": lambda: P.test_dot_spec_follows_stated_order(1000),
    "exp_libm": P.test_exp_spec_against_libm,
    "sigmoid_libm": P.test_sigmoid_spec_against_libm_fp32,
    "topk_brute": P.test_select_topk_brute_force_with_ties,
    "bias_hand": P.test_bias_changes_choice_but_not_weights,
    "weights_sum": P.test_weights_sum_to_scaling_factor,
    "group_enum": lambda: P.test_group_mask_against_enumeration(12, 4, 2),
    "group_hand": P.test_group_routing_hand_example,
    "dispatch_sort": P.test_dispatch_against_comparison_sort,
    "e2m1_ties": P.test_e2m1_exhaustive_roundtrip_and_ties,
    "e4m3": P.test_e4m3_exhaustive,
    "rms_closed": P.test_rmsnorm_closed_forms_and_invariants,
    "rms_eps": P.test_rmsnorm_eps_inside_the_root,
    "bf16_grid": P.test_bf16_rounding_from_fp64_against_brute_force,
}


def test_every_pin_holds_for_the_oracle():
    assert [n for n, p in PINS.items() if not _holds(p)] == []


def _group_mask_by_max(choice, n_group, topk_group):
    """A group scored by its single largest member instead of its top two."""
    T, E = choice.shape
    G = E // n_group
    sc = choice.reshape(T, n_group, G).max(axis=2)
    out = np.zeros((T, E), dtype=bool)
    for t in range(T):
        keep = np.lexsort((np.arange(n_group), -sc[t]))[:topk_group]
        for g in keep:
            out[t, g * G:(g + 1) * G] = True
    return out


def _rmsnorm_eps_outside(x, g, eps):
    """eps added after the square root instead of under it."""
    x64 = np.asarray(x, np.float64)
    ms = (x64 * x64).mean(axis=-1)
    return (x64 / (np.sqrt(ms) + np.float64(np.float32(eps)))[..., None]) * np.asarray(g, np.float64)


def _rmsnorm_mean_abs(x, g, eps):
    """Normalised by the mean absolute value instead of the root mean square."""
    x64 = np.asarray(x, np.float64)
    m = np.abs(x64).mean(axis=-1) + np.float64(np.float32(eps))
    return (x64 / m[..., None]) * np.asarray(g, np.float64)


def _plant(monkeypatch, mistake):
    exp, topk, route, disp = O.exp_spec, O.select_topk, O.route, O.dispatch
    e2m1, e4m3 = O.e2m1_encode, O.e4m3_encode
    if mistake == "dot_plain_sum":                 # the fixed summation order ignored
        monkeypatch.setattr(O, "dot_spec", lambda a, b: np.sum(
            np.asarray(a, np.float64) * np.asarray(b, np.float64), axis=-1))
    elif mistake == "ln2_lo_sign":                 # Cody-Waite low part with the wrong sign
        monkeypatch.setattr(O, "LN2_LO", -O.LN2_LO)
    elif mistake == "taylor_truncated":            # exp(r) polynomial cut at degree 7
        monkeypatch.setattr(O, "EXP_TAYLOR", O.EXP_TAYLOR[:8] + [0.0] * (len(O.EXP_TAYLOR) - 8))
    elif mistake == "sigmoid_sign":                # 1 / (1 + exp(+l))
        monkeypatch.setattr(O, "exp_spec", lambda a: exp(-np.asarray(a)))
    elif mistake == "ties_to_higher_index":
        def topk_hi(c, k, eligible=None):
            E = c.shape[1]
            el = None if eligible is None else eligible[:, ::-1]
            return (E - 1 - topk(np.ascontiguousarray(c[:, ::-1]), k, el)).astype(np.int32)
        monkeypatch.setattr(O, "select_topk", topk_hi)
    elif mistake == "weights_from_choice":         # the biased score weights the experts
        def route_choice(l, bias, k, rsf, *a, **kw):
            s, choice, idx, w = route(l, bias, k, rsf, *a, **kw)
            r = np.take_along_axis(choice, idx.astype(np.int64), axis=1).astype(np.float32)
            return s, choice, idx, (r / r.sum(1, keepdims=True) * np.float32(rsf)).astype(np.float32)
        monkeypatch.setattr(O, "route", route_choice)
    elif mistake == "normalised_over_all_experts":  # divided by the sum of every score
        def route_all(l, bias, k, rsf, *a, **kw):
            s, choice, idx, w = route(l, bias, k, rsf, *a, **kw)
            r = np.take_along_axis(s, idx.astype(np.int64), axis=1)
            return s, choice, idx, (r / s.sum(1, keepdims=True) * np.float32(rsf)).astype(np.float32)
        monkeypatch.setattr(O, "route", route_all)
    elif mistake == "group_score_max":
        monkeypatch.setattr(O, "group_mask", _group_mask_by_max)
    elif mistake == "dispatch_tokens_descending":  # within an expert, later tokens first
        def disp_desc(idx, E):
            counts, offsets, perm, pos = disp(idx, E)
            perm = perm.copy()
            for e in range(E):
                perm[offsets[e]:offsets[e + 1]] = perm[offsets[e]:offsets[e + 1]][::-1]
            pos = np.empty_like(pos)
            pos.reshape(-1)[perm] = np.arange(perm.size, dtype=np.int32)
            return counts, offsets, perm, pos
        monkeypatch.setattr(O, "dispatch", disp_desc)
    elif mistake == "e2m1_ties_away":              # round half away from zero
        def enc(x):
            c = e2m1(x)
            a = abs(float(x))
            vals = [O.e2m1_value(i) for i in range(8)]
            for i in range(7):
                if a == (vals[i] + vals[i + 1]) / 2:
                    c = (i + 1) | (8 if x < 0 else 0)
            return c
        monkeypatch.setattr(O, "e2m1_encode", enc)
    elif mistake == "e4m3_no_satfinite":           # overflow to the NaN code
        monkeypatch.setattr(O, "e4m3_encode", lambda x: 0x7F if abs(x) > 464 else e4m3(x))
    elif mistake == "rms_eps_outside_root":
        monkeypatch.setattr(O, "rmsnorm_spec", _rmsnorm_eps_outside)
    elif mistake == "rms_mean_abs":
        monkeypatch.setattr(O, "rmsnorm_spec", _rmsnorm_mean_abs)
    elif mistake == "bf16_truncate":               # chop to 8 bits instead of rounding
        monkeypatch.setattr(O, "round_fp64_to_bf16", lambda y: (
            lambda m, e: np.ldexp(np.trunc(m * 256.0) / 256.0, e).astype(np.float32))(
                *np.frexp(np.asarray(y, np.float64))))
    else:
        raise ValueError(mistake)


@pytest.mark.parametrize("mistake,caught_by", [
    ("dot_plain_sum", "dot_order"),
    ("ln2_lo_sign", "exp_libm"),
    ("taylor_truncated", "exp_libm"),
    ("sigmoid_sign", "sigmoid_libm"),
    ("ties_to_higher_index", "topk_brute"),
    ("weights_from_choice", "bias_hand"),
    ("normalised_over_all_experts", "weights_sum"),
    ("group_score_max", "group_enum"),
    ("group_score_max", "group_hand"),
    ("dispatch_tokens_descending", "dispatch_sort"),
    ("e2m1_ties_away", "e2m1_ties"),
    ("e4m3_no_satfinite", "e4m3"),
    ("rms_eps_outside_root", "rms_eps"),
    ("rms_mean_abs", "rms_closed"),
    ("bf16_truncate", "bf16_grid"),
])
def test_planted_mistake_breaks_a_pin(monkeypatch, mistake, caught_by):
    _plant(monkeypatch, mistake)
    assert not _holds(PINS[caught_by])
