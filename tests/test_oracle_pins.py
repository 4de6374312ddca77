"""Pins of the CPU oracle against facts the pages and mathematics fix.

Each test checks the oracle against something other than itself: numbers the
Nemotron-3-Ultra architecture report prints (section 2.3.4 parameter shapes,
section 3.1.3 FLOP total, section 8.1 E2M1 value set), closed forms, brute force
on tiny inputs, libm and exact rational arithmetic.
"""
import fractions
import itertools
import math

import numpy as np
import pytest

from oracle import moe_oracle as O

ULTRA = dict(D=8192, L=2048, E=512, F=5120, Fs=10240)


# --- shapes and work (report section 2.3.4, 2.3.8, 3.1.3) -------------------

def test_param_counts_match_report():
    c = O.param_count(**ULTRA)
    assert c["gate"] == 4_194_304            # gate.weight 512 x 8192
    assert c["bias"] == 512                  # e_score_correction_bias
    assert c["latent"] == 2 * 16_777_216     # fc1 + fc2 latent projections
    assert c["experts"] == 10_737_418_240    # 512 experts x 20,971,520
    assert c["shared"] == 2 * 83_886_080     # shared up + down
    assert c["total"] == 10_942_939_648      # "approx 10.94B"
    assert round(c["total"] / 1e9, 2) == 10.94


def test_tiny_param_count():
    assert O.param_count(D=256, L=64, E=16, F=128, Fs=256)["total"] == 430_096


def test_activated_params_and_flops_match_report():
    # activated parameters per MoE layer ~ 667.5M (section 2.3.8, which sums
    # rounded terms: 4.19M + 33.55M + 22 x 21M + 167.77M)
    act = 4_194_304 + 2 * 16_777_216 + 22 * 20_971_520 + 167_772_160
    assert abs(act / 667.5e6 - 1) < 1e-3
    f = O.flops_per_token(D=8192, L=2048, E=512, k=22, F=5120, Fs=10240)
    # every activated weight is used once per token in a multiply-add
    assert f["total"] == 2 * act
    assert round(f["total"] / 1e9, 2) == 1.33   # section 3.1.3: ~1.33e9 * T


# --- router logits: fixed-order fp64 dot products ----------------------------

def _dot_sequential(a, b):
    """The stated order, one scalar at a time, from dot_spec_order."""
    order = O.dot_spec_order(len(a))
    part = [0.0] * 32
    for p in range(32):
        for k in order[p]:
            part[p] = part[p] + float(a[k]) * float(b[k])
    for off in (16, 8, 4, 2, 1):
        for j in range(off):
            part[j] = part[j] + part[j + off]
    return part[0]


@pytest.mark.parametrize("K", [8, 256, 300, 1000])
def test_dot_spec_follows_stated_order(K):
    rng = np.random.RandomState(K)
    a = (rng.standard_normal(K) * np.exp(rng.uniform(-8, 8, K))).astype(np.float32)
    b = rng.standard_normal(K).astype(np.float32)
    assert O.dot_spec(a, b) == _dot_sequential(a, b)


@pytest.mark.parametrize("K", [256, 8192])
def test_dot_spec_within_summation_bound(K):
    rng = np.random.RandomState(1)
    a = rng.standard_normal(K).astype(np.float32)
    b = rng.standard_normal(K).astype(np.float32)
    exact = sum(fractions.Fraction(float(x)) * fractions.Fraction(float(y))
                for x, y in zip(a, b))
    got = O.dot_spec(a, b)
    u = 2.0 ** -53
    bound = (K * u / (1 - K * u)) * float(np.sum(np.abs(a.astype(np.float64) * b)))
    assert abs(got - float(exact)) <= bound


def test_dot_spec_exact_on_integers():
    rng = np.random.RandomState(2)
    a = rng.randint(-100, 100, 4096).astype(np.float64)
    b = rng.randint(-100, 100, 4096).astype(np.float64)
    assert O.dot_spec(a, b) == float(np.dot(a.astype(np.int64), b.astype(np.int64)))


def test_router_logits_broadcast_shape():
    x = np.ones((3, 256), np.float32)
    w = np.arange(5 * 256, dtype=np.float32).reshape(5, 256) / 256
    l = O.router_logits(x, w)
    assert l.dtype == np.float32 and l.shape == (3, 5)
    assert l[0, 1] == np.float32(sum(range(256, 512)) / 256)


# --- sigmoid gating (section 5.3) --------------------------------------------

# ln 2 to 40 digits, as a rational
_LN2_Q = fractions.Fraction("0.6931471805599453094172321214581765680755")


def _ulp_diff(a, b):
    ia = np.asarray(a, np.float64).view(np.int64)
    ib = np.asarray(b, np.float64).view(np.int64)
    return np.abs(ia - ib)


def test_exp_spec_against_libm():
    a = np.concatenate([np.linspace(-80, 80, 200001),
                        np.random.RandomState(3).uniform(-80, 80, 100000)])
    ref = np.array([math.exp(v) for v in a])
    assert _ulp_diff(O.exp_spec(a), ref).max() <= 2


def test_exp_spec_special_values():
    assert O.exp_spec(np.array([0.0]))[0] == 1.0
    for n in range(-100, 101, 7):        # 2**n at n*ln 2 (argument rounded to fp64)
        a = n * math.log(2)
        v = O.exp_spec(np.array([a]))[0]
        rel_arg = abs(float(fractions.Fraction(a) - n * _LN2_Q))   # |a - n ln 2|
        assert abs(v / 2.0 ** n - 1) <= rel_arg + 4e-16
    x = np.linspace(-80, 80, 100001)
    assert np.all(np.diff(O.exp_spec(x)) > 0)            # strictly increasing


def test_sigmoid_spec_against_libm_fp32():
    l = np.concatenate([np.linspace(-90, 90, 100001),
                        np.random.RandomState(4).standard_normal(100000) * 3]
                       ).astype(np.float32)
    ref = np.array([1.0 / (1.0 + math.exp(-min(max(float(v), -80), 80)))
                    for v in l]).astype(np.float32)
    got = O.sigmoid_spec(l)
    d = np.abs(got.view(np.int32).astype(np.int64) - ref.view(np.int32))
    assert d.max() <= 1 and (d == 0).mean() > 0.999
    assert O.sigmoid_spec(np.array([0.0], np.float32))[0] == np.float32(0.5)
    assert np.all((got > 0) & (got <= 1))


# --- selection (sections 5.4-5.6) ---------------------------------------------

def _brute_topk(c, k):
    """The subset of size k whose members all rank above every non-member under
    the order (score desc, index asc), found by enumerating every subset."""
    E = len(c)
    key = lambda e: (-float(c[e]), e)
    found = []
    for sub in itertools.combinations(range(E), k):
        rest = [e for e in range(E) if e not in sub]
        if all(key(a) < key(b) for a in sub for b in rest):
            found.append(sub)
    assert len(found) == 1
    return sorted(found[0], key=key)


def test_select_topk_brute_force_with_ties():
    rng = np.random.RandomState(5)
    for _ in range(300):
        E = rng.randint(2, 9)
        k = rng.randint(1, min(3, E) + 1)
        c = (rng.randint(0, 4, size=(1, E)) / 4.0).astype(np.float32)  # many ties
        got = O.select_topk(c, k)[0].tolist()
        assert got == _brute_topk(c[0], k)


def test_zero_bias_gives_plain_topk_of_scores():
    rng = np.random.RandomState(6)
    l = rng.standard_normal((50, 64)).astype(np.float32)
    s, _, idx, _ = O.route(l, np.zeros(64, np.float32), 6, 5.0)
    for t in range(50):
        ref = sorted(range(64), key=lambda e: (-float(s[t, e]), e))[:6]
        assert idx[t].tolist() == ref


def test_bias_changes_choice_but_not_weights():
    # hand example: s = sigmoid(l) with l = 0, ln 3, -ln 3, 0  ->  .5 .75 .25 .5
    l = np.array([[0.0, math.log(3), -math.log(3), 0.0]], np.float32)
    bias = np.array([0.0, -1.0, 0.0, 0.3], np.float32)
    s, choice, idx, w = O.route(l, bias, 2, 5.0)
    assert np.allclose(s[0], [0.5, 0.75, 0.25, 0.5], atol=1e-7)
    assert idx[0].tolist() == [3, 0]          # choices .8, .5, .25, -.25
    # weights use the raw scores .5 and .5: normalised to 1/2 each, times 5
    assert w[0].tolist() == [2.5, 2.5]


def test_weights_sum_to_scaling_factor():
    rng = np.random.RandomState(7)
    l = (rng.standard_normal((200, 512)) * 2).astype(np.float32)
    b = (rng.standard_normal(512) * 0.1).astype(np.float32)
    _, _, idx, w = O.route(l, b, 22, 5.0)
    assert np.all(np.abs(w.astype(np.float64).sum(1) / 5.0 - 1) < 2 ** -20)
    assert np.all((w > 0) & (w <= 5.0))
    assert np.all([len(set(r)) == 22 for r in idx.tolist()])


def test_top1_weight_is_exactly_the_scaling_factor():
    l = np.random.RandomState(8).standard_normal((30, 16)).astype(np.float32)
    _, _, _, w = O.route(l, np.zeros(16, np.float32), 1, 5.0)
    assert np.all(w == np.float32(5.0))


def test_group_routing_hand_example():
    # 2 groups of 3; group scores (top-2 sums): g0 = .9+.1 = 1.0, g1 = .8+.7 = 1.5
    c = np.array([[0.9, 0.1, 0.0, 0.8, 0.7, 0.05]], np.float32)
    m = O.group_mask(c, 2, 1)
    assert m[0].tolist() == [False] * 3 + [True] * 3
    assert O.select_topk(c, 2, m)[0].tolist() == [3, 4]
    assert O.group_mask(c, 1, 1).all()


def test_max_violation_when_one_set_takes_everything():
    idx = np.tile(np.arange(22, dtype=np.int32), (64, 1))
    counts, _, _, _ = O.dispatch(idx, 512)
    assert abs(O.max_violation(counts) - 512 / 22) < 1e-12
    assert round(512 / 22, 2) == 23.27   # report section 10.3 / explainer figure


def test_dispatch_against_comparison_sort():
    rng = np.random.RandomState(9)
    T, E, k = 97, 40, 5
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    counts, offsets, perm, pos = O.dispatch(idx, E)
    flat = idx.reshape(-1)
    order = np.argsort(flat.astype(np.int64) * (T * k) + np.arange(T * k), kind="stable")
    assert perm.tolist() == order.tolist()
    assert counts.tolist() == np.bincount(flat, minlength=E).tolist()
    assert offsets[-1] == T * k and np.all(np.diff(offsets) == counts)
    assert np.all(perm[pos.reshape(-1)] == np.arange(T * k))


# --- printed values (tests/golden/report_values.json) ------------------------

import json
import os

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                     "report_values.json")))


def test_golden_param_counts():
    g = GOLDEN["param_counts"]
    c = O.param_count(**ULTRA)
    assert c["gate"] == g["gate_weight"] and c["bias"] == g["e_score_correction_bias"]
    assert c["latent"] == g["fc1_latent_proj"] + g["fc2_latent_proj"]
    assert c["experts"] == g["all_experts"] == 512 * g["one_expert"]
    assert c["shared"] == g["shared_up"] + g["shared_down"]
    assert round(c["total"] / 1e9, 2) == g["layer_total_billions_2dp"]
    assert round(O.flops_per_token(D=8192, L=2048, E=512, k=22, F=5120, Fs=10240)
                 ["total"] / 1e9, 2) == GOLDEN["moe_flops_per_token_billions_2dp"]


# --- NVFP4 codec (section 8.1; NVFP4 format details) -------------------------

def test_e2m1_value_set_matches_report():
    vals = sorted(set(abs(v) for v in O.E2M1_TABLE.tolist()))
    assert vals == GOLDEN["e2m1_values"]
    assert sorted(set(O.E2M1_TABLE.tolist())) == sorted(
        set(GOLDEN["e2m1_values"]) | {-v for v in GOLDEN["e2m1_values"]})


def test_e2m1_exhaustive_roundtrip_and_ties():
    for c in range(16):
        v = O.e2m1_value(c)
        assert O.e2m1_encode(v) == (0 if c == 8 else c)     # -0 encodes as +0
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0,
            5.0: 4.0, 7.0: 6.0, 100.0: 6.0}
    for x, v in ties.items():
        assert O.e2m1_value(O.e2m1_encode(x)) == v
        assert O.e2m1_value(O.e2m1_encode(-x)) == -v


def test_e4m3_exhaustive():
    finite = [c for c in range(256) if (c & 0x7F) != 0x7F]
    assert len(finite) == 254
    assert max(O.e4m3_value(c) for c in finite) == 448.0
    assert O.e4m3_value(1) == 2.0 ** -9                      # smallest subnormal
    assert O.e4m3_value(0x08) == 2.0 ** -6                   # smallest normal
    for c in range(0x7F):
        assert O.e4m3_encode(O.e4m3_value(c)) == c
    assert O.e4m3_encode(1000.0) == 0x7E                      # satfinite
    # ties between neighbours go to the even code
    for c in range(0, 0x7E):
        mid = (O.e4m3_value(c) + O.e4m3_value(c + 1)) / 2
        assert O.e4m3_encode(mid) == (c if c % 2 == 0 else c + 1)


def test_nvfp4_roundtrip_of_representable_values_is_exact():
    rng = np.random.RandomState(10)
    rows, K = 24, 128
    sg = np.float32(1.25 * 2.0 ** -7)      # short mantissa: q*s_b*s_g exact in fp32
    sb = rng.randint(0x20, 0x60, size=(rows, K // 16)).astype(np.uint8)
    q = rng.randint(0, 16, size=(rows, K)).astype(np.uint8)
    q[:, ::16] = 7                      # every block holds +6: its amax is 6*scale
    w = O.nvfp4_dequantize(q, sb, sg).astype(np.float32)
    assert np.all(w.astype(np.float64) == O.nvfp4_dequantize(q, sb, sg))
    q2, sb2 = O.nvfp4_quantize(w, sg)
    assert np.array_equal(O.nvfp4_dequantize(q2, sb2, sg),
                          O.nvfp4_dequantize(q, sb, sg))


def test_nvfp4_error_bound_and_scales():
    rng = np.random.RandomState(11)
    w = (rng.standard_normal((64, 256)) * 0.02).astype(np.float32)
    sg = O.nvfp4_global_scale(w)
    assert sg == np.float32(np.abs(w).max() / np.float32(2688.0))
    q, sb = O.nvfp4_quantize(w, sg)
    assert q.max() < 16 and np.all((sb & 0x7F) != 0x7F)
    deq = O.nvfp4_dequantize(q, sb, sg)
    scale = O.E4M3_TABLE[sb].astype(np.float32) * sg
    err = np.abs(deq - w).reshape(64, 16, 16)
    # worst grid gap is 2 (between 4 and 6): half of it times the block scale,
    # or the saturation overshoot when the rounded block scale came out small
    over = np.maximum(np.abs(w).reshape(64, 16, 16) - 6 * scale[..., None], 0)
    assert np.all(err <= scale[..., None] * 1.0 + over + 1e-12)
    rel = np.linalg.norm(deq - w) / np.linalg.norm(w)
    assert rel < 0.12


def test_nvfp4_partial_block_hand_example():
    """A row of 24 elements: one full block and a partial block of 8.  The
    partial block's scale comes from its own 8 values (amax 7: 7/6 = 1.1667
    lies nearer the E4M3 value 1.125 than 1.25), and each value rounds on the
    E2M1 grid scaled by 1.125 (7/1.125 = 6.22 -> 6; 0.3/1.125 = 0.267 -> 0.5;
    -2/1.125 = -1.78 -> -2; 1/1.125 = 0.89 -> 1), worked out by hand."""
    full = np.full(16, 0.75, np.float32)              # amax 0.75: s_b = 0.125 exactly
    part = np.array([7.0, 0.3, -2.0, 1.0, 0.0, 0.0, 0.0, 0.0], np.float32)
    w = np.concatenate([full, part])[None, :]
    q, sb = O.nvfp4_quantize(w, np.float32(1.0))
    assert q.shape == (1, 24) and sb.shape == (1, 2)
    assert O.e4m3_value(int(sb[0, 0])) == 0.125 and O.e4m3_value(int(sb[0, 1])) == 1.125
    deq = O.nvfp4_dequantize(q, sb, np.float32(1.0))
    assert deq[0, :16].tolist() == [0.75] * 16
    assert deq[0, 16:].tolist() == [6.75, 0.5625, -2.25, 1.125, 0.0, 0.0, 0.0, 0.0]


def test_nvfp4_partial_block_is_local_and_roundtrips_representable_values():
    rng = np.random.RandomState(13)
    rows, K = 6, 40                                   # blocks of 16, 16 and 8
    sg = np.float32(1.0)
    sb = rng.randint(0x20, 0x48, size=(rows, 3)).astype(np.uint8)
    q = rng.randint(0, 16, size=(rows, K)).astype(np.uint8)
    q[:, [0, 16, 32]] = 7                            # +6 in every block, partial included
    w = O.nvfp4_dequantize(q, sb, sg).astype(np.float32)
    q2, sb2 = O.nvfp4_quantize(w, sg)
    assert np.array_equal(sb2, sb)
    assert np.array_equal(O.nvfp4_dequantize(q2, sb2, sg), O.nvfp4_dequantize(q, sb, sg))
    # changing the full blocks changes neither the partial block's scale nor its codes
    w3 = w.copy()
    w3[:, :32] *= 3.0
    q3, sb3 = O.nvfp4_quantize(w3, sg)
    assert np.array_equal(sb3[:, 2], sb2[:, 2]) and np.array_equal(q3[:, 32:], q2[:, 32:])


def test_pack_e2m1_low_nibble_first():
    c = np.array([[1, 2, 15, 0]], np.uint8)
    assert O.pack_e2m1(c).tolist() == [[0x21, 0x0F]]


def test_e2m1_vector_encoder_matches_scalar_definition():
    x = np.concatenate([np.linspace(-7, 7, 5601), np.array([0.25, 0.75, 1.25, 1.75, 2.5,
                                                             3.5, 5.0, -0.25, -5.0, 0.0])])
    assert [O.e2m1_encode(v) for v in x] == O.e2m1_encode_vec(x.astype(np.float32)).tolist()


def test_e4m3_vector_encoder_matches_scalar_definition():
    y = np.abs(np.random.RandomState(12).standard_normal(4000)) * np.logspace(-4, 3, 4000)
    mids = [(O.e4m3_value(c) + O.e4m3_value(c + 1)) / 2 for c in range(0, 0x7E)]
    y = np.concatenate([y, mids, [0.0, 448.0, 500.0]])
    assert [O.e4m3_encode(v) for v in y] == O.e4m3_encode_vec(y).tolist()


def _brute_group_mask(c, n_group, topk_group):
    """Group selection written independently: a group's score is the largest
    fp32 sum over pairs of its experts (= the sum of its two largest), and the
    kept set is the one subset of topk_group groups whose every member ranks
    above every non-member ((score, -index) order), found by enumeration."""
    import itertools
    T, E = c.shape
    G = E // n_group
    out = np.zeros((T, E), dtype=bool)
    for t in range(T):
        sc = []
        for g in range(n_group):
            vals = c[t, g * G:(g + 1) * G]
            sc.append(max(np.float32(vals[i]) + np.float32(vals[j])
                          for i in range(G) for j in range(i + 1, G)))
        above = lambda a, b: sc[a] > sc[b] or (sc[a] == sc[b] and a < b)
        kept = [S for S in itertools.combinations(range(n_group), topk_group)
                if all(above(a, b) for a in S for b in range(n_group) if b not in S)]
        assert len(kept) == 1
        for g in kept[0]:
            out[t, g * G:(g + 1) * G] = True
    return out


@pytest.mark.parametrize("E,n_group,topk_group", [(12, 4, 2), (16, 8, 3), (12, 6, 1), (8, 2, 2)])
def test_group_mask_against_enumeration(E, n_group, topk_group):
    rng = np.random.RandomState(E * 100 + n_group)
    c = rng.standard_normal((40, E)).astype(np.float32)
    c[:5] = np.round(c[:5])                    # exact ties between group scores
    assert np.array_equal(O.group_mask(c, n_group, topk_group),
                          _brute_group_mask(c, n_group, topk_group))


def test_group_routing_selects_inside_kept_groups_and_reduces_to_plain_topk():
    rng = np.random.RandomState(21)
    l = rng.standard_normal((50, 32)).astype(np.float32)
    b = (0.1 * rng.standard_normal(32)).astype(np.float32)
    _, choice, idx, w = O.route(l, b, 6, 5.0, n_group=8, topk_group=3)
    m = O.group_mask(choice, 8, 3)
    assert all(m[t, idx[t]].all() for t in range(50))
    # within the kept groups the choice is the plain top-k
    ref = O.select_topk(np.where(m, choice, -np.inf).astype(np.float32), 6)
    assert np.array_equal(idx, ref)
    # keeping every group is plain routing
    assert np.array_equal(O.route(l, b, 6, 5.0, n_group=8, topk_group=8)[2],
                          O.route(l, b, 6, 5.0)[2])
    assert np.allclose(w.sum(axis=1), 5.0, rtol=1e-6)


# ---- block wrapper: RMSNorm and the residual add ---------------------------


def test_rmsnorm_closed_forms_and_invariants():
    """Pins of rmsnorm_spec that do not restate its formula:
    * eps = 0, x = c * ones with c a power of two: every step is exact, so
      y = sign(c) * g exactly;
    * eps = 0: scaling x by a power of two changes nothing, bit for bit;
    * eps = 0, g = 1: the normalised rows have mean square 1 (to rounding);
    * x = 0 gives y = 0 (eps keeps the root positive);
    * eps shrinks the result: |y(eps)| < |y(0)| for eps > 0."""
    D = 512
    rng = np.random.RandomState(5)
    g = (1.0 + 0.1 * rng.standard_normal(D)).astype(np.float32)
    for c in (1.0, -0.25, 8.0):
        x = np.full((1, D), c)
        assert np.array_equal(O.rmsnorm_spec(x, g, 0.0), (np.sign(c) * g.astype(np.float64))[None])
    x = rng.standard_normal((6, D)).astype(np.float32)
    assert np.array_equal(O.rmsnorm_spec(4.0 * x, g, 0.0), O.rmsnorm_spec(x, g, 0.0))
    y = O.rmsnorm_spec(x, np.ones(D, np.float32), 0.0)
    assert np.allclose((y ** 2).mean(axis=1), 1.0, rtol=1e-12)
    assert np.array_equal(O.rmsnorm_spec(np.zeros((2, D)), g, 1e-5), np.zeros((2, D)))
    assert np.all(np.abs(O.rmsnorm_spec(x, g, 1e-2)) < np.abs(O.rmsnorm_spec(x, g, 0.0)))


def test_rmsnorm_eps_inside_the_root():
    """eps sits under the square root: with mean(x^2) + eps a perfect square
    every step is exact, so x = 0.75 (eps 0.4375: root 1) and x = 1.5 (eps
    1.75: root 2) give y = 0.75 g exactly; eps added after the root would give
    0.75 / 1.1875 and 1.5 / 3.25."""
    D = 512
    g = (1.0 + 0.1 * np.random.RandomState(6).standard_normal(D)).astype(np.float32)
    for c, eps in ((0.75, 0.4375), (1.5, 1.75)):
        y = O.rmsnorm_spec(np.full((2, D), c), g, eps)
        assert np.array_equal(y, np.tile(0.75 * g.astype(np.float64), (2, 1)))
    half = np.zeros((1, D))
    half[0, ::2] = 1.0                              # mean square 0.5, eps 0.5: root 1
    assert np.array_equal(O.rmsnorm_spec(half, g, 0.5), half * g.astype(np.float64))


def test_bf16_rounding_from_fp64_against_brute_force():
    """round_fp64_to_bf16 equals the nearest point of an enumerated bf16 grid
    (ties to the even significand), including exact midpoints."""
    grid = np.array(sorted({float(np.float32(np.uint32(b << 16).view(np.float32)))
                            for b in range(0x3E00, 0x4100)}))       # 2^-3 .. 8
    rng = np.random.RandomState(9)
    mids = (grid[:-1] + grid[1:]) / 2
    ys = np.concatenate([grid, mids, mids + 2.0 ** -40, mids - 2.0 ** -40,
                         rng.uniform(0.2, 7.0, 2000)])
    ys = np.concatenate([ys, -ys])
    got = O.round_fp64_to_bf16(ys).astype(np.float64)
    for y, r in zip(ys, got):
        a = np.abs(y)
        i = np.searchsorted(grid, a)
        lo, hi = grid[max(i - 1, 0)], grid[min(i, len(grid) - 1)]
        if a - lo < hi - a:
            want = lo
        elif hi - a < a - lo:
            want = hi
        else:                                   # tie: the even significand
            even = lambda v: (np.float32(v).view(np.uint32) >> 16) % 2 == 0
            want = lo if even(lo) else hi
        assert r == np.copysign(want, y), (y, r, want)


def test_block_forward_residual_pins():
    """With zero experts, zero shared expert and zero fc2 the layer adds
    nothing and the block returns its input; with g = 0 the layer reads zero
    rows, whose output is zero whatever the routing."""
    rng = np.random.RandomState(3)
    T, D, L, E, k, F, Fs = 5, 64, 16, 8, 2, 32, 32
    x = rng.standard_normal((T, D)).astype(np.float32)
    wg = rng.standard_normal((E, D)).astype(np.float32)
    b = (0.1 * rng.standard_normal(E)).astype(np.float32)
    zero = lambda *s: np.zeros(s, np.float32)
    r = O.block_forward(x, np.ones(D, np.float32), 1e-5, wg, b, rng.standard_normal((L, D)),
                        zero(D, L), rng.standard_normal((Fs, D)), zero(D, Fs),
                        lambda e: zero(F, L), lambda e: zero(L, F), k=k, rsf=5.0, dtype="fp32")
    assert np.array_equal(r["out"], x.astype(np.float64))
    up = rng.standard_normal((E, F, L)).astype(np.float32)
    dn = rng.standard_normal((E, L, F)).astype(np.float32)
    r = O.block_forward(x, np.zeros(D, np.float32), 1e-5, wg, b, rng.standard_normal((L, D)),
                        rng.standard_normal((D, L)), rng.standard_normal((Fs, D)),
                        rng.standard_normal((D, Fs)), lambda e: up[e], lambda e: dn[e],
                        k=k, rsf=5.0, dtype="fp32")
    assert np.array_equal(r["y_in"], np.zeros((T, D), np.float32))
    assert np.array_equal(r["out"], x.astype(np.float64))
