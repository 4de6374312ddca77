"""Pins of the oracle's NVFP4 layer (report section 8.1; zhichai.net "NVFP4
format details": E2M1 elements, 16-element blocks along K, one E4M3 scale per
block, one FP32 global scale per expert matrix).

The NVFP4 branches of the layer are fixed by three kinds of cases that do not
call the oracle's own codec to make their expected values:

* experts built from NVFP4-representable values (q * s_b * s_g with every block
  holding a +-6 element, one block per matrix at s_b = 448, so amax = 2688 s_g
  exactly): quantising them changes nothing, so the W4A16 layer must equal the
  dense layer bit for bit, with a different, non-power-of-two-related global
  scale for every matrix;
* the same experts plus latent rows and squared-ReLU activations that lie on
  the E2M1 x E4M3 grid with global scale 1: the W4A4 layer must then equal the
  dense layer bit for bit as well;
* one token worked by hand (below), where a latent element sits on every E2M1
  tie, one squared-ReLU element saturates and one sits on the 0 / 0.5 tie.

The last test plants the plausible mistakes (no rounding of the activations,
rounding along the wrong axis, one global scale shared by all matrices,
rounding before the squared ReLU) into the oracle on the CPU and checks that
each one breaks at least one of these pins.
"""
import numpy as np
import pytest

from oracle import moe_oracle as O

# ---------------------------------------------------------------------------
# helpers: representable matrices built from codes, written from the format
# ---------------------------------------------------------------------------

_E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]        # magnitudes of codes 0..7


def _e4m3(code):
    """Value of a non-negative E4M3 code (bias 7, 3 mantissa bits, exponent 0
    subnormal), written out independently of the oracle's table."""
    e, m = code >> 3, code & 7
    return (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)


def representable(rng, rows, K, s_g):
    """[rows, K] fp32 matrix of values q * s_b * s_g: every 16-block holds a +-6
    element, block (0, 0) has s_b = 448 (so the matrix amax is 2688 * s_g), one
    other block is all zero.  K may end in a partial block of 8 elements (its
    +-6 then lies among those 8)."""
    nb = -(-K // 16)
    codes = rng.randint(0, 16, size=(rows, nb, 16))
    codes[:, :, rng.randint(0, 8)] = 7 + 8 * rng.randint(0, 2)      # +-6 in each block
    sb = np.array([[_e4m3(c) for c in r] for r in rng.randint(0x28, 0x70, size=(rows, nb))])
    sb[0, 0] = 448.0
    q = np.array([[[(-1.0 if c & 8 else 1.0) * _E2M1[c & 7] for c in b] for b in r]
                  for r in codes])
    w = q * sb[..., None] * float(s_g)
    if rows > 1 and nb > 1:
        w[rows - 1, nb - 1] = 0.0
    w = w.reshape(rows, nb * 16)[:, :K]
    assert np.array_equal(w.astype(np.float32).astype(np.float64), w)
    assert np.max(np.abs(w)) == 2688.0 * float(s_g)
    return w.astype(np.float32)


def _run(x, wg, bias, fc1, fc2, su, sd, up, down, k, fmt, rsf=5.0):
    return O.forward(x, wg, bias, fc1, fc2, su, sd,
                     lambda e: up[e].astype(np.float64), lambda e: down[e].astype(np.float64),
                     k=k, rsf=rsf, expert_fmt=fmt)["out"]


# global scales whose pairwise ratios are not powers of two, each with a short
# significand so that 2688 * s_g and the products q * s_b * s_g are exact in fp32
SG = [2.0 ** -9, 3 * 2.0 ** -10, 5 * 2.0 ** -11, 7 * 2.0 ** -12,
      9 * 2.0 ** -12, 11 * 2.0 ** -13, 13 * 2.0 ** -13, 15 * 2.0 ** -14]


def _w4a16_case(seed=0):
    rng = np.random.RandomState(seed)
    T, D, L, E, k, F, Fs = 6, 48, 32, 4, 2, 48, 32
    up = np.stack([representable(rng, F, L, SG[e]) for e in range(E)])
    down = np.stack([representable(rng, L, F, SG[E + e]) for e in range(E)])
    f32 = lambda *s: (rng.standard_normal(s) / np.sqrt(s[-1])).astype(np.float32)
    x = rng.standard_normal((T, D)).astype(np.float32)
    return (x, f32(E, D), (0.1 * rng.standard_normal(E)).astype(np.float32), f32(L, D),
            f32(D, L), f32(Fs, D), f32(D, Fs), up, down, k)


def test_w4a16_equals_dense_on_representable_experts():
    a = _w4a16_case()
    dense, q = _run(*a, "dense"), _run(*a, "w4a16")
    assert np.array_equal(q, dense)
    assert np.abs(dense).max() > 0


def test_w4a16_equals_dense_with_partial_blocks():
    """Expert width F = 40: the down projection's rows (K = F) end in a block of
    8 elements, quantised as a block whose missing elements are zero; on
    representable experts the W4A16 layer still equals the dense one."""
    rng = np.random.RandomState(3)
    T, D, L, E, k, F, Fs = 6, 48, 32, 4, 2, 40, 32
    up = np.stack([representable(rng, F, L, SG[e]) for e in range(E)])
    down = np.stack([representable(rng, L, F, SG[E + e]) for e in range(E)])
    f32 = lambda *s: (rng.standard_normal(s) / np.sqrt(s[-1])).astype(np.float32)
    x = rng.standard_normal((T, D)).astype(np.float32)
    a = (x, f32(E, D), (0.1 * rng.standard_normal(E)).astype(np.float32), f32(L, D),
         f32(D, L), f32(Fs, D), f32(D, Fs), up, down, k)
    dense, q = _run(*a, "dense"), _run(*a, "w4a16")
    assert np.array_equal(q, dense)
    assert np.abs(dense).max() > 0
    # a mistaken reading (the partial block's scale from a 16-element window
    # that reaches into the next row) would change the codes: the oracle's
    # quantiser keeps each row's blocks to that row
    q0, sb0 = O.nvfp4_quantize(down[0], np.float32(O.nvfp4_global_scale(down[0])))
    assert sb0.shape == (L, 3) and q0.shape == (L, F)


def _w4a4_case(seed=1):
    """Latent rows z = x (fc1 = identity) on the grid along L, every expert's
    up projection a signed selection of latent columns, so relu(h)^2 lies on
    the grid along F with block scale 1.5 * 4^j:

    * token t's latent values are {0, +-1.5, +-3} * 2^j_t, column 0 and column 16
      (one per 16-block) are +3 * 2^j_t, the block maximum (s_b = 2^(j_t - 1));
    * up row f has one +-1 at column src[f] (a latent column) plus a pad 6c at
      column 15 or 31, where every token's latent value is 0;
    * each 16-block of up rows holds a row reading column 0 with +1, so every
      F-block of relu(h)^2 holds its maximum 9 * 4^j_t; the other elements are
      0, 2.25 * 4^j_t or 9 * 4^j_t, i.e. codes 0, 3 (1.5) and 7 (6).
    Every matrix has global scale 2^-9 (amax 5.25 from a pad row)."""
    rng = np.random.RandomState(seed)
    T, L, E, k, F, Fs = 16, 32, 4, 2, 32, 16
    D = L
    j = rng.randint(-2, 3, size=T)
    z = rng.choice([0.0, 1.5, -1.5, 3.0, -3.0], size=(T, L))
    z[:, [0, 16]] = 3.0
    z[:, [15, 31]] = 0.0
    x = (z * 2.0 ** j[:, None]).astype(np.float32)
    ups = []
    for e in range(E):
        u = np.zeros((F, L))
        for f in range(F):
            if f % 16 == 15:                 # the row carrying the matrix amax
                u[f, 15] = 5.25
                continue
            src = 0 if f % 16 == e % 16 else rng.choice([c for c in range(L) if c not in (15, 31)])
            sign = 1.0 if src == 0 else rng.choice([1.0, -1.0])
            q = rng.choice([2, 4])            # +-1 = q * c with c = 1 / q
            u[f, src] = sign
            u[f, 15 if src < 16 else 31] = 6.0 / q
        ups.append(u)
    up = np.stack(ups).astype(np.float32)
    down = np.stack([representable(rng, L, F, SG[e]) for e in range(E)])
    f32 = lambda *s: (rng.standard_normal(s) / np.sqrt(s[-1])).astype(np.float32)
    return (x, f32(E, D), (0.1 * rng.standard_normal(E)).astype(np.float32),
            np.eye(L, D, dtype=np.float32), f32(D, L), f32(Fs, D), f32(D, Fs), up, down, k)


def test_w4a4_equals_dense_when_activations_lie_on_the_grid():
    a = _w4a4_case()
    dense, q4, q16 = _run(*a, "dense"), _run(*a, "w4a4"), _run(*a, "w4a16")
    assert np.array_equal(q16, dense)
    assert np.array_equal(q4, dense)


# ---------------------------------------------------------------------------
# One token by hand.  D = L = F = Fs = 16, one expert, k = 1 (weight 5.0
# exactly), fc1 = fc2 = identity, shared expert zero: out = 5 * down . h.
#
# x = z = [6, 1.25, 2.5, 5, 0.25, -3.5, 0, ...].
#   W4A4: block amax 6 -> s_b = E4M3(6 / 6) = 1, codes by round-to-nearest-even
#   on 0 .5 1 1.5 2 3 4 6: 1.25 -> 1, 2.5 -> 2, 5 -> 4, 0.25 -> 0, -3.5 -> -4
#   (every one a tie going to the even code), so zq = [6, 1, 2, 4, 0, -4, 0, ...].
# up (global amax 5.25 -> s_g = 5.25 / 2688 = 2^-9; row pads in column 15):
#   row 0: 2.5 at col 1 (pad 3.75: s_b 320, scale .625, code 4)
#   row 1: 1.5 at col 1; row 2: .5 at col 1; row 3: -1 at col 2; row 4: 1 at col 1
#   (pad 3: s_b 256, scale .5); row 15: 5.25 at col 15 (s_b 448, scale .875).
#   Every weight is representable, so the weights are exact.
#   W4A4: h = [2.5, 1.5, .5, -2, 1, 0, ...]; relu^2 = [6.25, 2.25, .25, 0, 1, 0...]
#   block amax 6.25 -> 6.25 / 6 = 1.0417 -> E4M3 rounds to 1.0 (the midpoint is
#   1.0625), so 6.25 saturates to 6, 2.25 -> 2, .25 (the 0 / .5 tie) -> 0:
#   hq = [6, 2, 0, 0, 1, 0, ...].
#   dense: h = [3.125, 1.875, .625, -2.5, 1.25]; relu^2 = [9.765625, 3.515625,
#   .390625, 0, 1.5625].
# down (global amax 7.875 -> s_g = 7.875 / 2688 = 3 * 2^-10, pads 2.25 in col 15
#   = 6 * .375 with s_b 128):
#   row 0: 7.875 at col 0 (s_b 448, scale 1.3125)
#   row 1: .75 at col 1, 1.5 at col 4;  row 2: .375 at col 0, -1.5 at col 4
#   row 3: -1.125 at col 1, .75 at col 2
#   W4A4: y = [7.875*6, .75*2 + 1.5*1, .375*6 - 1.5*1, -1.125*2 + .75*0]
#           = [47.25, 3, .75, -2.25]
#   dense: y = [76.904296875, 4.98046875, 1.318359375, -3.662109375]
# out = 5 y.
# ---------------------------------------------------------------------------

HAND_X = [6.0, 1.25, 2.5, 5.0, 0.25, -3.5] + [0.0] * 10
HAND_OUT_W4A4 = [236.25, 15.0, 3.75, -11.25] + [0.0] * 12
HAND_OUT_DENSE = [384.521484375, 24.90234375, 6.591796875, -18.310546875] + [0.0] * 12


def _hand_case():
    n = 16
    up = np.zeros((1, n, n))
    up[0, 0, 1], up[0, 0, 15] = 2.5, 3.75
    for f, col, v in [(1, 1, 1.5), (2, 1, 0.5), (3, 2, -1.0), (4, 1, 1.0)]:
        up[0, f, col], up[0, f, 15] = v, 3.0
    up[0, 15, 15] = 5.25
    down = np.zeros((1, n, n))
    down[0, 0, 0] = 7.875
    down[0, 1, 1], down[0, 1, 4] = 0.75, 1.5
    down[0, 2, 0], down[0, 2, 4] = 0.375, -1.5
    down[0, 3, 1], down[0, 3, 2] = -1.125, 0.75
    down[0, 1:4, 15] = 2.25
    eye = np.eye(n, dtype=np.float32)
    zero = np.zeros((n, n), np.float32)
    x = np.array([HAND_X], np.float32)
    return (x, np.zeros((1, n), np.float32), np.zeros(1, np.float32), eye, eye, zero, zero,
            up.astype(np.float32), down.astype(np.float32), 1)


def test_hand_worked_token():
    a = _hand_case()
    assert _run(*a, "w4a4").tolist() == [HAND_OUT_W4A4]
    assert _run(*a, "w4a16").tolist() == [HAND_OUT_DENSE]
    assert _run(*a, "dense").tolist() == [HAND_OUT_DENSE]


# ---------------------------------------------------------------------------
# Planted mistakes (in the oracle, on the CPU): each must break a pin above.
# ---------------------------------------------------------------------------


_CALLS = {"n": 0}           # activation roundings since the forward began


def _pins():
    """Each pin above as a bool, for the oracle as currently patched (a pin
    whose forward raises counts as broken)."""
    def check(f):
        try:
            return bool(f())
        except (AssertionError, ValueError):
            return False

    def run(a, fmt):
        _CALLS["n"] = 0
        return _run(*a, fmt)
    a, b, c = _w4a16_case(), _w4a4_case(), _hand_case()
    return {
        "w4a16": check(lambda: np.array_equal(run(a, "w4a16"), run(a, "dense"))),
        "w4a4": check(lambda: np.array_equal(run(b, "w4a4"), run(b, "dense"))),
        "hand": check(lambda: run(c, "w4a4").tolist() == [HAND_OUT_W4A4]),
    }


def _z_then_h(fz, fh):
    """fz on the first activation rounding of a forward (the latent z), fh on
    the later ones (each expert's relu(h)^2)."""
    def wrapped(a, *scale):
        _CALLS["n"] += 1
        return fz(a, *scale) if _CALLS["n"] == 1 else fh(a, *scale)
    return wrapped


def test_pins_hold_for_the_oracle():
    assert all(_pins().values())


@pytest.mark.parametrize("mistake,caught_by", [
    ("no_h_rounding", "hand"), ("no_z_rounding", "hand"), ("z_wrong_axis", "w4a4"),
    ("shared_gscale", "w4a16"), ("round_before_relu2", "hand")])
def test_planted_mistakes_break_a_pin(monkeypatch, mistake, caught_by):
    rt = O.nvfp4_roundtrip_activation
    ident = lambda a, *scale: np.asarray(a, dtype=np.float32).astype(np.float64)
    if mistake == "no_h_rounding":
        monkeypatch.setattr(O, "nvfp4_roundtrip_activation", _z_then_h(rt, ident))
    elif mistake == "no_z_rounding":
        monkeypatch.setattr(O, "nvfp4_roundtrip_activation", _z_then_h(ident, rt))
    elif mistake == "z_wrong_axis":           # blocks of 16 tokens instead of 16 latents
        monkeypatch.setattr(O, "nvfp4_roundtrip_activation",
                            _z_then_h(lambda a, *scale: rt(np.asarray(a).T, *scale).T, rt))
    elif mistake == "shared_gscale":          # the first matrix's s_g for every matrix
        first = {}
        g = O.nvfp4_global_scale
        monkeypatch.setattr(O, "nvfp4_global_scale", lambda w: first.setdefault("s", g(w)))
    elif mistake == "round_before_relu2":     # h rounded, then squared
        r2 = O.relu2
        monkeypatch.setattr(O, "nvfp4_roundtrip_activation", _z_then_h(rt, ident))
        monkeypatch.setattr(O, "relu2", lambda v: r2(rt(v)))
    assert not _pins()[caught_by]


# ---------------------------------------------------------------------------
# The latent's per-tensor global scale (act_scale "tensor"): s_g = amax(z) /
# (6 * 448) in fp32, the weights' rule applied to the activation tensor.
# ---------------------------------------------------------------------------


def _quantise_with_own_scale(z):
    sg = O.nvfp4_global_scale(z)
    return O.nvfp4_quantize(np.asarray(z, np.float32), sg), sg


@pytest.mark.parametrize("j", [-7, -1, 3, 9])
def test_tensor_scale_codes_invariant_under_power_of_two_scaling(j):
    """Scaling a tensor by 2^j scales its amax, hence its global scale and every
    block's ratio, by 2^j exactly: the codes and E4M3 scales do not change."""
    rng = np.random.RandomState(20 + j)
    z = (rng.standard_normal((24, 128)) * np.exp(rng.uniform(-3, 3, (24, 1)))).astype(np.float32)
    (q0, s0), g0 = _quantise_with_own_scale(z)
    (q1, s1), g1 = _quantise_with_own_scale(z * np.float32(2.0 ** j))
    assert g1 == np.float32(g0 * np.float32(2.0 ** j))
    assert np.array_equal(q0, q1) and np.array_equal(s0, s1)


def test_tensor_scale_keeps_what_unit_scale_saturates():
    """A block maximum of 10000 exceeds what global scale 1 can represent
    (6 * 448 = 2688): with the tensor's own scale it survives up to the fp32
    rounding of that scale."""
    z = np.zeros((1, 16), np.float32)
    z[0, 0], z[0, 1] = 10000.0, 1.0
    unit = O.nvfp4_roundtrip_activation(z)
    assert unit[0, 0] == 2688.0
    sg = O.nvfp4_global_scale(z)
    tens = O.nvfp4_roundtrip_activation(z, sg)
    assert abs(tens[0, 0] - 10000.0) <= 10000.0 * 2.0 ** -22
    assert tens[0, 1] == 0.0          # 1 / (448 * s_g) = 0.27 rounds to code 0 next to 10000


def test_tensor_scale_equals_unit_scale_when_it_is_a_power_of_two():
    """With amax(z) = 2688 * 2^-10 the tensor's scale is exactly 2^-10; every
    block's E4M3 scale is then the unit-scale one times 2^10 (both normal) and
    the codes agree, so the two W4A4 layers are equal bit for bit."""
    rng = np.random.RandomState(31)
    T, L, E, k, F, Fs = 8, 32, 4, 2, 32, 16
    z = rng.uniform(-1, 1, (T, L)) * 2.0
    z[:, ::16] = 0.25 * np.sign(z[:, ::16])          # every block's amax >= 0.25
    z[0, 5] = 2688.0 * 2.0 ** -10                     # the tensor's amax, 2.625
    x = z.astype(np.float32)
    f32 = lambda *s: (rng.standard_normal(s) / np.sqrt(s[-1])).astype(np.float32)
    up, down = f32(E, F, L), f32(E, L, F)
    args = (x, f32(E, L), (0.1 * rng.standard_normal(E)).astype(np.float32),
            np.eye(L, dtype=np.float32), f32(L, L), f32(Fs, L), f32(L, Fs), up, down, k)
    assert O.nvfp4_global_scale(x) == np.float32(2.0 ** -10)
    unit = O.forward(*args[:7], lambda e: up[e].astype(np.float64),
                     lambda e: down[e].astype(np.float64), k=k, rsf=5.0, expert_fmt="w4a4")
    tens = O.forward(*args[:7], lambda e: up[e].astype(np.float64),
                     lambda e: down[e].astype(np.float64), k=k, rsf=5.0, expert_fmt="w4a4",
                     act_scale="tensor")
    assert np.array_equal(unit["out"], tens["out"])
    # and a tensor whose scale is not a power of two gives a different layer
    x2 = x * np.float32(1.5)
    a2 = (x2,) + args[1:7]
    u2 = O.forward(*a2, lambda e: up[e].astype(np.float64), lambda e: down[e].astype(np.float64),
                   k=k, rsf=5.0, expert_fmt="w4a4")
    t2 = O.forward(*a2, lambda e: up[e].astype(np.float64), lambda e: down[e].astype(np.float64),
                   k=k, rsf=5.0, expert_fmt="w4a4", act_scale="tensor")
    assert not np.array_equal(u2["out"], t2["out"])
