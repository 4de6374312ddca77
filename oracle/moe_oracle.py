"""CPU oracle for the LatentMoE feed-forward layer -- TEST INFRASTRUCTURE ONLY.

Plain, slow, fp64 numpy restatement of what the layer computes, written from
the Nemotron-3-Ultra architecture report (pillumina.github.io), chapter 5
"LatentMoE router", section 5.6 (the seven-step data flow of NemotronHMoE),
sections 5.3-5.5 (sigmoid gating, correction bias, group routing), section
2.3.4 (parameter shapes) and section 8.1 / the zhichai.net commentary "NVFP4
format details" (E2M1 elements, 16-element blocks, E4M3 block scale, FP32
global scale).

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference leg
may import this module.  It shares no code with the CUDA library and never
imports it; its inputs come from latentmoe_expert_routing_b200.inputs (a seeded
generator with none of the layer's arithmetic).

Readings where the pages leave a step open:
  * router logits: the reference computes x.W^T in fp32 with an unspecified
    summation order.  Here the logit is DEFINED as the fp64 sum of the exact
    products in the fixed order of `dot_spec`, rounded once to fp32.
  * sigmoid: 1/(1+exp(-l)) in fp64 with our own `exp_spec` (Cody-Waite range
    reduction + degree-13 Taylor polynomial, + and * only), rounded to fp32.
  * top-k ties go to the lower expert index; slots are ordered by (choice score
    descending, expert ascending).
  * weights: fp32 sum of the raw scores in slot order, w = (r/(S+1e-20))*rsf.
  * no intermediate rounding in the expert / projection math (fp64 throughout).
"""
from __future__ import annotations

import math

import numpy as np

# ---------------------------------------------------------------------------
# Router logits (section 5.6, step 1: the gate logits, x times W_gate^T in fp32)
# ---------------------------------------------------------------------------


def dot_spec_order(K: int) -> list:
    """The fixed summation order of a length-K dot product.

    32 partial sums; partial p takes, in increasing k, every element with
    (k // 8) % 32 == p.  The partials are then combined as p[j] += p[j + off]
    for off = 16, 8, 4, 2, 1 and the result is p[0].  Returns, per partial,
    the list of k it sums."""
    return [[k for k in range(K) if (k // 8) % 32 == p] for p in range(32)]


def dot_spec(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Batched fp64 dot products a[..., K] . b[..., K] in the dot_spec order.

    a and b broadcast against each other; each product of two bf16 or fp32
    values is exact in fp64, so only the order of the additions matters.
    K is padded with zero products to a multiple of 256 (adding an exact zero
    changes no partial sum), after which element k = 256*i + 8*p + r belongs to
    partial p and is added at step (i, r) in lexicographic order."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    K = a.shape[-1]
    Kp = -(-K // 256) * 256
    if Kp != K:
        a = np.concatenate([a, np.zeros(a.shape[:-1] + (Kp - K,))], axis=-1)
        b = np.concatenate([b, np.zeros(b.shape[:-1] + (Kp - K,))], axis=-1)
    a = a.reshape(a.shape[:-1] + (Kp // 256, 32, 8))
    b = b.reshape(b.shape[:-1] + (Kp // 256, 32, 8))
    shape = np.broadcast_shapes(a.shape[:-3], b.shape[:-3])
    part = np.zeros(shape + (32,), dtype=np.float64)
    for i in range(Kp // 256):
        for r in range(8):
            part = part + a[..., i, :, r] * b[..., i, :, r]
    for off in (16, 8, 4, 2, 1):
        part[..., :off] = part[..., :off] + part[..., off:2 * off]
    return part[..., 0]


def router_logits(x: np.ndarray, w_gate: np.ndarray) -> np.ndarray:
    """l[t, e] = fp32(dot_spec(x[t], W_gate[e]))  ->  float32 [T, E]."""
    return dot_spec(x[:, None, :], w_gate[None, :, :]).astype(np.float32)


# ---------------------------------------------------------------------------
# Sigmoid gating (section 5.3; section 5.6 step 2: s = sigmoid(l))
# ---------------------------------------------------------------------------

# Cody-Waite split of ln 2: LN2_HI carries 32 significant bits, so n*LN2_HI is
# exact for |n| < 2**20; LN2_LO = ln 2 - LN2_HI rounded to fp64.
LN2_HI = float.fromhex("0x1.62e42fee00000p-1")
LN2_LO = float.fromhex("0x1.a39ef35793c76p-33")
INV_LN2 = float.fromhex("0x1.71547652b82fep+0")
# Taylor coefficients 1/i! for i = 0..13, each rounded to fp64
EXP_TAYLOR = [1.0 / math.factorial(i) for i in range(14)]


def exp_spec(a: np.ndarray) -> np.ndarray:
    """exp(a) in fp64 for |a| <= 80 using only IEEE +, *, rint and ldexp.

    a = n*ln2 + r with n = rint(a/ln2), |r| <= ln2/2 (Cody-Waite, two-part ln2);
    exp(r) by Horner on the degree-13 Taylor polynomial (truncation error below
    1e-17 relative); exp(a) = 2**n * exp(r)."""
    a = np.asarray(a, dtype=np.float64)
    n = np.rint(a * INV_LN2)
    r = (a - n * LN2_HI) - n * LN2_LO
    p = np.full_like(a, EXP_TAYLOR[13])
    for c in EXP_TAYLOR[12::-1]:
        p = p * r + c
    return np.ldexp(p, n.astype(np.int64))


def sigmoid_spec(logits: np.ndarray) -> np.ndarray:
    """s = fp32(1 / (1 + exp_spec(-clamp(l, -80, 80)))) for fp32 logits."""
    a = -np.clip(np.asarray(logits, dtype=np.float64), -80.0, 80.0)
    return (1.0 / (1.0 + exp_spec(a))).astype(np.float32)


# ---------------------------------------------------------------------------
# Selection and weights (sections 5.4-5.5; section 5.6 steps 2-4)
# ---------------------------------------------------------------------------


def group_mask(choice: np.ndarray, n_group: int, topk_group: int) -> np.ndarray:
    """Section 5.5 group routing: score each of n_group equal groups by the sum
    of its two largest choice scores, keep the topk_group best groups (ties to
    the lower group index) and mask the experts of the others.  At n_group == 1
    every expert stays eligible.  Returns a bool mask [T, E]."""
    T, E = choice.shape
    if n_group == 1:
        return np.ones((T, E), dtype=bool)
    g = choice.reshape(T, n_group, E // n_group).astype(np.float64)
    top2 = -np.sort(-g, axis=-1)[..., :2]
    gscore = (top2[..., 0].astype(np.float32) + top2[..., 1].astype(np.float32))
    keep = np.zeros((T, n_group), dtype=bool)
    for t in range(T):
        order = sorted(range(n_group), key=lambda i: (-gscore[t, i], i))
        keep[t, order[:topk_group]] = True
    return np.repeat(keep, E // n_group, axis=1)


def select_topk(choice: np.ndarray, k: int, eligible=None) -> np.ndarray:
    """Indices of the k largest choice scores per row, ordered by (score
    descending, expert index ascending): ties go to the lower index.  -> int32."""
    T, E = choice.shape
    idx = np.empty((T, k), dtype=np.int32)
    for t in range(T):
        c = choice[t].astype(np.float64)
        if eligible is not None:
            c = np.where(eligible[t], c, -np.inf)
        order = np.lexsort((np.arange(E), -c))     # primary: -c, secondary: e
        idx[t] = order[:k]
    return idx


def route(logits: np.ndarray, bias: np.ndarray, k: int, rsf: float,
          n_group: int = 1, topk_group: int = 1, norm_topk_prob: bool = True):
    """Router from fp32 logits: returns (s, choice, topk_idx, topk_w).

    s = sigmoid(l); choice = s + bias (one fp32 add, used for selection only);
    topk over choice; the weights gather the raw s; when norm_topk_prob they are
    divided by (sum + 1e-20), the sum taken in fp32 in slot order; then scaled by
    routed_scaling_factor (normalise first, then scale)."""
    s = sigmoid_spec(logits)
    choice = (s + bias.astype(np.float32)).astype(np.float32)
    elig = group_mask(choice, n_group, topk_group)
    idx = select_topk(choice, k, None if n_group == 1 else elig)
    r = np.take_along_axis(s, idx.astype(np.int64), axis=1).astype(np.float32)
    if norm_topk_prob:
        S = np.zeros(r.shape[0], dtype=np.float32)
        for j in range(k):
            S = (S + r[:, j]).astype(np.float32)
        den = (S + np.float32(1e-20)).astype(np.float32)
        r = (r / den[:, None]).astype(np.float32)
    w = (r * np.float32(rsf)).astype(np.float32)
    return s, choice, idx, w


# ---------------------------------------------------------------------------
# Token -> expert bookkeeping (section 5.6 step 6: the expert mask and hit list),
# written as its plain definition: a stable grouping of the (token, slot) pairs.
# ---------------------------------------------------------------------------


def dispatch(topk_idx: np.ndarray, E: int):
    """counts[E], offsets[E+1] (exclusive prefix sum), perm[T*k] and pos[T, k].

    perm lists the pair ids t*k + j grouped by expert ascending, then token
    ascending; pos[t, j] is the position of pair (t, j) inside perm."""
    T, k = topk_idx.shape
    pairs = [(int(topk_idx[t, j]), t, j) for t in range(T) for j in range(k)]
    pairs.sort()
    counts = np.zeros(E, dtype=np.int32)
    for e, _, _ in pairs:
        counts[e] += 1
    offsets = np.zeros(E + 1, dtype=np.int32)
    for e in range(E):
        offsets[e + 1] = offsets[e] + counts[e]
    perm = np.array([t * k + j for _, t, j in pairs], dtype=np.int32)
    pos = np.empty((T, k), dtype=np.int32)
    for p, (_, t, j) in enumerate(pairs):
        pos[t, j] = p
    return counts, offsets, perm, pos


def max_violation(counts: np.ndarray) -> float:
    """MaxVio read as max expert load / mean expert load (512/22 = 23.27 is the
    value when one expert takes every token)."""
    return float(counts.max()) / float(counts.mean())


# ---------------------------------------------------------------------------
# NVFP4 (section 8.1; zhichai.net "NVFP4 format details"): E2M1 elements,
# 16-element micro-blocks along K, E4M3 block scales, FP32 global scale.
# ---------------------------------------------------------------------------


def e2m1_value(code: int) -> float:
    """Value of a 4-bit E2M1 code: sign bit 3, exponent bits 2-1, mantissa bit 0,
    exponent bias 1, exponent 0 is subnormal (0 or 0.5)."""
    sign = -1.0 if code & 8 else 1.0
    ex = (code >> 1) & 3
    m = code & 1
    mag = m * 0.5 if ex == 0 else (1.0 + 0.5 * m) * 2.0 ** (ex - 1)
    return sign * mag


def e4m3_value(code: int) -> float:
    """Value of an 8-bit E4M3 (fn) code: sign bit 7, exponent bits 6-3 (bias 7),
    mantissa bits 2-0; exponent 0 is subnormal; S.1111.111 is NaN; max 448."""
    sign = -1.0 if code & 0x80 else 1.0
    ex = (code >> 3) & 15
    m = code & 7
    if ex == 15 and m == 7:
        return float("nan")
    mag = (m / 8.0) * 2.0 ** -6 if ex == 0 else (1.0 + m / 8.0) * 2.0 ** (ex - 7)
    return sign * mag


E2M1_TABLE = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)
E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


def _rne_to_grid(x: float, codes, values, maxcode):
    """Round |x| to the nearest of the non-negative grid (codes, values),
    ties to the code whose lowest bit is 0; saturate above the largest."""
    ax = abs(x)
    if ax >= values[-1]:
        return maxcode
    best = None
    for c, v in zip(codes, values):
        d = abs(ax - v)
        if best is None or d < best[0] or (d == best[0] and (c & 1) == 0):
            best = (d, c)
    return best[1]


_E2M1_POS = list(range(8))
_E2M1_POS_V = [e2m1_value(c) for c in _E2M1_POS]
_E4M3_POS = list(range(0x7F))                   # 0 .. 448, NaN code excluded
_E4M3_POS_V = [e4m3_value(c) for c in _E4M3_POS]


def e2m1_encode(x: float) -> int:
    """fp value -> E2M1 code, round to nearest, ties to even, saturating at 6."""
    c = _rne_to_grid(x, _E2M1_POS, _E2M1_POS_V, 7)
    return c | 8 if (x < 0 and c != 0) else c


def e4m3_encode(x: float) -> int:
    """non-negative fp value -> E4M3 code, round to nearest even, saturating at
    448 (satfinite); subnormals kept."""
    assert x >= 0
    return _rne_to_grid(x, _E4M3_POS, _E4M3_POS_V, 0x7E)


def _rne_grid_vec(ax: np.ndarray, values: np.ndarray) -> np.ndarray:
    """Vector form of _rne_to_grid over non-negative ax and an ascending grid
    whose index is the code: nearest grid point, ties to the even code,
    saturating at the last point."""
    ax = np.asarray(ax, dtype=np.float64)
    hi = np.clip(np.searchsorted(values, ax, side="left"), 0, len(values) - 1)
    lo = np.clip(hi - 1, 0, len(values) - 1)
    dlo = np.abs(ax - values[lo])
    dhi = np.abs(values[hi] - ax)
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    return np.where(ax >= values[-1], len(values) - 1, code)


def e2m1_encode_vec(x: np.ndarray) -> np.ndarray:
    """Vector e2m1_encode -> uint8 codes.  The nearest point of the grid
    0, .5, 1, 1.5, 2, 3, 4, 6 with ties to the even code is the number of
    midpoints below |x|, where a midpoint counts when |x| passes it strictly if
    the code below it is even (.25, 1.25, 2.5, 5) and when |x| reaches it if the
    code above it is even (.75, 1.75, 3.5)."""
    x = np.asarray(x)
    a = np.abs(x)
    code = np.zeros(a.shape, dtype=np.uint8)
    for t in (0.25, 1.25, 2.5, 5.0):
        code += a > t
    for t in (0.75, 1.75, 3.5):
        code += a >= t
    code |= ((x < 0) & (code != 0)).astype(np.uint8) << 3
    return code


def e4m3_encode_vec(x: np.ndarray) -> np.ndarray:
    """Vector e4m3_encode over non-negative values -> uint8 codes."""
    return _rne_grid_vec(x, np.array(_E4M3_POS_V)).astype(np.uint8)


def nvfp4_global_scale(w: np.ndarray) -> np.float32:
    """Per-matrix FP32 second-level scale s_g = amax / (6 * 448), in fp32."""
    amax = np.float32(np.max(np.abs(np.asarray(w, dtype=np.float32))))
    return np.float32(amax / np.float32(6.0 * 448.0))


def nvfp4_quantize(w: np.ndarray, s_g) -> tuple:
    """Quantise w[rows, K] in 16-element blocks along K.

    Per block: s_b = E4M3(amax_b / (6 * s_g)); scale = value(s_b) * s_g;
    q_i = E2M1(w_i / scale) (0 when scale == 0).  All arithmetic before the
    encodings is fp32 (IEEE division).  A row whose length is not a multiple of
    16 ends in a partial block: it is quantised like a full block whose missing
    elements are zero (they change neither its maximum nor its other codes).
    Returns (codes uint8 [rows, K] one code per element, scales uint8
    [rows, ceil(K/16)])."""
    w = np.asarray(w, dtype=np.float32)
    rows, K = w.shape
    nb = -(-K // 16)
    if K % 16:
        w = np.concatenate([w, np.zeros((rows, nb * 16 - K), np.float32)], axis=1)
    blk = w.reshape(rows, nb, 16)
    amax = np.max(np.abs(blk), axis=-1).astype(np.float32)
    den = np.float32(np.float32(6.0) * np.float32(s_g))
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(den > 0, amax / den, np.float32(0)).astype(np.float32)
    sb = e4m3_encode_vec(ratio)
    scale = (E4M3_TABLE[sb].astype(np.float32) * np.float32(s_g)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        y = np.where(scale[..., None] > 0, blk / scale[..., None],
                     np.float32(0)).astype(np.float32)
    q = e2m1_encode_vec(y).reshape(rows, nb * 16)[:, :K]
    return q, sb


def nvfp4_dequantize(codes: np.ndarray, scales: np.ndarray, s_g) -> np.ndarray:
    """fp64 values q * value(s_b) * s_g (exact: each product fits in fp64);
    element k takes the scale of block k // 16."""
    rows, K = codes.shape
    blk_of_k = np.arange(K) // 16
    return E2M1_TABLE[codes] * E4M3_TABLE[scales][:, blk_of_k] * float(s_g)


def nvfp4_roundtrip_activation(a: np.ndarray, s_g=np.float32(1.0)) -> np.ndarray:
    """W4A4 activation path: round to fp32, quantise along the last axis with
    global scale s_g (1.0 unless the layer uses the tensor's own scale),
    dequantise (fp64)."""
    a32 = np.asarray(a, dtype=np.float32)
    q, sb = nvfp4_quantize(a32, s_g)
    return nvfp4_dequantize(q, sb, s_g)


def pack_e2m1(codes: np.ndarray) -> np.ndarray:
    """Two codes per byte along the last axis, the even element in the low nibble."""
    c = codes.astype(np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


# ---------------------------------------------------------------------------
# The layer (section 5.6 steps 1-7), fp64 with no intermediate rounding
# ---------------------------------------------------------------------------


def relu2(v: np.ndarray) -> np.ndarray:
    """Squared ReLU, max(v, 0)**2 (the non-gated activation of section 5.1)."""
    return np.square(np.maximum(v, 0.0))


def expert_weights_fp64(w: np.ndarray, fmt: str) -> np.ndarray:
    """The expert matrix the layer multiplies by: the stored values for dense
    experts, the NVFP4-dequantised values (per-matrix global scale) otherwise."""
    w = np.asarray(w, dtype=np.float64)
    if fmt == "dense":
        return w
    sg = nvfp4_global_scale(w)
    q, sb = nvfp4_quantize(w.astype(np.float32), sg)
    return nvfp4_dequantize(q, sb, sg)


def forward(x, w_gate, bias, w_fc1, w_fc2, w_su, w_sd, get_up, get_down, *,
            k, rsf, expert_fmt="dense", n_group=1, topk_group=1,
            norm_topk_prob=True, experts_prepared=False, act_scale="unit"):
    """One LatentMoE layer on token rows x[T, D].

    get_up(e) -> up_proj[e] [F, L] and get_down(e) -> down_proj[e] [L, F] return
    the stored (bf16 / fp32) expert weights; NVFP4 formats quantise them here.
    With experts_prepared they return instead what expert_weights_fp64 makes of
    the stored weights (a caller may compute those once and reuse them).
    W4A4 rounds the latent z with global scale 1.0 (act_scale "unit") or with
    the tensor's own, amax(z) / (6 * 448) over all of z in fp32 ("tensor"), and
    each expert's ReLU^2 activations with global scale 1.0.
    Returns a dict with out [T, D] fp64 and every routing intermediate."""
    x64 = np.asarray(x, dtype=np.float64)
    T = x64.shape[0]
    E = w_gate.shape[0]
    logits = router_logits(x64, np.asarray(w_gate, dtype=np.float64))  # step 1
    s, choice, idx, w = route(logits, np.asarray(bias, np.float32), k, rsf,
                              n_group, topk_group, norm_topk_prob)   # steps 2-4
    counts, offsets, perm, pos = dispatch(idx, E)
    z = x64 @ np.asarray(w_fc1, dtype=np.float64).T                   # step 5
    if expert_fmt == "w4a4":
        zg = nvfp4_global_scale(z) if act_scale == "tensor" else np.float32(1.0)
        z_in = nvfp4_roundtrip_activation(z, zg)
    else:
        z_in = z
    y = np.zeros((T, k, z.shape[1]), dtype=np.float64)                # step 6
    for e in np.nonzero(counts)[0]:
        tok, slot = np.nonzero(idx == e)
        if experts_prepared:
            up, down = get_up(int(e)), get_down(int(e))
        else:
            up = expert_weights_fp64(get_up(int(e)), expert_fmt)
            down = expert_weights_fp64(get_down(int(e)), expert_fmt)
        h = relu2(z_in[tok] @ up.T)
        if expert_fmt == "w4a4":
            h = nvfp4_roundtrip_activation(h)
        y[tok, slot] = h @ down.T
    zc = np.zeros_like(z)
    for j in range(k):                                 # weighted combine, slot order
        zc = zc + w[:, j:j + 1].astype(np.float64) * y[:, j]
    out = zc @ np.asarray(w_fc2, dtype=np.float64).T                  # step 7
    sh = relu2(x64 @ np.asarray(w_su, dtype=np.float64).T)
    out = out + sh @ np.asarray(w_sd, dtype=np.float64).T
    return dict(out=out, logits=logits, s=s, choice=choice, topk_idx=idx,
                topk_w=w, counts=counts, offsets=offsets, perm=perm, pos=pos,
                z=z)


# ---------------------------------------------------------------------------
# Block wrapper (report "Nemotron-3-Ultra architecture", the layer stack of
# NemotronHModel.forward: every NemotronHBlock applies a pre-norm RMSNorm,
# runs its mixer -- here the LatentMoE layer -- and adds the result to the
# residual stream).  The pages give neither the RMSNorm formula's rounding
# nor its epsilon: the norm is the textbook y = g * x / sqrt(mean(x^2) + eps)
# with eps a parameter, evaluated in fp64 in a defined order, and the mixer
# reads y rounded once to the layer's dtype.
# ---------------------------------------------------------------------------


def rmsnorm_spec(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """y[t] = (x[t] * r_t) * g, r_t = 1 / sqrt(dot_spec(x[t], x[t]) / D + eps),
    one IEEE fp64 rounding per operation (squares are exact); eps is taken as
    its fp32 value."""
    x64 = np.asarray(x, dtype=np.float64)
    g64 = np.asarray(g, dtype=np.float64)
    ss = dot_spec(x64, x64)
    r = 1.0 / np.sqrt(ss / np.float64(x64.shape[-1]) + np.float64(np.float32(eps)))
    return (x64 * r[..., None]) * g64


def round_fp64_to_bf16(y: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bf16 (8 significant bits), ties to the
    even significand, returned as float32 (exact).  With y = m * 2**e, m in
    [0.5, 1), the result is rint(m * 256) / 256 * 2**e: rint rounds half to
    even and every step is exact.  Values must be 0 or normal in bf16
    (|y| >= 2**-126), which holds for normalised activations."""
    y = np.asarray(y, dtype=np.float64)
    m, e = np.frexp(y)
    nz = y != 0
    assert np.all(np.abs(y[nz]) >= 2.0 ** -126), "bf16 subnormal range"
    return np.ldexp(np.rint(m * 256.0) / 256.0, e).astype(np.float32)


def block_forward(x, norm_weight, eps, *layer_args, dtype="bf16", **layer_kw):
    """out = x + layer(RMSNorm(x)): the layer (`forward`) reads the normalised
    rows rounded to `dtype` ("bf16" or "fp32"); returns forward's dict with
    out replaced by the block output and y_in = the rows the layer read."""
    y = rmsnorm_spec(x, norm_weight, eps)
    y_in = round_fp64_to_bf16(y) if dtype == "bf16" else y.astype(np.float32)
    r = forward(y_in, *layer_args, **layer_kw)
    r["layer_out"] = r["out"]
    r["out"] = np.asarray(x, dtype=np.float64) + r["out"]
    r["y_in"] = y_in
    return r


# ---------------------------------------------------------------------------
# Shapes and work (section 2.3.4 parameter list; section 3.1.3 MoE FLOPs)
# ---------------------------------------------------------------------------


def param_count(D, L, E, F, Fs) -> dict:
    """Per-layer parameter counts: gate, bias, fc1+fc2, routed experts, shared."""
    c = dict(gate=E * D, bias=E, latent=2 * D * L, experts=E * 2 * F * L,
             shared=2 * D * Fs)
    c["total"] = sum(c.values())
    return c


def flops_per_token(D, L, E, k, F, Fs) -> dict:
    """Multiply-add FLOPs (2 per MAC) per token of each part of the layer."""
    c = dict(gate=2 * D * E, fc1=2 * D * L, experts=k * 4 * L * F,
             fc2=2 * L * D, shared=4 * D * Fs)
    c["total"] = sum(c.values())
    return c
