"""Pins for the fp64 oracle: each checks it against something other than itself.

Every function takes an ``oracle.Oracle`` handle and raises AssertionError on a
mismatch.  tests/test_oracle_pins.py runs them on the committed oracle;
tests/test_oracle_mutants.py runs them on copies of the oracle with planted
mistakes and requires that each mistake trips at least one pin.

Kinds of pin used (none retypes the oracle's recurrence):
  * brute force: the unrolled O(T^2) sums of tests/ref_defs.py on tiny inputs;
  * closed forms: T = 1, the very-fast-decay limit, the no-decay case (causal
    linear attention as a masked matmul);
  * hand-worked examples with exact rational values (tests/golden/);
  * invariants: WKV-4 shift invariance in k and convex-hull bounds, WKV-6
    linearity in (v, s0) and head independence, split-sequence chaining;
  * head LayerNorm + SiLU gate: the two-channel closed form, SiLU at +-ln 3 (sigmoid 3/4
    and 1/4), shift/scale invariance and unit moments, affinity in the per-channel
    parameters, per-head parameter rows;
  * decay from its logit, w = exp(-exp(omega)): points with closed forms (ln ln 2 -> 1/2),
    inversion by numpy's logarithms, monotonicity and range, the slow-decay asymptote,
    and the -inf / +inf limits through the recurrence (no decay, instant forgetting);
  * WKV-6 backward: central finite differences of the pinned forward oracle, element by
    element on a tiny case and along random directions at head size 64; an exact hand-worked
    scalar example (tests/golden); the chain rule through the decay map against differences
    of the map and of the logit forward.
"""
import json
import os
from fractions import Fraction

import numpy as np

import ref_defs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = max(np.max(np.abs(b)), 1e-300)
    return float(np.max(np.abs(a - b)) / den)


def _wkv4_rand(rng, B, T, C, kshift=0.0):
    w = np.exp(rng.uniform(-3, 1, C))
    u = rng.normal(0, 0.5, C)
    k = rng.normal(0, 1, (B, T, C)) + kshift
    v = rng.normal(0, 1, (B, T, C))
    return w, u, k, v


def _wkv6_rand(rng, B, T, H, N, with_s0=True):
    sc = 1.0 / np.sqrt(N)
    r = rng.normal(0, 1, (B, T, H, N)) * sc
    k = rng.normal(0, 1, (B, T, H, N)) * sc
    v = rng.normal(0, 1, (B, T, H, N)) * sc
    om = rng.uniform(-6, -0.5, (H, N))[None, None] + 0.3 * rng.normal(0, 1, (B, T, H, N))
    w = np.exp(-np.exp(om))
    u = rng.normal(0, 0.5, (H, N))
    s0 = rng.normal(0, 0.1, (B, H, N, N)) if with_s0 else None
    return r, k, v, w, u, s0


def _state_num_den(sT):
    """WKV-4 (a, b, p) -> absolute numerator and denominator."""
    a, b, p = sT[:, 0], sT[:, 1], sT[:, 2]
    scale = np.where(np.isfinite(p), np.exp(np.where(np.isfinite(p), p, 0.0)), 0.0)
    return a * scale, b * scale


# ----------------------------------------------------------------------------- WKV-4

def pin_wkv4_bruteforce(O):
    rng = np.random.default_rng(11)
    for trial in range(4):
        B, T, C = 2, 12, 5
        w, u, k, v = _wkv4_rand(rng, B, T, C)
        y, sT = O.wkv4(w, u, k, v, want_state=True)
        y_ref, num_ref, den_ref = ref_defs.wkv4_sums(w, u, k, v)
        assert _rel(y, y_ref) < 1e-12, ("wkv4 brute force y", trial, _rel(y, y_ref))
        num, den = _state_num_den(sT)
        assert _rel(num, num_ref) < 1e-12 and _rel(den, den_ref) < 1e-12, "wkv4 brute force state"
    # with a carried-in state
    B, T, C = 2, 7, 4
    w, u, k, v = _wkv4_rand(rng, B, T, C)
    s0 = np.stack([rng.normal(0, 1, (B, C)), rng.uniform(0.5, 2.0, (B, C)),
                   rng.normal(0, 1, (B, C))], axis=1)
    y, sT = O.wkv4(w, u, k, v, s0=s0, want_state=True)
    y_ref, num_ref, den_ref = ref_defs.wkv4_sums(w, u, k, v, s0=s0)
    assert _rel(y, y_ref) < 1e-12, ("wkv4 brute force with s0", _rel(y, y_ref))
    num, den = _state_num_den(sT)
    assert _rel(num, num_ref) < 1e-12 and _rel(den, den_ref) < 1e-12, "wkv4 state with s0"


def pin_wkv4_T1(O):
    """T = 1 from an empty state: y = v exactly (the bonus term is alone)."""
    rng = np.random.default_rng(12)
    w, u, k, v = _wkv4_rand(rng, 3, 1, 9)
    y = O.wkv4(w, u, k, v)
    assert np.array_equal(y, v), "wkv4 T=1 must return v"


def pin_wkv4_fast_decay(O):
    """w -> inf: only the previous token survives, undecayed."""
    rng = np.random.default_rng(13)
    B, T, C = 2, 9, 6
    _, u, k, v = _wkv4_rand(rng, B, T, C)
    w = np.full(C, 1000.0)  # e^{-1000} == 0 in fp64
    y = O.wkv4(w, u, k, v)
    ek_prev = np.exp(k[:, :-1])
    ebon = np.exp(u + k[:, 1:])
    expect = (ek_prev * v[:, :-1] + ebon * v[:, 1:]) / (ek_prev + ebon)
    assert _rel(y[:, 1:], expect) < 1e-13, ("wkv4 fast decay", _rel(y[:, 1:], expect))
    assert np.array_equal(y[:, 0], v[:, 0])


def pin_wkv4_invariants(O):
    rng = np.random.default_rng(14)
    B, T, C = 2, 40, 6
    w, u, k, v = _wkv4_rand(rng, B, T, C)
    y = O.wkv4(w, u, k, v)
    # k -> k + c leaves y unchanged (c = 60 would overflow a naive evaluation)
    y_shift = O.wkv4(w, u, k + 60.0, v)
    assert _rel(y_shift, y) < 1e-12, "wkv4 shift invariance"
    # y_t is a convex combination of v_0..v_t
    lo = np.minimum.accumulate(v, axis=1)
    hi = np.maximum.accumulate(v, axis=1)
    assert np.all(y >= lo - 1e-12) and np.all(y <= hi + 1e-12), "wkv4 convex hull"
    # constant v gives constant y
    vc = np.broadcast_to(rng.normal(0, 1, (B, 1, C)), (B, T, C))
    yc = O.wkv4(w, u, k, vc)
    assert _rel(yc, vc) < 1e-14, "wkv4 constant v"


def pin_wkv4_chaining(O):
    rng = np.random.default_rng(15)
    B, T, C = 2, 30, 5
    w, u, k, v = _wkv4_rand(rng, B, T, C)
    y, sT = O.wkv4(w, u, k, v, want_state=True)
    for cut in (1, 13, 29):
        y1, s1 = O.wkv4(w, u, k[:, :cut], v[:, :cut], want_state=True)
        y2, s2 = O.wkv4(w, u, k[:, cut:], v[:, cut:], s0=s1, want_state=True)
        assert _rel(np.concatenate([y1, y2], 1), y) < 1e-13, ("wkv4 chaining", cut)
        n_a, d_a = _state_num_den(s2)
        n_b, d_b = _state_num_den(sT)
        assert _rel(n_a, n_b) < 1e-13 and _rel(d_a, d_b) < 1e-13


def pin_wkv4_golden(O):
    with open(os.path.join(GOLDEN, "wkv4_hand_example.json")) as f:
        g = json.load(f)
    w = np.array([np.log(float(Fraction(g["decay_factor"]))) * -1.0])
    u = np.array([np.log(float(Fraction(g["exp_u"])))])
    k = np.log(np.array([float(Fraction(x)) for x in g["exp_k"]]))[None, :, None]
    v = np.array([float(Fraction(x)) for x in g["v"]])[None, :, None]
    y, sT = O.wkv4(w, u, k, v, want_state=True)
    expect = np.array([float(Fraction(x)) for x in g["y"]])
    assert _rel(y[0, :, 0], expect) < 1e-14, ("wkv4 golden", y[0, :, 0], expect)
    num, den = _state_num_den(sT)
    assert abs(num[0, 0] - float(Fraction(g["final_num"]))) < 1e-13
    assert abs(den[0, 0] - float(Fraction(g["final_den"]))) < 1e-13


# ----------------------------------------------------------------------------- WKV-6

def pin_wkv6_bruteforce(O):
    rng = np.random.default_rng(21)
    for (B, T, H, N, with_s0) in [(2, 8, 2, 1, True), (1, 7, 2, 2, False), (2, 6, 1, 4, True),
                                  (1, 3, 1, 64, True), (1, 5, 2, 4, False)]:
        r, k, v, w, u, s0 = _wkv6_rand(rng, B, T, H, N, with_s0)
        y, sT = O.wkv6(r, k, v, w, u, s0=s0)
        y_ref, sT_ref = ref_defs.wkv6_def(r, k, v, w, u, s0=s0)
        assert _rel(y, y_ref) < 1e-12, ("wkv6 brute force y", (B, T, H, N), _rel(y, y_ref))
        assert _rel(sT, sT_ref) < 1e-12, ("wkv6 brute force sT", (B, T, H, N))


def pin_wkv6_T1(O):
    """T = 1: o = r (s0 + diag(u) k^T v), sT = diag(w) s0 + k^T v; s0 = 0 gives o = (r.(u*k)) v."""
    rng = np.random.default_rng(22)
    B, H, N = 2, 3, 8
    r, k, v, w, u, s0 = _wkv6_rand(rng, B, 1, H, N, True)
    y, sT = O.wkv6(r, k, v, w, u, s0=None)
    for b in range(B):
        for h in range(H):
            rr, kk, vv = r[b, 0, h], k[b, 0, h], v[b, 0, h]
            assert _rel(y[b, 0, h], np.dot(rr, u[h] * kk) * vv) < 1e-13, "wkv6 T1 zero state y"
            assert _rel(sT[b, h], np.outer(kk, vv)) < 1e-14, "wkv6 T1 zero state sT"
    y, sT = O.wkv6(r, k, v, w, u, s0=s0)
    for b in range(B):
        for h in range(H):
            rr, kk, vv, ww = r[b, 0, h], k[b, 0, h], v[b, 0, h], w[b, 0, h]
            o = rr @ (s0[b, h] + np.outer(u[h] * kk, vv))
            assert _rel(y[b, 0, h], o) < 1e-13, "wkv6 T1 with state y"
            assert _rel(sT[b, h], ww[:, None] * s0[b, h] + np.outer(kk, vv)) < 1e-14


def pin_wkv6_fast_decay(O):
    """w = 0: o_t = (r_t.k_{t-1}) v_{t-1} + (r_t.(u*k_t)) v_t; sT = k_{T-1}^T v_{T-1}."""
    rng = np.random.default_rng(23)
    B, T, H, N = 2, 6, 2, 8
    r, k, v, w, u, s0 = _wkv6_rand(rng, B, T, H, N, True)
    w = np.zeros_like(w)
    y, sT = O.wkv6(r, k, v, w, u, s0=s0)
    for t in range(1, T):
        expect = (np.einsum("bhi,bhi->bh", r[:, t], k[:, t - 1])[..., None] * v[:, t - 1]
                  + np.einsum("bhi,hi,bhi->bh", r[:, t], u, k[:, t])[..., None] * v[:, t])
        assert _rel(y[:, t], expect) < 1e-13, ("wkv6 fast decay", t)
    assert _rel(sT, np.einsum("bhi,bhj->bhij", k[:, -1], v[:, -1])) < 1e-14


def pin_wkv6_no_decay(O):
    """w = 1 reduces to causal linear attention with a bonus diagonal (masked matmul)."""
    rng = np.random.default_rng(24)
    B, T, H, N = 1, 12, 2, 16
    r, k, v, w, u, s0 = _wkv6_rand(rng, B, T, H, N, True)
    w = np.ones_like(w)
    y, sT = O.wkv6(r, k, v, w, u, s0=s0)
    for h in range(H):
        o_ref, s_ref = ref_defs.causal_linear_attention(r[0, :, h], k[0, :, h], v[0, :, h],
                                                       u[h], s0[0, h])
        assert _rel(y[0, :, h], o_ref) < 1e-12, "wkv6 no decay y"
        assert _rel(sT[0, h], s_ref) < 1e-12, "wkv6 no decay sT"


def pin_wkv6_chaining(O):
    rng = np.random.default_rng(25)
    B, T, H, N = 2, 24, 2, 8
    r, k, v, w, u, s0 = _wkv6_rand(rng, B, T, H, N, True)
    y, sT = O.wkv6(r, k, v, w, u, s0=s0)
    for cut in (1, 10, 23):
        sl1, sl2 = slice(0, cut), slice(cut, T)
        y1, s1 = O.wkv6(r[:, sl1], k[:, sl1], v[:, sl1], w[:, sl1], u, s0=s0)
        y2, s2 = O.wkv6(r[:, sl2], k[:, sl2], v[:, sl2], w[:, sl2], u, s0=s1)
        assert _rel(np.concatenate([y1, y2], 1), y) < 1e-13, ("wkv6 chaining", cut)
        assert _rel(s2, sT) < 1e-13


def pin_wkv6_linearity(O):
    """(y, sT) is linear in (v, s0) jointly."""
    rng = np.random.default_rng(26)
    B, T, H, N = 1, 10, 2, 8
    r, k, v1, w, u, s01 = _wkv6_rand(rng, B, T, H, N, True)
    _, _, v2, _, _, s02 = _wkv6_rand(rng, B, T, H, N, True)
    a, b = 0.7, -1.3
    y1, t1 = O.wkv6(r, k, v1, w, u, s0=s01)
    y2, t2 = O.wkv6(r, k, v2, w, u, s0=s02)
    y3, t3 = O.wkv6(r, k, a * v1 + b * v2, w, u, s0=a * s01 + b * s02)
    assert _rel(y3, a * y1 + b * y2) < 1e-12 and _rel(t3, a * t1 + b * t2) < 1e-12


def pin_wkv6_head_independence(O):
    """Permuting heads (with their u) permutes outputs; batch rows are independent."""
    rng = np.random.default_rng(27)
    B, T, H, N = 2, 7, 3, 4
    r, k, v, w, u, s0 = _wkv6_rand(rng, B, T, H, N, True)
    y, sT = O.wkv6(r, k, v, w, u, s0=s0)
    perm = np.array([2, 0, 1])
    yp, sTp = O.wkv6(r[:, :, perm], k[:, :, perm], v[:, :, perm], w[:, :, perm], u[perm],
                     s0=s0[:, perm])
    assert _rel(yp, y[:, :, perm]) < 1e-15 and _rel(sTp, sT[:, perm]) < 1e-15
    y1, s1 = O.wkv6(r[1:], k[1:], v[1:], w[1:], u, s0=s0[1:])
    assert _rel(y1, y[1:]) < 1e-15 and _rel(s1, sT[1:]) < 1e-15


def pin_wkv6_golden(O):
    with open(os.path.join(GOLDEN, "wkv6_hand_example.json")) as f:
        g = json.load(f)
    conv = lambda x: np.array(x, dtype=object).astype(float)  # noqa: E731
    r = conv(g["r"])[None, :, None, :]
    k = conv(g["k"])[None, :, None, :]
    v = conv(g["v"])[None, :, None, :]
    w = np.array([[float(Fraction(x)) for x in row] for row in g["w"]])[None, :, None, :]
    u = conv(g["u"])[None, :]
    s0 = conv(g["s0"])[None, None]
    y, sT = O.wkv6(r, k, v, w, u, s0=s0)
    y_exp = np.array([[float(Fraction(x)) for x in row] for row in g["y"]])
    s_exp = np.array([[float(Fraction(x)) for x in row] for row in g["sT"]])
    assert np.array_equal(y[0, :, 0, :], y_exp), ("wkv6 golden y", y[0, :, 0, :], y_exp)
    assert np.array_equal(sT[0, 0], s_exp), ("wkv6 golden sT", sT[0, 0], s_exp)


# ----------------------------------------------------------- head LayerNorm + SiLU gate
# SiLU at two points with closed forms: sigma(ln 3) = 3/4, sigma(-ln 3) = 1/4.
_LN3 = float(np.log(3.0))
_SILU_LN3, _SILU_MLN3 = 0.75 * _LN3, -0.25 * _LN3


def pin_norm_gate_two_channels(O):
    """N = 2: the deviations from the mean are +-d with d = (a - b) / 2, so the normalised
    pair is +-d / sqrt(d^2 + eps) -- exactly +-1 for eps = 0."""
    rng = np.random.default_rng(41)
    B, T, H, N = 2, 3, 2, 2
    o = rng.normal(0, 2, (B, T, H, N))
    g = np.empty_like(o)
    g[..., 0], g[..., 1] = _LN3, -_LN3
    gam = rng.uniform(0.5, 2, (H, N))
    bet = rng.normal(0, 1, (H, N))
    for eps in (0.0, 0.3):
        y = O.head_norm_gate(o, g, gam, bet, eps)
        d = (o[..., 0] - o[..., 1]) / 2
        xh0 = d / np.sqrt(d * d + eps)
        exp0 = _SILU_LN3 * (gam[None, None, :, 0] * xh0 + bet[None, None, :, 0])
        exp1 = _SILU_MLN3 * (gam[None, None, :, 1] * -xh0 + bet[None, None, :, 1])
        assert _rel(y[..., 0], exp0) < 1e-12 and _rel(y[..., 1], exp1) < 1e-12, ("two-channel closed form", eps)


def pin_norm_gate_invariants(O):
    """eps = 0: the normalised part is unchanged by a per-row shift or positive scale of o,
    and has zero mean and unit mean square over the head's channels."""
    rng = np.random.default_rng(42)
    B, T, H, N = 2, 4, 3, 8
    o = rng.normal(0, 1, (B, T, H, N))
    g = np.full_like(o, _LN3)
    one, zero = np.ones((H, N)), np.zeros((H, N))
    y = O.head_norm_gate(o, g, one, zero, 0.0)
    xh = y / _SILU_LN3
    assert np.max(np.abs(xh.mean(-1))) < 1e-12, "normalised mean"
    assert np.max(np.abs((xh * xh).mean(-1) - 1.0)) < 1e-12, "normalised mean square"
    shift = rng.normal(0, 5, (B, T, H, 1))
    scale = rng.uniform(0.1, 10, (B, T, H, 1))
    assert _rel(O.head_norm_gate(o + shift, g, one, zero, 0.0), y) < 1e-10, "shift invariance"
    assert _rel(O.head_norm_gate(o * scale, g, one, zero, 0.0), y) < 1e-10, "scale invariance"


def pin_norm_gate_affine(O):
    """Linear in (ln_w, ln_b): y(w, b) = y(w, 0) + y(0, b), and y(0, b) = SiLU(g) * b."""
    rng = np.random.default_rng(43)
    B, T, H, N = 1, 3, 2, 8
    o = rng.normal(0, 1, (B, T, H, N))
    g = np.where(rng.uniform(size=o.shape) < 0.5, _LN3, -_LN3)
    silu = np.where(g > 0, _SILU_LN3, _SILU_MLN3)
    gam = rng.normal(0, 1, (H, N))
    bet = rng.normal(0, 1, (H, N))
    zero = np.zeros((H, N))
    y = O.head_norm_gate(o, g, gam, bet, 1e-3)
    yw = O.head_norm_gate(o, g, gam, zero, 1e-3)
    yb = O.head_norm_gate(o, g, zero, bet, 1e-3)
    assert _rel(y, yw + yb) < 1e-12, "additivity in (w, b)"
    assert _rel(yb, silu * bet[None, None]) < 1e-12, "shift term is SiLU(g) * b"


def pin_norm_gate_heads(O):
    """Each head uses its own row of (ln_w, ln_b): permuting the heads of o and g together
    with those rows permutes y."""
    rng = np.random.default_rng(44)
    B, T, H, N = 2, 2, 4, 8
    o = rng.normal(0, 1, (B, T, H, N))
    g = rng.normal(0, 2, (B, T, H, N))
    gam = rng.normal(0, 1, (H, N))
    bet = rng.normal(0, 1, (H, N))
    perm = np.array([2, 0, 3, 1])
    y = O.head_norm_gate(o, g, gam, bet, 1e-5)
    yp = O.head_norm_gate(o[:, :, perm], g[:, :, perm], gam[perm], bet[perm], 1e-5)
    assert _rel(yp, y[:, :, perm]) < 1e-12, "per-head parameters"


# ------------------------------------------------------------ decay from its logit omega
def pin_logit_closed_forms(O):
    """w = exp(-exp(omega)): omega = ln ln 2 gives 1/2, ln ln 4 gives 1/4, 0 gives 1/e,
    ln 3 gives e^-3; the limits -inf and +inf give 1 and 0."""
    om = np.array([np.log(np.log(2.0)), np.log(np.log(4.0)), 0.0, np.log(3.0), -np.inf, np.inf])
    w = O.decay_from_logit(om)
    expect = np.array([0.5, 0.25, np.exp(-1.0), np.exp(-3.0), 1.0, 0.0])
    assert np.max(np.abs(w - expect)) < 1e-15, ("logit closed forms", w)


def pin_logit_inverse_and_shape(O):
    """omega = ln(-ln w) inverts the map (numpy's logarithms, not the map), the map keeps
    the array's shape, is strictly decreasing and stays in (0, 1); for omega << 0,
    -ln w = e^omega, i.e. the decay distance 1 - w is about e^omega."""
    rng = np.random.default_rng(45)
    w_true = rng.uniform(1e-6, 1 - 1e-9, (3, 5, 2, 4))
    w = O.decay_from_logit(np.log(-np.log(w_true)))
    assert w.shape == w_true.shape, "shape"
    assert np.max(np.abs(w - w_true) / w_true) < 1e-13, "inverse"
    om = np.linspace(-30.0, 3.0, 331)
    ws = O.decay_from_logit(om)
    assert np.all(np.diff(ws) < 0) and np.all((ws > 0) & (ws < 1)), "monotone, in (0, 1)"
    small = np.array([-12.0, -16.0, -20.0])
    assert _rel(-np.log(O.decay_from_logit(small)), np.exp(small)) < 1e-6, "slow-decay asymptote"


def pin_wkv6_logit_limits(O):
    """Through the WKV-6 recurrence: omega = -inf everywhere is the no-decay case (causal
    linear attention, masked matmul); omega = +inf is the instant-forget case,
    o_t = (r_t.k_{t-1}) v_{t-1} + (r_t.(u*k_t)) v_t; omega = ln ln 2 halves the state."""
    rng = np.random.default_rng(46)
    B, T, H, N = 1, 10, 2, 8
    r, k, v, w, u, s0 = _wkv6_rand(rng, B, T, H, N, True)
    y, sT = O.wkv6_logit(r, k, v, np.full_like(w, -np.inf), u, s0=s0)
    for h in range(H):
        o_ref, s_ref = ref_defs.causal_linear_attention(r[0, :, h], k[0, :, h], v[0, :, h],
                                                       u[h], s0[0, h])
        assert _rel(y[0, :, h], o_ref) < 1e-12 and _rel(sT[0, h], s_ref) < 1e-12, "logit no decay"
    y, sT = O.wkv6_logit(r, k, v, np.full_like(w, np.inf), u, s0=s0)
    for t in range(1, T):
        expect = (np.einsum("bhi,bhi->bh", r[:, t], k[:, t - 1])[..., None] * v[:, t - 1]
                  + np.einsum("bhi,hi,bhi->bh", r[:, t], u, k[:, t])[..., None] * v[:, t])
        assert _rel(y[:, t], expect) < 1e-13, ("logit instant forget", t)
    # T = 1 with w = 1/2 on every channel: sT = s0 / 2 + k^T v
    r1, k1, v1 = r[:, :1], k[:, :1], v[:, :1]
    _, sT = O.wkv6_logit(r1, k1, v1, np.full_like(r1, np.log(np.log(2.0))), u, s0=s0)
    assert _rel(sT, 0.5 * s0 + np.einsum("bhi,bhj->bhij", k1[:, 0], v1[:, 0])) < 1e-14, "logit halving"


# ------------------------------------------------------------------- WKV-6 backward
# The backward is pinned against central finite differences of the (separately pinned)
# forward oracle: L = sum(dy * y) + sum(dsT * sT), so dL/dx is what the backward returns.
def _wkv6_loss(O, r, k, v, w, u, s0, dy, dsT):
    y, sT = O.wkv6(r, k, v, w, u, s0=s0)
    return float(np.sum(dy * y) + np.sum(dsT * sT))


def pin_wkv6_backward_fd_elementwise(O):
    """Every element of every input of a tiny case against its central difference."""
    rng = np.random.default_rng(47)
    B, T, H, N = 2, 4, 2, 3
    r, k, v, w, u, s0 = _wkv6_rand(rng, B, T, H, N, True)
    dy = rng.normal(0, 1, r.shape)
    dsT = rng.normal(0, 1, s0.shape)
    g = O.wkv6_backward(r, k, v, w, u, dy, s0=s0, dsT=dsT)
    args = {"r": r, "k": k, "v": v, "w": w, "u": u, "s0": s0}
    h = 1e-6
    for name, grad in (("r", "dr"), ("k", "dk"), ("v", "dv"), ("w", "dw"), ("u", "du"), ("s0", "ds0")):
        x = args[name]
        fd = np.empty_like(x)
        for idx in np.ndindex(x.shape):
            a = dict(args)
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            a[name] = xp
            lp = _wkv6_loss(O, **a, dy=dy, dsT=dsT)
            a[name] = xm
            lm = _wkv6_loss(O, **a, dy=dy, dsT=dsT)
            fd[idx] = (lp - lm) / (2 * h)
        assert _rel(g[grad], fd) < 1e-6, ("backward vs finite differences", name, _rel(g[grad], fd))


def pin_wkv6_backward_fd_directional(O):
    """Head size 64, no initial state, no state gradient: directional derivatives along a
    random direction per input."""
    rng = np.random.default_rng(48)
    B, T, H, N = 1, 5, 2, 64
    r, k, v, w, u, _ = _wkv6_rand(rng, B, T, H, N, False)
    s0 = np.zeros((B, H, N, N))
    dy = rng.normal(0, 1, r.shape)
    dsT = np.zeros_like(s0)
    g = O.wkv6_backward(r, k, v, w, u, dy)
    args = {"r": r, "k": k, "v": v, "w": w, "u": u, "s0": s0}
    h = 1e-5
    for name, grad in (("r", "dr"), ("k", "dk"), ("v", "dv"), ("w", "dw"), ("u", "du"), ("s0", "ds0")):
        d = rng.normal(0, 1, args[name].shape)
        a = dict(args)
        a[name] = args[name] + h * d
        lp = _wkv6_loss(O, **a, dy=dy, dsT=dsT)
        a[name] = args[name] - h * d
        lm = _wkv6_loss(O, **a, dy=dy, dsT=dsT)
        fd = (lp - lm) / (2 * h)
        an = float(np.sum(g[grad] * d))
        assert abs(an - fd) <= 1e-7 * max(1.0, abs(fd)), ("directional derivative", name, an, fd)


def pin_wkv6_backward_golden(O):
    """Exact hand-worked gradients of a scalar two-token case (tests/golden), derived from the
    loss written out as a polynomial; every value is dyadic, so fp64 must match exactly."""
    with open(os.path.join(GOLDEN, "wkv6_backward_hand_example.json")) as f:
        g = json.load(f)
    q = lambda x: float(Fraction(str(x)))  # noqa: E731
    seq = lambda xs: np.array([q(x) for x in xs]).reshape(1, 2, 1, 1)  # noqa: E731
    out = O.wkv6_backward(seq(g["r"]), seq(g["k"]), seq(g["v"]), seq(g["w"]), np.array([[q(g["u"])]]),
                          seq(g["dy"]), s0=np.array([[[[q(g["s0"])]]]]), dsT=np.array([[[[q(g["dsT"])]]]]))
    for name in ("dr", "dk", "dv", "dw"):
        assert np.array_equal(out[name].reshape(2), np.array([q(x) for x in g[name]])), ("backward golden", name)
    assert out["du"].reshape(()) == q(g["du"]), ("backward golden du", out["du"])
    assert out["ds0"].reshape(()) == q(g["ds0"]), ("backward golden ds0", out["ds0"])


def pin_logit_backward_fd(O):
    """The chain rule through w = exp(-exp(omega)): elementwise against central differences
    of the map, and through the recurrence against differences of wkv6_logit."""
    om = np.linspace(-8.0, 3.0, 45)
    h = 1e-6
    fd = (O.decay_from_logit(om + h) - O.decay_from_logit(om - h)) / (2 * h)
    dw = np.linspace(-2.0, 2.0, 45)
    assert _rel(O.decay_from_logit_grad(om, dw), dw * fd) < 1e-7, "map derivative"
    rng = np.random.default_rng(49)
    B, T, H, N = 1, 3, 1, 4
    r, k, v, w, u, s0 = _wkv6_rand(rng, B, T, H, N, True)
    omega = rng.uniform(-3.0, 1.0, r.shape)
    dy = rng.normal(0, 1, r.shape)
    g = O.wkv6_logit_backward(r, k, v, omega, u, dy, s0=s0)
    fd = np.empty_like(omega)
    for idx in np.ndindex(omega.shape):
        op, omm = omega.copy(), omega.copy()
        op[idx] += h
        omm[idx] -= h
        yp, _ = O.wkv6_logit(r, k, v, op, u, s0=s0)
        ym, _ = O.wkv6_logit(r, k, v, omm, u, s0=s0)
        fd[idx] = np.sum(dy * (yp - ym)) / (2 * h)
    assert _rel(g["domega"], fd) < 1e-6, ("logit backward", _rel(g["domega"], fd))


ALL_PINS = [
    pin_wkv4_bruteforce, pin_wkv4_T1, pin_wkv4_fast_decay, pin_wkv4_invariants,
    pin_wkv4_chaining, pin_wkv4_golden,
    pin_wkv6_bruteforce, pin_wkv6_T1, pin_wkv6_fast_decay, pin_wkv6_no_decay,
    pin_wkv6_chaining, pin_wkv6_linearity, pin_wkv6_head_independence, pin_wkv6_golden,
    pin_norm_gate_two_channels, pin_norm_gate_invariants, pin_norm_gate_affine, pin_norm_gate_heads,
    pin_logit_closed_forms, pin_logit_inverse_and_shape, pin_wkv6_logit_limits,
    pin_wkv6_backward_fd_elementwise, pin_wkv6_backward_fd_directional, pin_wkv6_backward_golden,
    pin_logit_backward_fd,
]


def failing_pins(O):
    """Names of the pins that fail (any exception counts) on oracle handle O."""
    bad = []
    for p in ALL_PINS:
        try:
            with np.errstate(all="ignore"):
                p(O)
        except Exception:  # noqa: BLE001 -- a crash in a mutant is a caught mistake too
            bad.append(p.__name__)
    return bad
