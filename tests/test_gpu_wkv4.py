"""GPU parity of the RWKV-4 WKV scan kernel against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import TOL, dev, f64, rel_inf, wkv4_state_views
from wkv_recurrence_02_b200 import inputs, ops

pytestmark = pytest.mark.gpu


def _run(B, T, C, dtype="fp32", seed=0, wu_seed=None, kshift=0.0):
    x = inputs.wkv4_inputs(B, T, C, dtype, seed=seed, wu_seed=wu_seed)
    k = x["k"]
    if kshift:
        k = (k.float() + kshift).to(k.dtype)
    y = ops.wkv4_forward(dev(x["w"]), dev(x["u"]), dev(k), dev(x["v"]))
    torch.cuda.synchronize()
    ref = oracle.wkv4(f64(x["w"]), f64(x["u"]), f64(k), f64(x["v"]))
    return rel_inf(f64(y), ref), y.dtype


def test_wkv4_small_fp32_workload():
    """B=1, T=64, C=128 fp32, seed 0: full comparison."""
    err, dt = _run(1, 64, 128, "fp32", seed=0)
    assert err <= TOL[dt], err


def test_wkv4_169m_all_layers_bf16():
    """B=8, T=1024, C=768 bf16; k,v seed 0, layer l's w,u seed l+1, all 12 layers in full."""
    kv = inputs.wkv4_kv(8, 1024, 768, 0, "bf16")
    kd, vd = dev(kv[0]), dev(kv[1])
    kf, vf = f64(kv[0]), f64(kv[1])
    for layer in range(12):
        w, u = inputs.wkv4_wu(768, layer + 1)
        y = ops.wkv4_forward(dev(w), dev(u), kd, vd)
        torch.cuda.synchronize()
        err = rel_inf(f64(y), oracle.wkv4(f64(w), f64(u), kf, vf))
        assert err <= TOL[torch.bfloat16], (layer, err)


@pytest.mark.parametrize("B,T,C", [(1, 1, 16), (2, 5, 16), (3, 33, 48), (2, 1000, 40),
                                   (1, 2049, 24), (2, 300, 37), (1, 4097, 8), (4, 64, 1)])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_wkv4_ragged_shapes(B, T, C, dtype):
    err, dt = _run(B, T, C, dtype, seed=B * 1000 + T + C)
    assert err <= TOL[dt], err


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_wkv4_large_keys_stay_stable(dtype):
    """k ~ N(60, 1): a naive exp(k) would overflow fp32; the running maximum must not."""
    err, dt = _run(2, 700, 64, dtype, seed=5, kshift=60.0)
    assert err <= TOL[dt], err


def test_wkv4_T1_returns_v():
    """T = 1 from an empty state: y = v (the bonus term alone), to fp32 rounding."""
    x = inputs.wkv4_inputs(3, 1, 64, "fp32", seed=9)
    y = ops.wkv4_forward(dev(x["w"]), dev(x["u"]), dev(x["k"]), dev(x["v"]))
    assert rel_inf(f64(y), f64(x["v"])) <= 1e-6


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_wkv4_state_chaining(dtype):
    """One call over T equals calls over pieces of T with the (a,b,p) state carried."""
    B, T, C = 2, 1500, 48
    x = inputs.wkv4_inputs(B, T, C, dtype, seed=3)
    w, u, k, v = dev(x["w"]), dev(x["u"]), dev(x["k"]), dev(x["v"])
    y_full, s_full = ops.wkv4_forward(w, u, k, v, want_state=True)
    pieces, s = [], None
    for lo, hi in [(0, 1), (1, 700), (700, 1033), (1033, T)]:
        yp, s = ops.wkv4_forward(w, u, k[:, lo:hi].contiguous(), v[:, lo:hi].contiguous(),
                                 s0=s, want_state=True)
        pieces.append(yp)
    y_chain = torch.cat(pieces, 1)
    torch.cuda.synchronize()
    ref_y, ref_s = oracle.wkv4(f64(x["w"]), f64(x["u"]), f64(x["k"]), f64(x["v"]),
                               want_state=True)
    tol = TOL[k.dtype]
    assert rel_inf(f64(y_full), ref_y) <= tol
    assert rel_inf(f64(y_chain), ref_y) <= tol
    for got in (f64(s_full), f64(s)):
        ga, gb = wkv4_state_views(got)
        ra, rb = wkv4_state_views(ref_s)
        assert rel_inf(ga, ra) <= 1e-4 and np.max(np.abs(gb - rb)) <= 1e-3


def test_wkv4_state_in_place_and_T0():
    B, T, C = 2, 100, 32
    x = inputs.wkv4_inputs(B, T, C, "fp32", seed=4)
    w, u, k, v = dev(x["w"]), dev(x["u"]), dev(x["k"]), dev(x["v"])
    _, s = ops.wkv4_forward(w, u, k[:, :50].contiguous(), v[:, :50].contiguous(), want_state=True)
    s_copy = s.clone()
    # T == 0: the state passes through unchanged
    y0, s0out = ops.wkv4_forward(w, u, k[:, :0].contiguous(), v[:, :0].contiguous(), s0=s,
                                 want_state=True)
    torch.cuda.synchronize()
    assert y0.numel() == 0 and torch.equal(s0out, s_copy)
    # in place: s0 and sT the same buffer
    y2, s2 = ops.wkv4_forward(w, u, k[:, 50:].contiguous(), v[:, 50:].contiguous(), s0=s, sT=s,
                              want_state=True)
    torch.cuda.synchronize()
    ref_y = oracle.wkv4(f64(x["w"]), f64(x["u"]), f64(x["k"]), f64(x["v"]))
    assert rel_inf(f64(y2), ref_y[:, 50:]) <= 1e-4
    assert s2.data_ptr() == s.data_ptr()


def test_wkv4_deterministic():
    x = inputs.wkv4_inputs(8, 1024, 768, "bf16", seed=0, wu_seed=1)
    args = [dev(x[n]) for n in ("w", "u", "k", "v")]
    a = ops.wkv4_forward(*args)
    b = ops.wkv4_forward(*args)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


# Several tiles (the carry between them), a last tile holding one segment, 16-byte rows.
@pytest.mark.parametrize("B,T,C", [(2, 2048, 64), (1, 1056, 32), (2, 4096, 16), (3, 64, 40), (1, 1024, 8)])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_wkv4_tile_shapes(B, T, C, dtype):
    err, dt = _run(B, T, C, dtype, seed=B * 7 + T + C)
    assert err <= TOL[dt], err


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_wkv4_spread_keys_take_the_exact_paths(dtype):
    """Keys shifted per token by N(60, 30^2): the fixed-frame and last-key shortcuts give way
    to the running-maximum steps for most segments, and pass-1 summaries whose denominator
    reaches 2^100 and more must still combine by their true magnitude."""
    x = inputs.wkv4_inputs(2, 1024, 48, dtype, seed=11)
    g = torch.Generator().manual_seed(12)
    k = (x["k"].float() * 4.0 + 60.0 + 30.0 * torch.randn(2, 1024, 1, generator=g)).to(x["k"].dtype)
    y = ops.wkv4_forward(dev(x["w"]), dev(x["u"]), dev(k), dev(x["v"]))
    torch.cuda.synchronize()
    ref = oracle.wkv4(f64(x["w"]), f64(x["u"]), f64(k), f64(x["v"]))
    assert rel_inf(f64(y), ref) <= TOL[y.dtype]


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_wkv4_state_chaining_full_tiles(dtype):
    """Two calls of 1024 tokens (whole tiles) with the state carried equal one call of 2048."""
    B, T, C = 2, 2048, 32
    x = inputs.wkv4_inputs(B, T, C, dtype, seed=13)
    w, u, k, v = dev(x["w"]), dev(x["u"]), dev(x["k"]), dev(x["v"])
    y1, s1 = ops.wkv4_forward(w, u, k[:, :1024].contiguous(), v[:, :1024].contiguous(), want_state=True)
    y2, s2 = ops.wkv4_forward(w, u, k[:, 1024:].contiguous(), v[:, 1024:].contiguous(), s0=s1,
                              want_state=True)
    torch.cuda.synchronize()
    ref_y, ref_s = oracle.wkv4(f64(x["w"]), f64(x["u"]), f64(x["k"]), f64(x["v"]), want_state=True)
    assert rel_inf(f64(torch.cat([y1, y2], 1)), ref_y) <= TOL[k.dtype]
    ga, gb = wkv4_state_views(f64(s2))
    ra, rb = wkv4_state_views(ref_s)
    assert rel_inf(ga, ra) <= 1e-4 and np.max(np.abs(gb - rb)) <= 1e-3


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_wkv4_key_spreads_straddle_the_fp16_weight_range(dtype):
    """Per-channel key scales from 1 to 8 (with u up to 3 where positive): a segment's key spread
    runs from well inside to well beyond the 28 log2 units within which bf16 tiles keep pass 1's
    weights as fp16 for pass 2, so lanes of one CTA take both forms side by side, over four
    16-token-segment tiles."""
    B, T, C = 2, 2048, 64
    x = inputs.wkv4_inputs(B, T, C, dtype, seed=31)
    scale = torch.linspace(1.0, 8.0, C)
    k = (x["k"].float() * scale).to(x["k"].dtype)
    u = x["u"] * 3.0
    y, sT = ops.wkv4_forward(dev(x["w"]), dev(u), dev(k), dev(x["v"]), want_state=True)
    torch.cuda.synchronize()
    ref_y, ref_s = oracle.wkv4(f64(x["w"]), f64(u), f64(k), f64(x["v"]), want_state=True)
    assert rel_inf(f64(y), ref_y) <= TOL[y.dtype]
    ga, gb = wkv4_state_views(f64(sT))
    ra, rb = wkv4_state_views(ref_s)
    assert rel_inf(ga, ra) <= 1e-4 and np.max(np.abs(gb - rb)) <= 1e-3


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_wkv4_carried_state_of_any_weight(dtype):
    """A carried state whose exponent p runs, channel by channel, from far below the new keys'
    to far above them (-60 to 160 in natural-log units): where the state dominates, the
    segments leave the fixed frame for the running-maximum steps (reading the keys from
    global memory when pass 1 kept fp16 weights in their place); where it is comparable, the
    stored weights are brought to its reference; where it is negligible it drops out."""
    B, T, C = 2, 1024, 48
    x = inputs.wkv4_inputs(B, T, C, dtype, seed=21)
    rng = np.random.default_rng(22)
    b = rng.uniform(0.5, 2.0, (B, C))
    s0 = np.stack([rng.standard_normal((B, C)) * b, b, np.tile(np.linspace(-60.0, 160.0, C), (B, 1))], 1)
    y, sT = ops.wkv4_forward(dev(x["w"]), dev(x["u"]), dev(x["k"]), dev(x["v"]),
                             s0=torch.from_numpy(s0).float().cuda(), want_state=True)
    torch.cuda.synchronize()
    ref_y, ref_s = oracle.wkv4(f64(x["w"]), f64(x["u"]), f64(x["k"]), f64(x["v"]),
                               s0=s0.astype(np.float32).astype(np.float64), want_state=True)
    assert rel_inf(f64(y), ref_y) <= TOL[y.dtype]
    ga, gb = wkv4_state_views(f64(sT))
    ra, rb = wkv4_state_views(ref_s)
    assert rel_inf(ga, ra) <= 1e-4 and np.max(np.abs(gb - rb)) <= 1e-3


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("C", [96, 98, 37])
def test_wkv4_decode_chained_in_place_matches_the_oracle(dtype, C):
    """40 single-token calls (the T = 1 decode kernel), the state updated in place, equal
    the oracle over all 40 tokens: every y and the final (a, b, p) state.  C = 96, 98 and 37
    take the kernel's 4-, 2- and 1-channel-per-thread forms."""
    B, T = 4, 40
    x = inputs.wkv4_inputs(B, T, C, dtype, seed=21)
    w, u, k, v = dev(x["w"]), dev(x["u"]), dev(x["k"]), dev(x["v"])
    y0, s = ops.wkv4_forward(w, u, k[:, :1].contiguous(), v[:, :1].contiguous(), want_state=True)
    ys = [y0]
    for t in range(1, T):
        yt, s2 = ops.wkv4_forward(w, u, k[:, t:t + 1].contiguous(), v[:, t:t + 1].contiguous(), s0=s, sT=s,
                                  want_state=True)
        assert s2.data_ptr() == s.data_ptr()
        ys.append(yt)
    torch.cuda.synchronize()
    ref_y, ref_s = oracle.wkv4(f64(x["w"]), f64(x["u"]), f64(x["k"]), f64(x["v"]), want_state=True)
    assert rel_inf(f64(torch.cat(ys, 1)), ref_y) <= TOL[k.dtype]
    ga, gb = wkv4_state_views(f64(s))
    ra, rb = wkv4_state_views(ref_s)
    assert rel_inf(ga, ra) <= 1e-4 and np.max(np.abs(gb - rb)) <= 1e-3


def test_wkv4_decode_large_keys_and_fresh_state():
    """One token from an empty state is v exactly (to fp32 rounding), for any key size."""
    x = inputs.wkv4_inputs(3, 1, 130, "fp32", seed=22)
    k = dev(x["k"]) * 40.0
    y, s = ops.wkv4_forward(dev(x["w"]), dev(x["u"]), k, dev(x["v"]), want_state=True)
    torch.cuda.synchronize()
    assert rel_inf(f64(y), f64(x["v"])) <= 1e-6
    assert torch.all(s[:, 1] == 1.0)  # one weight, referenced to itself
