"""GPU parity of WKV-6 fed the decay logit omega_t (w_t = exp(-exp(omega_t)), formed by the
kernels) against the fp64 oracle (oracle.wkv6_logit = the pinned decay map followed by the
WKV-6 oracle, and the head LayerNorm + SiLU gate when asked), through the C ABI.

Covers the chunked kernel (ragged tail, sequence split, sub-block and exact-diagonal paths
with w = 0 and w = 1 exactly), the decode kernel (T = 1), the serial kernel, the fused
output stage, chaining, and slowly decaying channels that a bf16 w cannot represent."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import TOL, dev, f64, rel_inf
from wkv_recurrence_02_b200 import inputs, ops

pytestmark = pytest.mark.gpu
TOL_BF16 = TOL[torch.bfloat16]


def _inputs(B, T, H, seed, s0=True):
    return inputs.wkv6_inputs(B, T, H, 64, "bf16", seed=seed, s0_std=0.1 if s0 else None, decay="omega")


def _gpu(x, gate=None, segments=None, algo=None):
    xd = {n: dev(t) for n, t in x.items() if t is not None}
    gd = {n: dev(t) for n, t in gate.items()} if gate is not None else {}
    lib = ops.load()
    if segments is not None:
        prev = lib.rwkv_get_wkv6_segments()
        lib.rwkv_set_wkv6_segments(segments)
    try:
        y, sT = ops.wkv6_forward_omega(xd["r"], xd["k"], xd["v"], xd["omega"], xd["u"], s0=xd.get("s0"),
                                       g=gd.get("g"), ln_w=gd.get("ln_w"), ln_b=gd.get("ln_b"), algo=algo)
    finally:
        if segments is not None:
            lib.rwkv_set_wkv6_segments(prev)
    torch.cuda.synchronize()
    return y, sT


def _oracle(x, gate=None):
    s0 = f64(x["s0"]) if x["s0"] is not None else None
    if gate is None:
        return oracle.wkv6_logit(f64(x["r"]), f64(x["k"]), f64(x["v"]), f64(x["omega"]), f64(x["u"]), s0=s0)
    return oracle.wkv6_logit(f64(x["r"]), f64(x["k"]), f64(x["v"]), f64(x["omega"]), f64(x["u"]), s0=s0,
                             g=f64(gate["g"]), ln_w=f64(gate["ln_w"]), ln_b=f64(gate["ln_b"]), eps=1e-5)


def _check(x, gate=None, **kw):
    y, sT = _gpu(x, gate, **kw)
    ry, rs = _oracle(x, gate)
    ey, es = rel_inf(f64(y), ry), rel_inf(f64(sT), rs)
    assert ey <= TOL_BF16 and es <= TOL_BF16, (ey, es)
    return ey, es


@pytest.mark.parametrize("B,T,H", [(2, 300, 4), (1, 64, 2), (3, 129, 3)])
def test_omega_chunked_matches_oracle(B, T, H):
    _check(_inputs(B, T, H, seed=B * 100 + T + H))


def test_omega_decode_matches_oracle():
    _check(_inputs(16, 1, 8, seed=21))


def test_omega_serial_kernel_matches_oracle():
    _check(_inputs(2, 100, 3, seed=22), algo="serial")


def test_omega_sequence_split_matches_oracle():
    """B1 H8 T2048 split into 4 segments: the first pass also forms w from omega."""
    _check(_inputs(1, 2048, 8, seed=23), segments=4)


@pytest.mark.parametrize("B,T,H", [(2, 300, 4), (16, 1, 8)])
def test_omega_gated_matches_oracle(B, T, H):
    """Logit input and the fused head LayerNorm + SiLU gate together (chunked, decode)."""
    _check(_inputs(B, T, H, seed=24 + T), gate=inputs.norm_gate_inputs(B, T, H, 64, seed=25))


def test_omega_extremes_zero_and_unit_decay():
    """omega = +8 or +inf (w = 0 exactly in fp32: the state forgets everything), -30 or -inf
    (w = 1 exactly in fp32) and U(-6, 1) mixed per element: chunks take the sub-block path
    with the exact diagonal."""
    B, T, H = 2, 257, 2
    x = _inputs(B, T, H, seed=26)
    g = torch.Generator().manual_seed(27)
    pick = torch.rand(B, T, H, 64, generator=g)
    om = torch.rand(B, T, H, 64, generator=g) * 7.0 - 6.0
    om = torch.where(pick < 0.15, torch.full_like(om, 8.0), om)
    om = torch.where((pick >= 0.15) & (pick < 0.3), torch.full_like(om, -30.0), om)
    om = torch.where((pick >= 0.3) & (pick < 0.33), torch.full_like(om, float("inf")), om)
    om = torch.where((pick >= 0.33) & (pick < 0.36), torch.full_like(om, -float("inf")), om)
    x["omega"] = om.to(torch.bfloat16)
    _check(x)
    _check(x, algo="serial")


def test_omega_chaining():
    """Two calls with the state carried equal one call."""
    B, T, H = 2, 256, 4
    x = _inputs(B, T, H, seed=28)
    xd = {n: dev(t) for n, t in x.items()}
    part = lambda sl: [xd[n][:, sl].contiguous() for n in ("r", "k", "v", "omega")]  # noqa: E731
    y1, s1 = ops.wkv6_forward_omega(*part(slice(0, 100)), xd["u"], s0=xd["s0"])
    y2, s2 = ops.wkv6_forward_omega(*part(slice(100, T)), xd["u"], s0=s1)
    torch.cuda.synchronize()
    ry, rs = _oracle(x)
    assert rel_inf(f64(torch.cat([y1, y2], 1)), ry) <= TOL_BF16
    assert rel_inf(f64(s2), rs) <= TOL_BF16


def test_omega_keeps_slow_decay_that_bf16_w_loses():
    """omega in [-9, -6.5]: w = exp(-exp(omega)) lies within 1.5e-3 of 1, where bf16 has no
    value between 1 - 2^-8 and 1.  Over T = 2048 the state's memory of s0 decays by
    prod w ~ e^-(0.3..3).  The logit path follows the exact decay; the same decay rounded
    to bf16 and passed as w does not."""
    B, T, H = 1, 2048, 4
    x = _inputs(B, T, H, seed=29)
    g = torch.Generator().manual_seed(30)
    x["omega"] = (torch.rand(B, T, H, 64, generator=g) * 2.5 - 9.0).to(torch.bfloat16)
    x["s0"] = torch.randn(B, H, 64, 64, generator=g)
    ey, es = _check(x)
    # the same decays rounded to bf16 and passed as w
    w_bf16 = torch.exp(-torch.exp(x["omega"].double())).to(torch.bfloat16)
    xd = {n: dev(t) for n, t in x.items()}
    _, sT_w = ops.wkv6_forward(xd["r"], xd["k"], xd["v"], dev(w_bf16), xd["u"], s0=xd["s0"])
    torch.cuda.synchronize()
    _, rs = _oracle(x)
    es_w = rel_inf(f64(sT_w), rs, what="expected miss: the bf16-rounded w path")
    assert es_w > 10 * es and es_w > TOL_BF16, (es, es_w)
