"""GPU parity of WKV-6 with the fused output stage (head LayerNorm, SiLU gate) against the
fp64 oracle (oracle.wkv6_gated = the WKV-6 oracle followed by the pinned head_norm_gate),
through the C ABI.  Covers the chunked kernel (ragged tail, sequence split, sub-block path)
and the decode kernel (T = 1)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import TOL, dev, f64, rel_inf
from wkv_recurrence_02_b200 import inputs, ops

pytestmark = pytest.mark.gpu
EPS = 1e-5


def _run(B, T, H, seed, s0=True, w_override=None, segments=None, eps=EPS):
    x = inputs.wkv6_inputs(B, T, H, 64, "bf16", seed=seed, s0_std=0.1 if s0 else None)
    if w_override is not None:
        x["w"] = w_override
    ng = inputs.norm_gate_inputs(B, T, H, 64, seed=seed + 1000)
    xd = {n: dev(t) for n, t in x.items() if t is not None}
    gd = {n: dev(t) for n, t in ng.items()}
    if segments is not None:
        prev = ops.load().rwkv_get_wkv6_segments()
        ops.load().rwkv_set_wkv6_segments(segments)
    try:
        y, sT = ops.wkv6_forward_gated(xd["r"], xd["k"], xd["v"], xd["w"], xd["u"], gd["g"], gd["ln_w"],
                                       gd["ln_b"], eps=eps, s0=xd.get("s0"))
    finally:
        if segments is not None:
            ops.load().rwkv_set_wkv6_segments(prev)
    torch.cuda.synchronize()
    ry, rs = oracle.wkv6_gated(f64(x["r"]), f64(x["k"]), f64(x["v"]), f64(x["w"]), f64(x["u"]),
                               f64(ng["g"]), f64(ng["ln_w"]), f64(ng["ln_b"]), eps,
                               s0=f64(x["s0"]) if x["s0"] is not None else None)
    return y, sT, ry, rs


@pytest.mark.parametrize("B,T,H", [(2, 300, 4), (1, 64, 2), (3, 129, 3)])
def test_gated_chunked_matches_oracle(B, T, H):
    y, sT, ry, rs = _run(B, T, H, seed=B * 100 + T + H)
    tol = TOL[torch.bfloat16]
    assert rel_inf(f64(y), ry) <= tol
    assert rel_inf(f64(sT), rs) <= tol


def test_gated_decode_matches_oracle():
    y, sT, ry, rs = _run(16, 1, 8, seed=7)
    tol = TOL[torch.bfloat16]
    assert rel_inf(f64(y), ry) <= tol
    assert rel_inf(f64(sT), rs) <= tol


def test_gated_sequence_split_matches_oracle():
    """B1 H8 T2048: the launcher splits each sequence (first pass, then the gated pass)."""
    y, sT, ry, rs = _run(1, 2048, 8, seed=8, segments=4)
    tol = TOL[torch.bfloat16]
    assert rel_inf(f64(y), ry) <= tol
    assert rel_inf(f64(sT), rs) <= tol


def test_gated_sub_block_path_matches_oracle():
    """Decays near 0.3 make every chunk decay product fall below 2^-100: the sub-block path."""
    B, T, H = 1, 256, 2
    g = torch.Generator().manual_seed(9)
    w = (0.25 + 0.1 * torch.rand(B, T, H, 64, generator=g)).to(torch.bfloat16)
    y, sT, ry, rs = _run(B, T, H, seed=9, w_override=w)
    tol = TOL[torch.bfloat16]
    assert rel_inf(f64(y), ry) <= tol
    assert rel_inf(f64(sT), rs) <= tol


def test_gated_chaining():
    """Two gated calls with the state carried equal one call (y concatenated, final state)."""
    B, T, H = 2, 256, 4
    x = inputs.wkv6_inputs(B, T, H, 64, "bf16", seed=10, s0_std=0.1)
    ng = inputs.norm_gate_inputs(B, T, H, 64, seed=11)
    xd = {n: dev(t) for n, t in x.items()}
    gd = {n: dev(t) for n, t in ng.items()}
    args = lambda sl: [xd[n][:, sl].contiguous() for n in ("r", "k", "v", "w")]  # noqa: E731
    y1, s1 = ops.wkv6_forward_gated(*args(slice(0, 100)), xd["u"], gd["g"][:, :100].contiguous(), gd["ln_w"],
                                    gd["ln_b"], s0=xd["s0"])
    y2, s2 = ops.wkv6_forward_gated(*args(slice(100, T)), xd["u"], gd["g"][:, 100:].contiguous(), gd["ln_w"],
                                    gd["ln_b"], s0=s1)
    torch.cuda.synchronize()
    ry, rs = oracle.wkv6_gated(f64(x["r"]), f64(x["k"]), f64(x["v"]), f64(x["w"]), f64(x["u"]), f64(ng["g"]),
                               f64(ng["ln_w"]), f64(ng["ln_b"]), EPS, s0=f64(x["s0"]))
    tol = TOL[torch.bfloat16]
    assert rel_inf(f64(torch.cat([y1, y2], 1)), ry) <= tol
    assert rel_inf(f64(s2), rs) <= tol


def test_gate_closed_forms():
    """g = 0 gives y = 0 exactly; ln_w = 0, ln_b = 1 gives y = SiLU(g) (to bf16 rounding)."""
    B, T, H = 2, 130, 2
    x = inputs.wkv6_inputs(B, T, H, 64, "bf16", seed=12, s0_std=0.1)
    xd = {n: dev(t) for n, t in x.items()}
    zeros = torch.zeros(B, T, H, 64, dtype=torch.bfloat16, device="cuda")
    one, zero = torch.ones(H, 64, device="cuda"), torch.zeros(H, 64, device="cuda")
    y0 = ops.wkv6_forward_gated(xd["r"], xd["k"], xd["v"], xd["w"], xd["u"], zeros, one, zero, s0=xd["s0"],
                                want_state=False)
    g = (torch.randn(B, T, H, 64, generator=torch.Generator().manual_seed(13)) * 2).to(torch.bfloat16)
    ys = ops.wkv6_forward_gated(xd["r"], xd["k"], xd["v"], xd["w"], xd["u"], dev(g), zero, one,
                                s0=xd["s0"], want_state=False)
    torch.cuda.synchronize()
    assert torch.count_nonzero(y0) == 0
    gf = f64(g)
    assert rel_inf(f64(ys), gf / (1.0 + np.exp(-gf))) <= 1e-2


def test_gate_silu_elementwise_on_a_grid():
    """ln_w = 0, ln_b = 1 gives y = SiLU(g); on a grid of g from -8 to 8 every element is within
    1 % of g / (1 + e^-g) (bf16 rounding of y alone is up to 0.39 %), through the chunked
    kernel and the decode kernel."""
    H = 2
    g = torch.linspace(-8.0, 8.0, 4096 * H * 64).to(torch.bfloat16)
    one, zero = torch.ones(H, 64, device="cuda"), torch.zeros(H, 64, device="cuda")
    for B, T in [(1, 4096), (4096, 1)]:
        x = inputs.wkv6_inputs(B, T, H, 64, "bf16", seed=14, s0_std=0.1)
        xd = {n: dev(t) for n, t in x.items()}
        gg = g.reshape(B, T, H, 64)
        y = ops.wkv6_forward_gated(xd["r"], xd["k"], xd["v"], xd["w"], xd["u"], dev(gg), zero, one,
                                   s0=xd["s0"], want_state=False)
        torch.cuda.synchronize()
        gf = f64(gg)
        ref = gf / (1.0 + np.exp(-gf))
        rel = np.abs(f64(y) - ref) / np.abs(ref)
        assert np.max(rel[np.abs(gf) > 0]) <= 1e-2, (B, T, np.max(rel[np.abs(gf) > 0]))
