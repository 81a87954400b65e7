"""GPU parity of the WKV-6 backward pass against the fp64 oracle's reverse-mode
derivative (oracle.wkv6_backward, pinned by finite differences of the forward oracle),
through the C ABI.

The kernels compute in fp32 from the exact input values and write fp32 gradients, so
the fp32 tolerance applies to every gradient whatever the input dtype.  Covers ragged
token counts around the 8-token checkpoint block, zero and random initial states and
state gradients, batch summation of du, the decay logit, T = 0, and the Finch prefill
shape (B8 T4096 H32) checked on every batch row of sampled heads."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import TOL, dev, f64, rel_inf
from wkv_recurrence_02_b200 import inputs, ops

pytestmark = pytest.mark.gpu
TOL_BWD = TOL[torch.float32]


def _grads(B, T, H, dtype, seed, s0=True, dsT=True):
    x = inputs.wkv6_inputs(B, T, H, 64, dtype, seed=seed, s0_std=0.1 if s0 else None)
    g = torch.Generator().manual_seed(seed + 500)
    x["dy"] = torch.randn(B, T, H, 64, generator=g).to(x["r"].dtype)
    x["dsT"] = torch.randn(B, H, 64, 64, generator=g) * 0.1 if dsT else None
    return x


def _compare(got, ref, names):
    for n in names:
        e = rel_inf(f64(got[n]), ref[n])
        assert e <= TOL_BWD, (n, e)


def _run(x, omega=False):
    xd = {n: dev(t) for n, t in x.items() if t is not None}
    wkey = "omega" if omega else "w"
    got = ops.wkv6_backward(xd["r"], xd["k"], xd["v"], xd[wkey], xd["u"], xd["dy"], s0=xd.get("s0"),
                            dsT=xd.get("dsT"), omega=omega)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    s0 = f64(x["s0"]) if x["s0"] is not None else None
    dsT = f64(x["dsT"]) if x["dsT"] is not None else None
    if omega:
        ref = oracle.wkv6_logit_backward(f64(x["r"]), f64(x["k"]), f64(x["v"]), f64(x["omega"]), f64(x["u"]),
                                         f64(x["dy"]), s0=s0, dsT=dsT)
    else:
        ref = oracle.wkv6_backward(f64(x["r"]), f64(x["k"]), f64(x["v"]), f64(x["w"]), f64(x["u"]), f64(x["dy"]),
                                   s0=s0, dsT=dsT)
    return got, ref


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("B,T,H", [(1, 1, 1), (2, 7, 2), (1, 8, 3), (2, 9, 2), (3, 67, 2)])
def test_backward_matches_oracle(dtype, B, T, H):
    x = _grads(B, T, H, dtype, seed=B * 1000 + T * 10 + H)
    got, ref = _run(x)
    _compare(got, ref, ("dr", "dk", "dv", "dw", "du", "ds0"))


def test_backward_zero_state_and_no_state_gradient():
    x = _grads(2, 40, 2, "bf16", seed=31, s0=False, dsT=False)
    got, ref = _run(x)
    _compare(got, ref, ("dr", "dk", "dv", "dw", "du", "ds0"))


def test_backward_longer_sequence():
    """T = 1000 in fp32: 125 checkpoint blocks."""
    x = _grads(1, 1000, 2, "fp32", seed=32)
    got, ref = _run(x)
    _compare(got, ref, ("dr", "dk", "dv", "dw", "du", "ds0"))


def test_backward_logit_matches_oracle():
    B, T, H = 2, 70, 2
    x = _grads(B, T, H, "bf16", seed=33)
    om = inputs.wkv6_inputs(B, T, H, 64, "bf16", seed=33, s0_std=0.1, decay="omega")["omega"]
    x["omega"] = om
    del x["w"]
    got, ref = _run(x, omega=True)
    _compare(got, ref, ("dr", "dk", "dv", "domega", "du", "ds0"))


def test_backward_no_tokens():
    """T = 0: du = 0 and ds0 = dsT."""
    B, H = 2, 3
    u = torch.randn(H, 64, device="cuda")
    e = torch.empty(B, 0, H, 64, device="cuda")
    dsT = torch.randn(B, H, 64, 64, device="cuda")
    got = ops.wkv6_backward(e, e, e, e, u, e, dsT=dsT)
    torch.cuda.synchronize()
    assert torch.count_nonzero(got["du"]) == 0
    assert torch.equal(got["ds0"], dsT)


def test_backward_finch_shape_sampled_heads():
    """B8 T4096 H32 bf16 (the Finch prefill): the full call on the GPU; the oracle on every
    batch row of two heads (their du sums over all batch rows)."""
    B, T, H = 8, 4096, 32
    x = _grads(B, T, H, "bf16", seed=34)
    xd = {n: dev(t) for n, t in x.items()}
    got = ops.wkv6_backward(xd["r"], xd["k"], xd["v"], xd["w"], xd["u"], xd["dy"], s0=xd["s0"], dsT=xd["dsT"])
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    for h in (5, 30):
        sl = slice(h, h + 1)
        ref = oracle.wkv6_backward(*(f64(x[n][:, :, sl]) for n in ("r", "k", "v", "w")), f64(x["u"][sl]),
                                   f64(x["dy"][:, :, sl]), s0=f64(x["s0"][:, sl]), dsT=f64(x["dsT"][:, sl]))
        for n in ("dr", "dk", "dv", "dw"):
            assert rel_inf(f64(got[n][:, :, sl]), ref[n]) <= TOL_BWD, (h, n)
        assert rel_inf(f64(got["du"][sl]), ref["du"]) <= TOL_BWD, (h, "du")
        assert rel_inf(f64(got["ds0"][:, sl]), ref["ds0"]) <= TOL_BWD, (h, "ds0")
