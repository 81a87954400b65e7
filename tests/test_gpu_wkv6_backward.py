"""GPU parity of the WKV-6 backward pass against the fp64 oracle's reverse-mode
derivative (oracle.wkv6_backward, pinned by finite differences of the forward oracle),
through the C ABI.

Two paths:
  * the exact fp32 walks (fp32 inputs, or bf16 inputs with algo="serial"): they compute in
    fp32 from the exact input values, so the fp32 tolerance 1e-4 applies to every gradient;
  * the chunked tensor-core path (bf16 inputs, the default): bf16 MMA operands with fp32
    accumulation, so the bf16 tolerance 2e-2 applies.  Sequences whose decay is too fast for
    its chunk algebra are served by the exact walks inside the same call.

Covers ragged token counts around the 64-token chunk and the 8-token checkpoint block, zero
and random initial states and state gradients, batch summation of du, the decay logit,
sequences handed to the exact walks (fast decays, tiny w) beside ones that are not, ds0 in
place of dsT, T = 0, determinism, and the Finch prefill shape (B8 T4096 H32) checked on
every batch row of sampled heads."""
import pytest
import torch

import oracle
from gpu_util import TOL, dev, f64, rel_inf
from wkv_recurrence_02_b200 import inputs, ops

pytestmark = pytest.mark.gpu
TOL_WALKS = TOL[torch.float32]
TOL_CHUNKED = TOL[torch.bfloat16]
NAMES = ("dr", "dk", "dv", "dw", "du", "ds0")


def _grads(B, T, H, dtype, seed, s0=True, dsT=True):
    x = inputs.wkv6_inputs(B, T, H, 64, dtype, seed=seed, s0_std=0.1 if s0 else None)
    g = torch.Generator().manual_seed(seed + 500)
    x["dy"] = torch.randn(B, T, H, 64, generator=g).to(x["r"].dtype)
    x["dsT"] = torch.randn(B, H, 64, 64, generator=g) * 0.1 if dsT else None
    return x


def _tol(x, algo):
    return TOL_CHUNKED if (x["r"].dtype == torch.bfloat16 and algo != "serial") else TOL_WALKS


def _compare(got, ref, names, tol):
    for n in names:
        e = rel_inf(f64(got[n]), ref[n], what=n)
        assert e <= tol, (n, e)


def _oracle(x, omega=False):
    s0 = f64(x["s0"]) if x.get("s0") is not None else None
    dsT = f64(x["dsT"]) if x.get("dsT") is not None else None
    if omega:
        return oracle.wkv6_logit_backward(f64(x["r"]), f64(x["k"]), f64(x["v"]), f64(x["omega"]), f64(x["u"]),
                                          f64(x["dy"]), s0=s0, dsT=dsT)
    return oracle.wkv6_backward(f64(x["r"]), f64(x["k"]), f64(x["v"]), f64(x["w"]), f64(x["u"]), f64(x["dy"]),
                                s0=s0, dsT=dsT)


def _run(x, omega=False, algo=None):
    xd = {n: dev(t) for n, t in x.items() if t is not None}
    wkey = "omega" if omega else "w"
    got = ops.wkv6_backward(xd["r"], xd["k"], xd["v"], xd[wkey], xd["u"], xd["dy"], s0=xd.get("s0"),
                            dsT=xd.get("dsT"), omega=omega, algo=algo)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    return got, _oracle(x, omega)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("B,T,H", [(1, 1, 1), (2, 7, 2), (1, 8, 3), (2, 9, 2), (3, 67, 2), (1, 63, 1),
                                   (1, 64, 1), (1, 65, 3), (2, 130, 2)])
def test_backward_matches_oracle(dtype, B, T, H):
    """Default path: the walks for fp32 inputs, the chunked tensor-core path for bf16."""
    x = _grads(B, T, H, dtype, seed=B * 1000 + T * 10 + H)
    got, ref = _run(x)
    _compare(got, ref, NAMES, _tol(x, None))


@pytest.mark.parametrize("B,T,H", [(2, 9, 2), (3, 67, 2)])
def test_backward_walks_on_bf16_inputs(B, T, H):
    """algo="serial" keeps bf16 inputs on the exact fp32 walks."""
    x = _grads(B, T, H, "bf16", seed=B * 1000 + T * 10 + H + 7)
    got, ref = _run(x, algo="serial")
    _compare(got, ref, NAMES, TOL_WALKS)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_backward_zero_state_and_no_state_gradient(dtype):
    x = _grads(2, 40, 2, dtype, seed=31, s0=False, dsT=False)
    got, ref = _run(x)
    _compare(got, ref, NAMES, _tol(x, None))


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_backward_longer_sequence(dtype):
    """T = 1000: 125 checkpoint blocks of the walks, 16 chunks (ragged last) of the chunked path."""
    x = _grads(2, 1000, 3, dtype, seed=32)
    got, ref = _run(x)
    _compare(got, ref, NAMES, _tol(x, None))


@pytest.mark.parametrize("algo", [None, "serial"])
def test_backward_logit_matches_oracle(algo):
    B, T, H = 2, 170, 2
    x = _grads(B, T, H, "bf16", seed=33)
    x["omega"] = inputs.wkv6_inputs(B, T, H, 64, "bf16", seed=33, s0_std=0.1, decay="omega")["omega"]
    del x["w"]
    got, ref = _run(x, omega=True, algo=algo)
    _compare(got, ref, ("dr", "dk", "dv", "domega", "du", "ds0"), _tol(x, algo))


def test_backward_fast_decay_heads_go_to_the_walks():
    """Head 0 has channels with w = 0.1 (a 64-token decay product of 1e-64, below the chunk
    algebra's 2^-100 guard), head 1 has none: head 0 is served by the exact walks (1e-4),
    head 1 by the chunked path (2e-2); du sums both kinds over the batch."""
    B, T, H = 2, 200, 2
    x = _grads(B, T, H, "bf16", seed=34)
    w = x["w"].float()
    w[:, :, 0, 24:40] = 0.1
    x["w"] = w.to(torch.bfloat16)
    got, ref = _run(x)
    for n in ("dr", "dk", "dv", "dw"):
        assert rel_inf(f64(got[n][:, :, 0]), ref[n][:, :, 0], what=n + " head 0") <= TOL_WALKS, n
        assert rel_inf(f64(got[n][:, :, 1]), ref[n][:, :, 1], what=n + " head 1") <= TOL_CHUNKED, n
    assert rel_inf(f64(got["ds0"][:, 0]), ref["ds0"][:, 0], what="ds0 head 0") <= TOL_WALKS
    assert rel_inf(f64(got["ds0"][:, 1]), ref["ds0"][:, 1], what="ds0 head 1") <= TOL_CHUNKED
    assert rel_inf(f64(got["du"]), ref["du"], what="du") <= TOL_CHUNKED


def test_backward_tiny_w_goes_to_the_walks():
    """A few tokens with w below 2^-5 (dw = d(log w) / w would magnify rounding) and w rounded
    to exactly 1.0 on other channels: the sequences holding the tiny w take the exact walks;
    the result matches the oracle."""
    B, T, H = 1, 300, 2
    x = _grads(B, T, H, "bf16", seed=35)
    w = x["w"].float()
    w[..., 0:8] = 0.9999           # rounds to 1.0 in bf16
    w[:, 100:103, 1, 8:12] = 1e-3  # head 1 only
    x["w"] = w.to(torch.bfloat16)
    got, ref = _run(x)
    _compare(got, ref, NAMES, TOL_CHUNKED)
    for n in ("dr", "dk", "dv", "dw"):
        assert rel_inf(f64(got[n][:, :, 1]), ref[n][:, :, 1], what=n + " head 1") <= TOL_WALKS, n


def test_backward_in_place_state_gradient():
    """ds0 written over dsT (the same array), on the chunked path and through the walks."""
    for seed, fast in ((36, False), (37, True)):
        x = _grads(2, 150, 2, "bf16", seed=seed)
        if fast:
            w = x["w"].float()
            w[..., 0:4] = 0.05
            x["w"] = w.to(torch.bfloat16)
        ref = _oracle(x)
        xd = {n: dev(t) for n, t in x.items() if t is not None}
        g = xd["dsT"].clone()
        got = ops.wkv6_backward(xd["r"], xd["k"], xd["v"], xd["w"], xd["u"], xd["dy"], s0=xd["s0"], dsT=g,
                                want_ds0=False)
        lib = ops.load()
        # the same call with ds0 == dsT through the C ABI
        ws = torch.empty(ops.wkv6_backward_workspace_bytes(2, 150, 2), device="cuda", dtype=torch.uint8)
        out = {n: torch.empty_like(got[n]) for n in ("dr", "dk", "dv", "dw", "du")}
        import ctypes
        p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
        ops._use_current_stream(lib, xd["r"].device)
        rc = lib.rwkv_wkv6_backward_bf16(2, 150, 2, 64, p(xd["r"]), p(xd["k"]), p(xd["v"]), p(xd["w"]), p(xd["u"]),
                                         p(xd["s0"]), p(xd["dy"]), p(g), p(out["dr"]), p(out["dk"]), p(out["dv"]),
                                         p(out["dw"]), p(out["du"]), p(g), p(ws), ctypes.c_size_t(ws.numel()))
        assert rc == 0, lib.rwkv_last_error()
        torch.cuda.synchronize()
        assert ops.device_status() == 0
        tol = TOL_WALKS if fast else TOL_CHUNKED
        assert rel_inf(f64(g), ref["ds0"], what="ds0 in place") <= tol
        for n in ("dr", "dk", "dv", "dw"):
            assert torch.equal(out[n], got[n]), n


def test_backward_deterministic():
    x = _grads(2, 500, 4, "bf16", seed=38)
    xd = {n: dev(t) for n, t in x.items() if t is not None}
    a = ops.wkv6_backward(xd["r"], xd["k"], xd["v"], xd["w"], xd["u"], xd["dy"], s0=xd["s0"], dsT=xd["dsT"])
    b = ops.wkv6_backward(xd["r"], xd["k"], xd["v"], xd["w"], xd["u"], xd["dy"], s0=xd["s0"], dsT=xd["dsT"])
    torch.cuda.synchronize()
    for n in NAMES:
        assert torch.equal(a[n], b[n]), n


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
    """B8 T4096 H32 bf16 (the Finch prefill) on the chunked path: the full call on the GPU;
    the oracle on every batch row of two heads (their du sums over all batch rows)."""
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
            assert rel_inf(f64(got[n][:, :, sl]), ref[n], what=f"{n} head {h}") <= TOL_CHUNKED, (h, n)
        assert rel_inf(f64(got["du"][sl]), ref["du"], what=f"du head {h}") <= TOL_CHUNKED, (h, "du")
        assert rel_inf(f64(got["ds0"][:, sl]), ref["ds0"], what=f"ds0 head {h}") <= TOL_CHUNKED, (h, "ds0")
