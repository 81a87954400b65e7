"""The bounds-checked debug build (libwkv_debug.so, compiled with WKV_DEBUG_BOUNDS) on the
ragged and edge shapes of every kernel.

In that build each kernel checks its global, shared-memory and tensor-memory indices and its
TMA coordinates before using them; a failed check skips the access and records
RWKV_ERR_BOUNDS (-9) in the device status word, nothing traps.  These tests route the
binding's calls to the debug library, run the shapes whose tails and special paths are the
likeliest to step outside a buffer, and require device status 0 and oracle parity: WKV-4 with
T in {1, 63, 65, 777}, C in {1, 37} (the cp.async kernel) and the 169M layer (the TMA kernel);
WKV-6 chunked with T in {1, 63, 65, 777}, the sub-block path, the sequence split, the decay
logit and the fused output stage, the decode and serial kernels; the backward (chunked, with a
sequence left to the exact walks, and the logit path).
"""
import os

import pytest
import torch

import oracle
from gpu_util import TOL, dev, f64, rel_inf
from wkv_recurrence_02_b200 import build, inputs, ops

pytestmark = pytest.mark.gpu
BF, FP = TOL[torch.bfloat16], TOL[torch.float32]


@pytest.fixture(scope="module")
def debug_lib():
    if not os.path.exists(build.LIB_DEBUG):
        build.build(debug_bounds=True)
    with ops.using_library(build.LIB_DEBUG) as lib:
        assert lib.rwkv_debug_bounds() == 1
        assert ops.device_status() == 0
        yield lib


def _status_ok():
    st = ops.device_status()
    assert st == 0, f"device status {st} (-9: a bounds check failed)"


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("B,T,C", [(2, 1, 37), (2, 63, 1), (1, 65, 37), (2, 777, 16), (2, 100, 37)])
def test_debug_wkv4_edges(debug_lib, dtype, B, T, C):
    x = inputs.wkv4_inputs(B, T, C, dtype, seed=T + C)
    g = torch.Generator().manual_seed(T)
    s0 = torch.zeros(B, 3, C)
    s0[:, 0] = torch.randn(B, C, generator=g)
    s0[:, 1] = 1.0 + torch.rand(B, C, generator=g)
    y, sT = ops.wkv4_forward(*(dev(x[n]) for n in ("w", "u", "k", "v")), s0=dev(s0), want_state=True)
    torch.cuda.synchronize()
    _status_ok()
    ry, _ = oracle.wkv4(*(f64(x[n]) for n in ("w", "u", "k", "v")), s0=f64(s0), want_state=True)
    assert rel_inf(f64(y), ry, what="y") <= (BF if dtype == "bf16" else FP)


def test_debug_wkv4_169m_layer(debug_lib):
    """B8 T1024 C768 bf16: the TMA-fed kernel."""
    x = inputs.wkv4_inputs(8, 1024, 768, "bf16", seed=0, wu_seed=1)
    y = ops.wkv4_forward(*(dev(x[n]) for n in ("w", "u", "k", "v")))
    torch.cuda.synchronize()
    _status_ok()
    assert rel_inf(f64(y), oracle.wkv4(*(f64(x[n]) for n in ("w", "u", "k", "v"))), what="y") <= BF


def _wkv6_ref(x, s0):
    return oracle.wkv6(*(f64(x[n]) for n in ("r", "k", "v", "w", "u")), s0=f64(s0))


@pytest.mark.parametrize("algo", ["chunked", "serial"])
@pytest.mark.parametrize("T", [1, 63, 65, 777])
def test_debug_wkv6_ragged(debug_lib, algo, T):
    x = inputs.wkv6_inputs(2, T, 2, 64, "bf16", seed=T, s0_std=0.1)
    y, sT = ops.wkv6_forward(*(dev(x[n]) for n in ("r", "k", "v", "w", "u")), s0=dev(x["s0"]), algo=algo)
    torch.cuda.synchronize()
    _status_ok()
    ry, rs = _wkv6_ref(x, x["s0"])
    assert rel_inf(f64(y), ry, what="y") <= BF and rel_inf(f64(sT), rs, what="sT") <= BF


def test_debug_wkv6_subblock_split_fp32_decode(debug_lib):
    # sub-block path (w = 0.1 channels) with a sequence split into 3 segments
    x = inputs.wkv6_inputs(2, 1000, 2, 64, "bf16", seed=41, s0_std=0.1)
    w = x["w"].float()
    w[..., 24:40] = 0.1
    x["w"] = w.to(torch.bfloat16)
    y, sT = ops.wkv6_forward(*(dev(x[n]) for n in ("r", "k", "v", "w", "u")), s0=dev(x["s0"]), algo="chunked",
                             segments=3)
    torch.cuda.synchronize()
    _status_ok()
    ry, rs = _wkv6_ref(x, x["s0"])
    assert rel_inf(f64(y), ry, what="y") <= BF and rel_inf(f64(sT), rs, what="sT") <= BF
    # fp32 serial kernel and the T = 1 decode kernel
    for (B, T, dt) in ((1, 65, "fp32"), (4, 1, "bf16")):
        x = inputs.wkv6_inputs(B, T, 3, 64, dt, seed=42 + T, s0_std=0.1)
        y, sT = ops.wkv6_forward(*(dev(x[n]) for n in ("r", "k", "v", "w", "u")), s0=dev(x["s0"]))
        torch.cuda.synchronize()
        _status_ok()
        ry, rs = _wkv6_ref(x, x["s0"])
        tol = FP if dt == "fp32" else BF
        assert rel_inf(f64(y), ry, what="y") <= tol and rel_inf(f64(sT), rs, what="sT") <= tol


@pytest.mark.parametrize("T", [1, 130])
def test_debug_wkv6_logit_and_gate(debug_lib, T):
    x = inputs.wkv6_inputs(2, T, 2, 64, "bf16", seed=43 + T, s0_std=0.1, decay="omega")
    ng = inputs.norm_gate_inputs(2, T, 2, 64, seed=44)
    xd = {n: dev(t) for n, t in x.items()}
    y, sT = ops.wkv6_forward_omega(xd["r"], xd["k"], xd["v"], xd["omega"], xd["u"], s0=xd["s0"],
                                   g=dev(ng["g"]), ln_w=dev(ng["ln_w"]), ln_b=dev(ng["ln_b"]))
    torch.cuda.synchronize()
    _status_ok()
    ry, rs = oracle.wkv6_logit(*(f64(x[n]) for n in ("r", "k", "v", "omega", "u")), s0=f64(x["s0"]),
                               g=f64(ng["g"]), ln_w=f64(ng["ln_w"]), ln_b=f64(ng["ln_b"]), eps=1e-5)
    assert rel_inf(f64(y), ry, what="y") <= BF and rel_inf(f64(sT), rs, what="sT") <= BF


@pytest.mark.parametrize("omega", [False, True])
def test_debug_backward(debug_lib, omega):
    """The chunked backward on a ragged T with one head left to the exact walks (w = 0.1
    channels; plain w only), and the logit path."""
    B, T, H = 2, 130, 2
    x = inputs.wkv6_inputs(B, T, H, 64, "bf16", seed=45, s0_std=0.1, decay="omega" if omega else "w")
    if not omega:
        w = x["w"].float()
        w[:, :, 0, 24:40] = 0.1
        x["w"] = w.to(torch.bfloat16)
    g = torch.Generator().manual_seed(46)
    dy = torch.randn(B, T, H, 64, generator=g).to(torch.bfloat16)
    dsT = torch.randn(B, H, 64, 64, generator=g) * 0.1
    wk = "omega" if omega else "w"
    got = ops.wkv6_backward(*(dev(x[n]) for n in ("r", "k", "v", wk, "u")), dev(dy), s0=dev(x["s0"]),
                            dsT=dev(dsT), omega=omega)
    torch.cuda.synchronize()
    _status_ok()
    args = [f64(x[n]) for n in ("r", "k", "v", wk, "u")] + [f64(dy)]
    if omega:
        ref = oracle.wkv6_logit_backward(*args, s0=f64(x["s0"]), dsT=f64(dsT))
    else:
        ref = oracle.wkv6_backward(*args, s0=f64(x["s0"]), dsT=f64(dsT))
    for n in ("dr", "dk", "dv", "domega" if omega else "dw", "du", "ds0"):
        assert rel_inf(f64(got[n]), ref[n], what=n) <= BF, n
