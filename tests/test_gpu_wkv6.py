"""GPU parity of the WKV-6 kernels (serial, decode, chunked) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import TOL, dev, f64, rel_inf
from wkv_recurrence_02_b200 import inputs, ops

pytestmark = pytest.mark.gpu


def _inputs(B, T, H, dtype, seed, s0_std=None):
    return inputs.wkv6_inputs(B, T, H, 64, dtype, seed=seed, s0_std=s0_std)


def _ref(x, s0=None):
    return oracle.wkv6(f64(x["r"]), f64(x["k"]), f64(x["v"]), f64(x["w"]), f64(x["u"]),
                       s0=f64(s0))


def _gpu(x, s0=None, algo=None, **kw):
    return ops.wkv6_forward(dev(x["r"]), dev(x["k"]), dev(x["v"]), dev(x["w"]), dev(x["u"]),
                            s0=dev(s0), algo=algo, **kw)


def _check(x, s0=None, algo=None, tol=None):
    y, sT = _gpu(x, s0=s0, algo=algo)
    torch.cuda.synchronize()
    ry, rs = _ref(x, s0)
    tol = tol or TOL[y.dtype]
    ey, es = rel_inf(f64(y), ry), rel_inf(f64(sT), rs)
    assert ey <= tol and es <= tol, (ey, es)
    return ey, es


def test_wkv6_small_fp32_workload():
    """B=1, T=256, H=4 fp32, zero initial state: y and sT in full."""
    _check(_inputs(1, 256, 4, "fp32", 0))


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_wkv6_decode_7b(dtype):
    """T=1 decode at B=256, H=64 with a random fp32 state (the bandwidth-bound kernel)."""
    x = _inputs(256, 1, 64, dtype, 7, s0_std=0.1)
    _check(x, s0=x["s0"])


@pytest.mark.parametrize("algo", ["serial", "chunked"])
@pytest.mark.parametrize("B,T,H", [(1, 1, 1), (1, 63, 2), (2, 64, 1), (1, 65, 3),
                                   (2, 200, 2), (1, 777, 1), (3, 130, 5)])
def test_wkv6_bf16_ragged(algo, B, T, H):
    x = _inputs(B, T, H, "bf16", 100 + B * T + H, s0_std=0.1)
    _check(x, s0=x["s0"], algo=algo)
    _check(x, s0=None, algo=algo)


def test_wkv6_finch_1b6_prefill():
    """B=8, T=4096, H=32 bf16 with a random fp32 initial state, in full (default kernel)."""
    x = _inputs(8, 4096, 32, "bf16", 0, s0_std=0.1)
    _check(x, s0=x["s0"])


def test_wkv6_7b_long_context_chained():
    """B=1, T=16384 as 4 chained calls of 4096 (sT -> s0), H=64 bf16, zero initial state."""
    x = _inputs(1, 16384, 64, "bf16", 0)
    ry, rs = _ref(x)
    s = None
    ys = []
    for c in range(4):
        sl = slice(c * 4096, (c + 1) * 4096)
        y, s = ops.wkv6_forward(dev(x["r"][:, sl]), dev(x["k"][:, sl]), dev(x["v"][:, sl]),
                                dev(x["w"][:, sl]), dev(x["u"]), s0=s)
        ys.append(y)
    torch.cuda.synchronize()
    y = torch.cat(ys, 1)
    assert rel_inf(f64(y), ry) <= TOL[torch.bfloat16]
    assert rel_inf(f64(s), rs) <= TOL[torch.bfloat16]


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_wkv6_chaining_matches_single_call(dtype):
    x = _inputs(2, 300, 3, dtype, 11, s0_std=0.1)
    y_full, s_full = _gpu(x, s0=x["s0"])
    s = dev(x["s0"])
    ys = []
    for lo, hi in [(0, 1), (1, 129), (129, 300)]:
        y, s = ops.wkv6_forward(*(dev(x[n][:, lo:hi]) for n in ("r", "k", "v", "w")),
                                dev(x["u"]), s0=s)
        ys.append(y)
    torch.cuda.synchronize()
    ry, rs = _ref(x, x["s0"])
    tol = TOL[y_full.dtype]
    assert rel_inf(f64(torch.cat(ys, 1)), ry) <= tol and rel_inf(f64(s), rs) <= tol
    assert rel_inf(f64(y_full), ry) <= tol and rel_inf(f64(s_full), rs) <= tol


def test_wkv6_in_place_state_and_T0():
    x = _inputs(2, 100, 2, "bf16", 12, s0_std=0.1)
    s = dev(x["s0"]).clone()
    y0, s_out = ops.wkv6_forward(*(dev(x[n][:, :0]) for n in ("r", "k", "v", "w")),
                                 dev(x["u"]), s0=s)
    torch.cuda.synchronize()
    assert y0.numel() == 0 and torch.equal(s_out, s)
    y, s2 = ops.wkv6_forward(*(dev(x[n]) for n in ("r", "k", "v", "w")), dev(x["u"]), s0=s, sT=s)
    torch.cuda.synchronize()
    ry, rs = _ref(x, x["s0"])
    assert s2.data_ptr() == s.data_ptr()
    assert rel_inf(f64(y), ry) <= 2e-2 and rel_inf(f64(s), rs) <= 2e-2


def test_wkv6_in_place_state_of_split_sequences_over_several_waves():
    """sT == s0 with every sequence cut into 4 segments and 512 CTAs per pass (more than one
    wave at two CTAs per SM): no segment may start from an s0 that the last segment has
    already overwritten.  Bit-identical to the out-of-place call with the same split."""
    x = _inputs(4, 1024, 32, "bf16", 19, s0_std=0.1)
    y_ref, s_ref = _gpu(x, s0=x["s0"], algo="chunked", segments=4)
    s = dev(x["s0"]).clone()
    y, s_out = ops.wkv6_forward(*(dev(x[n]) for n in ("r", "k", "v", "w")), dev(x["u"]), s0=s, sT=s,
                                algo="chunked", segments=4)
    torch.cuda.synchronize()
    assert s_out.data_ptr() == s.data_ptr()
    assert torch.equal(y, y_ref) and torch.equal(s, s_ref)
    ry, rs = _ref(x, x["s0"])
    assert rel_inf(f64(y), ry) <= 2e-2 and rel_inf(f64(s), rs) <= 2e-2


@pytest.mark.parametrize("algo", ["serial", "chunked"])
def test_wkv6_extreme_decays(algo):
    """w rounded to exactly 1.0 in bf16 on some channels, tiny w (1e-30) on others."""
    x = _inputs(1, 333, 2, "bf16", 13, s0_std=0.1)
    w = x["w"].float()
    w[..., 0:8] = 0.9999          # rounds to 1.0 in bf16
    w[..., 8:16] = 1e-30          # decays to nothing within a token
    w[:, 100:140, :, 16:24] = 1e-3
    x["w"] = w.to(torch.bfloat16)
    _check(x, s0=x["s0"], algo=algo)


@pytest.mark.parametrize("wval", [0.1, 0.3])
def test_wkv6_fast_decay_channels(wval):
    """Channels whose decay product over a 64-token chunk drops below 2^-100 (w = 0.1) take
    the sub-block path; w = 0.3 stays on the chunk-end path.  Both must match the oracle."""
    x = _inputs(2, 300, 2, "bf16", 16, s0_std=0.1)
    w = x["w"].float()
    w[..., 24:40] = wval
    x["w"] = w.to(torch.bfloat16)
    _check(x, s0=x["s0"], algo="chunked")


def test_wkv6_paths_alternate_between_chunks():
    """Chunks 2, 3 and 6 hold channels with w = 0.1 (chunk decay below 2^-100: the sub-block
    path), chunk 8 a few tokens of w = 1e-30 (the exact diagonal blocks), every other chunk the
    chunk-end path.  A sub-block chunk right after a chunk-end chunk reuses the tensor-memory
    columns that held the previous chunk's P; every switch between the paths must match the
    oracle."""
    x = _inputs(2, 640, 2, "bf16", 21, s0_std=0.1)
    w = x["w"].float()
    w[:, 128:256, :, 24:32] = 0.1
    w[:, 384:448, :, 24:32] = 0.1
    w[:, 530:534, :, 40:44] = 1e-30
    x["w"] = w.to(torch.bfloat16)
    _check(x, s0=x["s0"], algo="chunked")


@pytest.mark.parametrize("segments", [1, 2, 3, 5])
def test_wkv6_sequence_split(segments):
    """The chunked kernel cut into segments (a first pass gives the end states of pieces of
    the segments, then every segment runs from its exact incoming state) matches the oracle,
    with a ragged last chunk and random s0."""
    x = _inputs(2, 1000, 2, "bf16", 17, s0_std=0.1)
    y, sT = _gpu(x, s0=x["s0"], algo="chunked", segments=segments)
    torch.cuda.synchronize()
    ry, rs = _ref(x, x["s0"])
    assert rel_inf(f64(y), ry) <= 2e-2 and rel_inf(f64(sT), rs) <= 2e-2


def test_wkv6_sequence_split_with_subblock_chunks():
    """Segments whose chunks take the sub-block path (fast-decaying channels)."""
    x = _inputs(1, 900, 2, "bf16", 18, s0_std=0.1)
    w = x["w"].float()
    w[..., 24:40] = 0.1
    x["w"] = w.to(torch.bfloat16)
    y, sT = _gpu(x, s0=x["s0"], algo="chunked", segments=4)
    torch.cuda.synchronize()
    ry, rs = _ref(x, x["s0"])
    assert rel_inf(f64(y), ry) <= 2e-2 and rel_inf(f64(sT), rs) <= 2e-2


def test_wkv6_deterministic():
    x = _inputs(2, 1000, 4, "bf16", 14, s0_std=0.1)
    a = _gpu(x, s0=x["s0"])
    b = _gpu(x, s0=x["s0"])
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_wkv6_chunked_timeout_is_reported_and_context_survives():
    """A bounded device wait that runs out (injected on the host side: a barrier nothing
    signals) must come back as RWKV_ERR_TIMEOUT through the status word, and the next
    call on the same context must be correct."""
    lib = ops.load()
    x = _inputs(1, 200, 2, "bf16", 15, s0_std=0.1)
    assert ops.device_status() == 0
    prev = lib.rwkv_debug_inject_timeout(1)
    try:
        _gpu(x, s0=x["s0"], algo="chunked")
        st = ops.device_status()
    finally:
        lib.rwkv_debug_inject_timeout(prev)
    assert st == -6, st
    _check(x, s0=x["s0"], algo="chunked")
    assert ops.device_status() == 0
