"""The allocation-free WKV-6 entry point, through the C ABI.

rwkv_wkv6_forward_bf16_noalloc serves callers that may not allocate device memory (a
serving process whose HBM is all handed to its own pool, or a runtime that forbids
allocation outside its set-up phase): it runs the chunked kernel with its sequence split,
keeping the split's scratch in a fixed device array inside the library.  These tests
check it against the fp64 oracle and, bit for bit, against the allocating entry point
rwkv_wkv6_forward_bf16 with the same split, on two calls in a row (the same kernel on the
same split must give identical bits, so leftovers of the first call in the shared array
cannot have leaked into the second); the automatic split capped to what the array holds;
an in-place state update (sT == s0) of a split sequence; and that a split larger than the
fixed array is refused before anything runs.

This file is collected last on purpose: a run that stops at the first failure has then
already run every other test.  It also passes alone in a fresh process, where the first
call performs the once-per-device set-up.
"""
import ctypes

import pytest
import torch

import oracle
from gpu_util import TOL, f64, rel_inf
from wkv_recurrence_02_b200 import inputs, ops

pytestmark = pytest.mark.gpu

RWKV_ERR_SHAPE = -2
SCRATCH_BYTES = 4 << 20  # RWKV_NOALLOC_SCRATCH_BYTES
SEG_STRIDE_BYTES = (64 * 64 + 64) * 4  # scratch per (b, h) per segment boundary


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(lib, x, s0, segments, sT=None):
    B, T, H, N = x["r"].shape
    y = torch.empty_like(x["r"])
    if sT is None:
        sT = torch.empty(B, H, N, N, device=x["r"].device, dtype=torch.float32)
    lib.rwkv_set_stream(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    rc = lib.rwkv_wkv6_forward_bf16_noalloc(B, T, H, N, _ptr(x["r"]), _ptr(x["k"]), _ptr(x["v"]),
                                            _ptr(x["w"]), _ptr(x["u"]), _ptr(s0), _ptr(y), _ptr(sT),
                                            segments)
    return rc, y, sT


def _oracle(x):
    return oracle.wkv6(*(f64(x[n]) for n in ("r", "k", "v", "w", "u")), s0=f64(x["s0"]))


def _split(nchunks, G):
    """The segment count a split into at most G segments ends with (whole segments)."""
    G = max(1, min(G, nchunks))
    per = -(-nchunks // G)
    return -(-nchunks // per)


def test_noalloc_matches_the_allocating_entry_point_on_two_calls():
    lib = ops.load()
    tol = TOL[torch.bfloat16]
    for call, seed in enumerate((31, 32)):
        x = inputs.wkv6_inputs(2, 1000, 8, 64, "bf16", seed=seed, s0_std=0.1)
        xd = {n: t.cuda() for n, t in x.items()}
        y_ref, s_ref = ops.wkv6_forward(xd["r"], xd["k"], xd["v"], xd["w"], xd["u"], s0=xd["s0"],
                                        algo="chunked", segments=4)
        rc, y, sT = _noalloc(lib, xd, xd["s0"], 4)
        assert rc == 0, (call, rc, lib.rwkv_last_error())
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref) and torch.equal(sT, s_ref), call
        ry, rs = _oracle(x)
        assert rel_inf(f64(y), ry) <= tol and rel_inf(f64(sT), rs) <= tol, call
    assert ops.device_status() == 0


def test_noalloc_automatic_split_is_capped_to_the_array():
    """segments = 0 at B2 H8 T8192: two CTAs per SM would want 18 segments (4.5 MB of
    scratch); the array holds 16.  The capped call matches the oracle and, bit for bit, the
    allocating call with the same split."""
    lib = ops.load()
    B, T, H = 2, 8192, 8
    bh, nchunks = B * H, T // 64
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    want = min(2 * sms // bh, nchunks // 4)
    cap = SCRATCH_BYTES // (SEG_STRIDE_BYTES * bh) + 1
    G = _split(nchunks, min(want, cap))
    assert (want - 1) * SEG_STRIDE_BYTES * bh > SCRATCH_BYTES and 1 < G < want
    x = inputs.wkv6_inputs(B, T, H, 64, "bf16", seed=35, s0_std=0.1)
    xd = {n: t.cuda() for n, t in x.items()}
    rc, y, sT = _noalloc(lib, xd, xd["s0"], 0)
    assert rc == 0, (rc, lib.rwkv_last_error())
    y_ref, s_ref = ops.wkv6_forward(xd["r"], xd["k"], xd["v"], xd["w"], xd["u"], s0=xd["s0"],
                                    algo="chunked", segments=G)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref) and torch.equal(sT, s_ref)
    ry, rs = _oracle(x)
    tol = TOL[torch.bfloat16]
    assert rel_inf(f64(y), ry) <= tol and rel_inf(f64(sT), rs) <= tol
    assert ops.device_status() == 0


def test_noalloc_in_place_state_of_a_split_sequence():
    """sT == s0 with 4 segments: the result equals the out-of-place call with the same split
    bit for bit (the array also keeps the copy of s0 that the segments start from)."""
    lib = ops.load()
    x = inputs.wkv6_inputs(2, 1000, 8, 64, "bf16", seed=36, s0_std=0.1)
    xd = {n: t.cuda() for n, t in x.items()}
    rc, y_ref, s_ref = _noalloc(lib, xd, xd["s0"], 4)
    assert rc == 0, (rc, lib.rwkv_last_error())
    s = xd["s0"].clone()
    rc, y, s_out = _noalloc(lib, xd, s, 4, sT=s)
    assert rc == 0, (rc, lib.rwkv_last_error())
    torch.cuda.synchronize()
    assert s_out.data_ptr() == s.data_ptr()
    assert torch.equal(y, y_ref) and torch.equal(s, s_ref)
    ry, rs = _oracle(x)
    tol = TOL[torch.bfloat16]
    assert rel_inf(f64(y), ry) <= tol and rel_inf(f64(s), rs) <= tol
    assert ops.device_status() == 0


def test_noalloc_refuses_a_split_beyond_its_fixed_array():
    """B*H*(G-1)*(N*N+N)*4 = 256 * 16640 bytes > 4 MiB for B=4, H=64 and two segments."""
    lib = ops.load()
    x = inputs.wkv6_inputs(4, 512, 64, 64, "bf16", seed=33)
    xd = {n: (t.cuda() if t is not None else None) for n, t in x.items()}
    rc, _, _ = _noalloc(lib, xd, None, 2)
    assert rc == RWKV_ERR_SHAPE
    assert b"fixed no-allocation buffer" in lib.rwkv_last_error()
    torch.cuda.synchronize()
    assert ops.device_status() == 0
