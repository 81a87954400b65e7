"""The allocation-free WKV-6 entry point, through the C ABI.

rwkv_wkv6_forward_bf16_noalloc serves callers that may not allocate device memory (a
serving process whose HBM is all handed to its own pool, or a runtime that forbids
allocation outside its set-up phase): it runs the chunked kernel with its sequence split,
keeping the split's scratch in a fixed device array inside the library.  These tests
check it against the allocating entry point rwkv_wkv6_forward_bf16 on two calls in a row
(so leftovers from the first call cannot leak into the second), and that a split larger
than the fixed array is refused before anything runs.

This file is collected last on purpose: a run that stops at the first failure has then
already run every other test.  It also passes alone in a fresh process, where the first
call performs the once-per-device set-up.
"""
import ctypes

import pytest
import torch

from gpu_util import TOL, f64, rel_inf
from wkv_recurrence_02_b200 import inputs, ops

pytestmark = pytest.mark.gpu

RWKV_ERR_SHAPE = -2


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(lib, x, s0, segments):
    B, T, H, N = x["r"].shape
    y = torch.empty_like(x["r"])
    sT = torch.empty(B, H, N, N, device=x["r"].device, dtype=torch.float32)
    lib.rwkv_set_stream(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    rc = lib.rwkv_wkv6_forward_bf16_noalloc(B, T, H, N, _ptr(x["r"]), _ptr(x["k"]), _ptr(x["v"]),
                                            _ptr(x["w"]), _ptr(x["u"]), _ptr(s0), _ptr(y), _ptr(sT),
                                            segments)
    return rc, y, sT


def test_noalloc_matches_the_allocating_entry_point_on_two_calls():
    lib = ops.load()
    for call, seed in enumerate((31, 32)):
        x = inputs.wkv6_inputs(2, 1000, 8, 64, "bf16", seed=seed, s0_std=0.1)
        xd = {n: t.cuda() for n, t in x.items()}
        y_ref, s_ref = ops.wkv6_forward(xd["r"], xd["k"], xd["v"], xd["w"], xd["u"], s0=xd["s0"],
                                        algo="chunked", segments=4)
        rc, y, sT = _noalloc(lib, xd, xd["s0"], 4)
        assert rc == 0, (call, rc, lib.rwkv_last_error())
        torch.cuda.synchronize()
        tol = TOL[torch.bfloat16]
        assert rel_inf(f64(y), f64(y_ref)) <= tol, call
        assert rel_inf(f64(sT), f64(s_ref)) <= tol, call
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
