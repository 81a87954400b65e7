"""The C ABI without a GPU: the library loads, exports every declared symbol, and
rejects bad arguments on the host before touching CUDA.

Pointers passed here are fake addresses that the library must never dereference:
every call either fails validation or has nothing to compute.
"""
import ctypes

import pytest
import torch

from wkv_recurrence_02_b200 import build, ops

FAKE = 0x7F0000000000  # 16-byte aligned, never dereferenced


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ops.load()


def test_every_declared_symbol_is_exported(lib):
    names = ops.declared_functions()
    assert len(names) >= 14
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_abi_version_and_strings(lib):
    assert lib.rwkv_abi_version() == 1
    for code, name in ops.STATUS_NAMES.items():
        assert lib.rwkv_status_string(code)
    assert lib.rwkv_status_string(12345) == b"unknown status"


def _p(off=0):
    return ctypes.c_void_p(FAKE + off)


def test_wkv4_validation(lib):
    f, fb = lib.rwkv_wkv4_forward, lib.rwkv_wkv4_forward_bf16
    assert f(-1, 4, 4, _p(), _p(1 << 20), _p(2 << 20), _p(3 << 20), _p(4 << 20)) == -2
    assert f(1, 4, 4, None, _p(1 << 20), _p(2 << 20), _p(3 << 20), _p(4 << 20)) == -1
    assert f(1, 4, 4, _p(), _p(1 << 20), None, _p(3 << 20), _p(4 << 20)) == -1
    assert f(1, 4, 4, _p(4), _p(1 << 20), _p(2 << 20), _p(3 << 20), _p(4 << 20)) == -7
    # y overlapping k
    assert fb(1, 4, 4, _p(), _p(1 << 20), _p(2 << 20), _p(3 << 20), _p(2 << 20)) == -4
    # nothing to compute: OK without CUDA
    assert f(0, 4, 4, None, None, None, None, None) == 0
    assert f(3, 0, 4, None, None, None, None, None) == 0
    assert f(3, 7, 0, None, None, None, None, None) == 0
    # size product overflow
    assert f(1 << 40, 1 << 40, 4, _p(), _p(1 << 20), _p(2 << 20), _p(3 << 20), _p(4 << 20)) == -2


def test_wkv4_state_validation(lib):
    f = lib.rwkv_wkv4_forward_state
    args = [_p(), _p(1 << 20), _p(2 << 20), _p(3 << 20)]
    # sT partially overlapping s0
    assert f(2, 4, 8, *args, _p(5 << 20), _p(6 << 20), _p((5 << 20) + 16)) == -4
    # sT overlapping k
    assert f(2, 4, 8, *args, _p(5 << 20), _p(6 << 20), _p(2 << 20)) == -4
    # y overlapping s0
    assert f(2, 4, 8, *args, _p(5 << 20), _p(5 << 20), _p(7 << 20)) == -4


def test_wkv6_validation(lib):
    f = lib.rwkv_wkv6_forward_bf16
    base = [_p(i << 24) for i in range(8)]
    assert f(1, 4, 2, 32, *base) == -3            # N != 64
    assert f(1, 4, 2, -64, *base) == -2
    assert f(1, 4, 2, 64, None, *base[1:]) == -1  # r null
    bad = list(base)
    bad[2] = _p((2 << 24) + 8)
    assert f(1, 4, 2, 64, *bad) == -7             # misaligned v
    alias = list(base)
    alias[6] = base[0]                            # y == r
    assert f(1, 4, 2, 64, *alias) == -4
    part = list(base)
    part[7] = _p((5 << 24) + 64)                  # sT inside s0, not equal
    assert f(1, 4, 2, 64, *part) == -4
    assert f(0, 4, 2, 64, *([None] * 8)) == 0     # empty: OK without CUDA
    assert f(2, 4, 0, 64, *([None] * 8)) == 0


def test_wkv6_gated_validation(lib):
    """Gate, LayerNorm parameters and eps are checked on the host like the other tensors."""
    f = lib.rwkv_wkv6_forward_gated_bf16
    r, k, v, w, u, s0, g, lw, lb, y, sT = (_p(i << 24) for i in range(11))

    def call(eps=1e-5, **kw):
        a = dict(r=r, k=k, v=v, w=w, u=u, s0=s0, g=g, lw=lw, lb=lb, y=y, sT=sT)
        a.update(kw)
        return f(1, 4, 2, 64, a["r"], a["k"], a["v"], a["w"], a["u"], a["s0"], a["g"], a["lw"], a["lb"],
                 ctypes.c_float(eps), a["y"], a["sT"])

    assert call(g=None) == -1                     # gate null
    assert call(lw=None) == -1                    # LayerNorm scale null
    assert call(lb=None) == -1
    assert call(eps=-1.0) == -8                   # eps < 0
    assert call(eps=float("nan")) == -8
    assert call(g=_p((6 << 24) + 4)) == -7        # misaligned gate
    assert call(y=g) == -4                        # y == g
    assert call(sT=lw) == -4                      # sT over the LayerNorm scale
    assert f(0, 4, 2, 64, *([None] * 9), ctypes.c_float(1e-5), None, None) == 0  # empty


def test_wkv6_omega_validation(lib):
    """The logit entry: the output-stage trio is all-or-nothing, eps is checked only with the
    gate, and the logit is an input like w."""
    f = lib.rwkv_wkv6_forward_omega_bf16
    r, k, v, om, u, s0, g, lw, lb, y, sT = (_p(i << 24) for i in range(11))

    def call(eps=1e-5, **kw):
        a = dict(r=r, k=k, v=v, om=om, u=u, s0=s0, g=g, lw=lw, lb=lb, y=y, sT=sT)
        a.update(kw)
        return f(1, 4, 2, 64, a["r"], a["k"], a["v"], a["om"], a["u"], a["s0"], a["g"], a["lw"], a["lb"],
                 ctypes.c_float(eps), a["y"], a["sT"])

    assert call(om=None) == -1                     # logit null
    assert call(g=None) == -1                      # gate missing, LayerNorm given
    assert call(g=None, lw=None) == -1             # shift alone
    assert call(lw=None, lb=None) == -1            # gate alone
    assert call(eps=-1.0) == -8                    # eps < 0 with the gate
    assert call(om=_p((3 << 24) + 8)) == -7        # misaligned logit
    assert call(y=om) == -4                        # y == omega
    assert call(sT=_p((3 << 24) + 512)) == -4      # sT over the logit
    assert f(2, 4, 0, 64, *([None] * 9), ctypes.c_float(1e-5), None, None) == 0  # empty
    if not torch.cuda.is_available():
        # without the gate, eps is ignored: a valid call gets as far as CUDA
        assert call(g=None, lw=None, lb=None, eps=-1.0) == -5


def test_wkv6_backward_validation(lib):
    """The backward's host checks: workspace size, nulls, alignment and aliasing."""
    f = lib.rwkv_wkv6_backward_bf16
    names = ["r", "k", "v", "w", "u", "s0", "dy", "dsT", "dr", "dk", "dv", "dw", "du", "ds0", "ws"]
    B, T, H = 1, 20, 2
    need = ops.wkv6_backward_workspace_bytes(B, T, H)
    bh, nblk, nch = B * H, 3, 1  # ceil(20 / 8) walk checkpoints, ceil(20 / 64) chunks per (b, h)
    walks = bh * nblk * 64 * 64 * 4                       # fp32 state every 8 tokens
    chunked = bh * ((nch + 1) + nch) * 64 * 64 * 2 + bh * nch * 64 * 4  # bf16 states, row dots
    assert need == max(walks, chunked) + bh * 64 * 4 + bh * nch * 64 * 4 + 16  # du shares, flags
    assert ops.wkv6_backward_workspace_bytes(B, 0, H) == 0
    with pytest.raises(ops.WkvError):
        ops.wkv6_backward_workspace_bytes(-1, T, H)
    with pytest.raises(ops.WkvError):  # checkpoint count x 64 x 64 overflows
        ops.wkv6_backward_workspace_bytes(1, 1 << 56, 1, 1)

    def call(wbytes=need, **kw):
        a = {n: _p(i << 24) for i, n in enumerate(names)}
        a.update(kw)
        return f(B, T, H, 64, *[a[n] for n in names], ctypes.c_size_t(wbytes))

    assert call(wbytes=need - 1) == -8            # workspace too small
    assert call(ws=None) == -1                    # workspace missing
    assert call(dy=None) == -1
    assert call(dw=None) == -1
    assert call(du=None) == -1
    assert call(dr=_p((8 << 24) + 8)) == -7       # misaligned gradient
    assert call(ws=_p((14 << 24) + 4)) == -7      # misaligned workspace
    assert call(dk=_p(1 << 24)) == -4             # dk over k
    assert call(ws=_p(8 << 24)) == -4             # workspace over dr
    assert call(du=_p((9 << 24) + 64)) == -4      # du inside dk
    assert call(ds0=_p(7 << 24)) != -4            # ds0 == dsT is allowed (in place)
    assert call(ds0=_p((7 << 24) + 16)) == -4     # but not a partial overlap
    assert f(B, T, H, 32, *[_p(i << 24) for i in range(15)], ctypes.c_size_t(need)) == -3
    assert f(0, T, 0, 64, *([None] * 15), ctypes.c_size_t(0)) == 0  # nothing to produce


def test_algo_selection(lib):
    assert lib.rwkv_set_wkv6_algo(7) == -8
    for a in (1, 2, 0):
        assert lib.rwkv_set_wkv6_algo(a) == 0
        assert lib.rwkv_get_wkv6_algo() == a


def test_stream_is_thread_local_setting(lib):
    lib.rwkv_set_stream(ctypes.c_void_p(0x1234))
    assert lib.rwkv_get_stream() == 0x1234
    lib.rwkv_set_stream(None)
    assert not lib.rwkv_get_stream()


@pytest.mark.skipif(torch.cuda.is_available(), reason="only meaningful without a GPU")
def test_valid_call_without_gpu_fails_cleanly(lib):
    """With no CUDA device a valid call must return RWKV_ERR_CUDA, not crash or fall back."""
    rc = lib.rwkv_wkv4_forward(1, 4, 16, _p(), _p(1 << 20), _p(2 << 20), _p(3 << 20), _p(4 << 20))
    assert rc == -5
    assert lib.rwkv_last_error()


def test_binding_refuses_cpu_tensors(lib):
    k = torch.zeros(1, 4, 16)
    with pytest.raises(TypeError):
        ops.wkv4_forward(torch.zeros(16), torch.zeros(16), k, k)
