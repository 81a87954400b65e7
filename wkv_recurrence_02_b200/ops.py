"""Thin ctypes binding of libwkv.so (include/rwkv_wkv.h) for torch CUDA tensors.

Argument marshalling only: every step of the recurrences runs in the library's CUDA
kernels.  There is no CPU fallback -- if the library is not built, or a tensor is
not on a CUDA device, the call raises.

Functions mirror the C entry points:
  wkv4_forward(w, u, k, v, s0=None, want_state=False)   -> y            | (y, sT)
  wkv6_forward(r, k, v, w, u, s0=None, want_state=True) -> (y, sT)      | y
The calls are asynchronous on torch's current CUDA stream.
"""
import contextlib
import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libwkv.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "rwkv_wkv.h")

RWKV_OK = 0
STATUS_NAMES = {0: "RWKV_OK", -1: "RWKV_ERR_NULL", -2: "RWKV_ERR_SHAPE", -3: "RWKV_ERR_UNSUPPORTED",
                -4: "RWKV_ERR_ALIAS", -5: "RWKV_ERR_CUDA", -6: "RWKV_ERR_TIMEOUT",
                -7: "RWKV_ERR_ALIGN", -8: "RWKV_ERR_ARG", -9: "RWKV_ERR_BOUNDS"}
ALGOS = {"auto": 0, "serial": 1, "chunked": 2}

_i64 = ctypes.c_int64
_vp = ctypes.c_void_p
_lib = None


class WkvError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


def declared_functions(header: str = HEADER):
    """Names of the functions include/rwkv_wkv.h declares."""
    with open(header) as f:
        text = f.read()
    return sorted(set(re.findall(r"\b(rwkv_[a-z0-9_]+)\s*\(", text)))


def load(path: str = LIB_PATH):
    """Load libwkv.so (once) and declare its signatures.  Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is not built: run `python -m wkv_recurrence_02_b200.build`")
    lib = ctypes.CDLL(path)
    wkv4 = [_i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp]
    wkv4s = [_i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
    wkv6 = [_i64, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
    for name, args in [("rwkv_wkv4_forward", wkv4), ("rwkv_wkv4_forward_bf16", wkv4),
                       ("rwkv_wkv4_forward_state", wkv4s), ("rwkv_wkv4_forward_state_bf16", wkv4s),
                       ("rwkv_wkv6_forward", wkv6), ("rwkv_wkv6_forward_bf16", wkv6)]:
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    lib.rwkv_set_stream.argtypes = [_vp]
    lib.rwkv_set_stream.restype = None
    lib.rwkv_get_stream.argtypes = []
    lib.rwkv_get_stream.restype = _vp
    lib.rwkv_set_wkv6_algo.argtypes = [ctypes.c_int]
    lib.rwkv_set_wkv6_algo.restype = ctypes.c_int
    lib.rwkv_get_wkv6_algo.argtypes = []
    lib.rwkv_get_wkv6_algo.restype = ctypes.c_int
    lib.rwkv_wkv6_forward_bf16_noalloc.argtypes = wkv6 + [ctypes.c_int]
    lib.rwkv_wkv6_forward_gated_bf16.argtypes = wkv6[:10] + [_vp, _vp, _vp, ctypes.c_float] + wkv6[10:]
    lib.rwkv_wkv6_forward_gated_bf16.restype = ctypes.c_int
    lib.rwkv_wkv6_forward_omega_bf16.argtypes = wkv6[:10] + [_vp, _vp, _vp, ctypes.c_float] + wkv6[10:]
    lib.rwkv_wkv6_forward_omega_bf16.restype = ctypes.c_int
    bwd = [_i64] * 4 + [_vp] * 14 + [_vp, ctypes.c_size_t]
    for name in ("rwkv_wkv6_backward", "rwkv_wkv6_backward_bf16", "rwkv_wkv6_backward_omega_bf16"):
        fn = getattr(lib, name)
        fn.argtypes = bwd
        fn.restype = ctypes.c_int
    lib.rwkv_wkv6_backward_workspace_bytes.argtypes = [_i64] * 4 + [ctypes.POINTER(ctypes.c_size_t)]
    lib.rwkv_wkv6_backward_workspace_bytes.restype = ctypes.c_int
    lib.rwkv_wkv6_forward_bf16_noalloc.restype = ctypes.c_int
    lib.rwkv_set_wkv6_segments.argtypes = [ctypes.c_int]
    lib.rwkv_set_wkv6_segments.restype = ctypes.c_int
    lib.rwkv_get_wkv6_segments.argtypes = []
    lib.rwkv_get_wkv6_segments.restype = ctypes.c_int
    lib.rwkv_debug_inject_timeout.argtypes = [ctypes.c_int]
    lib.rwkv_debug_inject_timeout.restype = ctypes.c_int
    lib.rwkv_get_device_status.argtypes = []
    lib.rwkv_get_device_status.restype = ctypes.c_int
    lib.rwkv_status_string.argtypes = [ctypes.c_int]
    lib.rwkv_status_string.restype = ctypes.c_char_p
    lib.rwkv_last_error.argtypes = []
    lib.rwkv_last_error.restype = ctypes.c_char_p
    lib.rwkv_abi_version.argtypes = []
    lib.rwkv_abi_version.restype = ctypes.c_int
    lib.rwkv_debug_bounds.argtypes = []
    lib.rwkv_debug_bounds.restype = ctypes.c_int
    _lib = lib
    return lib


@contextlib.contextmanager
def using_library(path: str):
    """Route the calls of this module to another build of the library (e.g. the bounds-checked
    debug build, libwkv_debug.so) inside the block; the default library is restored after."""
    global _lib
    prev = _lib
    _lib = None
    try:
        yield load(path)
    finally:
        _lib = prev


def _check(rc):
    if rc != RWKV_OK:
        lib = load()
        raise WkvError(rc, (lib.rwkv_last_error() or b"").decode() or
                       lib.rwkv_status_string(rc).decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _cuda(t, name, dtype=None, shape=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _use_current_stream(lib, device):
    lib.rwkv_set_stream(ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream))


def wkv4_forward(w, u, k, v, s0=None, want_state=False, y=None, sT=None):
    """RWKV-4 WKV.  k, v: [B,T,C] fp32|bf16; w, u: [C] fp32; s0: [B,3,C] fp32 or None."""
    lib = load()
    _cuda(k, "k")
    B, T, C = k.shape
    dt = k.dtype
    if dt not in (torch.float32, torch.bfloat16):
        raise TypeError("k must be float32 or bfloat16")
    _cuda(v, "v", dt, (B, T, C))
    _cuda(w, "w", torch.float32, (C,))
    _cuda(u, "u", torch.float32, (C,))
    _cuda(s0, "s0", torch.float32, (B, 3, C))
    if y is None:
        y = torch.empty_like(k)
    _cuda(y, "y", dt, (B, T, C))
    stateful = want_state or s0 is not None or sT is not None
    if stateful and sT is None and want_state:
        sT = torch.empty(B, 3, C, device=k.device, dtype=torch.float32)
    _cuda(sT, "sT", torch.float32, (B, 3, C))
    _use_current_stream(lib, k.device)
    bf = dt == torch.bfloat16
    if stateful:
        fn = lib.rwkv_wkv4_forward_state_bf16 if bf else lib.rwkv_wkv4_forward_state
        _check(fn(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(s0), _ptr(y), _ptr(sT)))
    else:
        fn = lib.rwkv_wkv4_forward_bf16 if bf else lib.rwkv_wkv4_forward
        _check(fn(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(y)))
    return (y, sT) if want_state else y


def wkv6_forward(r, k, v, w, u, s0=None, want_state=True, y=None, sT=None, algo=None,
                 segments=None):
    """Eagle/Finch WKV-6.  r,k,v,w: [B,T,H,N] fp32|bf16; u: [H,N] fp32; s0: [B,H,N,N] fp32.

    algo: None (library default), "auto", "serial" or "chunked" (this call only).
    segments: None (library default), 0 (auto), 1 (no sequence split) or n (at most n).
    """
    lib = load()
    _cuda(r, "r")
    B, T, H, N = r.shape
    dt = r.dtype
    if dt not in (torch.float32, torch.bfloat16):
        raise TypeError("r must be float32 or bfloat16")
    for name, t in (("k", k), ("v", v), ("w", w)):
        _cuda(t, name, dt, (B, T, H, N))
    _cuda(u, "u", torch.float32, (H, N))
    _cuda(s0, "s0", torch.float32, (B, H, N, N))
    if y is None:
        y = torch.empty_like(r)
    _cuda(y, "y", dt, (B, T, H, N))
    if sT is None and want_state:
        sT = torch.empty(B, H, N, N, device=r.device, dtype=torch.float32)
    _cuda(sT, "sT", torch.float32, (B, H, N, N))
    _use_current_stream(lib, r.device)
    fn = lib.rwkv_wkv6_forward_bf16 if dt == torch.bfloat16 else lib.rwkv_wkv6_forward
    prev = prev_seg = None
    if algo is not None:
        prev = lib.rwkv_get_wkv6_algo()
        _check(lib.rwkv_set_wkv6_algo(ALGOS[algo]))
    if segments is not None:
        prev_seg = lib.rwkv_get_wkv6_segments()
        _check(lib.rwkv_set_wkv6_segments(int(segments)))
    try:
        _check(fn(B, T, H, N, _ptr(r), _ptr(k), _ptr(v), _ptr(w), _ptr(u), _ptr(s0), _ptr(y),
                  _ptr(sT)))
    finally:
        if prev is not None:
            lib.rwkv_set_wkv6_algo(prev)
        if prev_seg is not None:
            lib.rwkv_set_wkv6_segments(prev_seg)
    return (y, sT) if want_state else y


def wkv6_forward_gated(r, k, v, w, u, g, ln_w, ln_b, eps=1e-5, s0=None, want_state=True, y=None,
                       sT=None):
    """WKV-6 (bf16) with the fused output stage: y = SiLU(g) * LayerNorm_head(o; ln_w, ln_b, eps).

    r,k,v,w,g: [B,T,H,N] bf16; u, ln_w, ln_b: [H,N] fp32; s0: [B,H,N,N] fp32.
    """
    lib = load()
    _cuda(r, "r", torch.bfloat16)
    B, T, H, N = r.shape
    for name, t in (("k", k), ("v", v), ("w", w), ("g", g)):
        _cuda(t, name, torch.bfloat16, (B, T, H, N))
    for name, t in (("u", u), ("ln_w", ln_w), ("ln_b", ln_b)):
        _cuda(t, name, torch.float32, (H, N))
    _cuda(s0, "s0", torch.float32, (B, H, N, N))
    if y is None:
        y = torch.empty_like(r)
    _cuda(y, "y", torch.bfloat16, (B, T, H, N))
    if sT is None and want_state:
        sT = torch.empty(B, H, N, N, device=r.device, dtype=torch.float32)
    _cuda(sT, "sT", torch.float32, (B, H, N, N))
    _use_current_stream(lib, r.device)
    _check(lib.rwkv_wkv6_forward_gated_bf16(B, T, H, N, _ptr(r), _ptr(k), _ptr(v), _ptr(w), _ptr(u),
                                             _ptr(s0), _ptr(g), _ptr(ln_w), _ptr(ln_b), float(eps),
                                             _ptr(y), _ptr(sT)))
    return (y, sT) if want_state else y


def wkv6_forward_omega(r, k, v, omega, u, s0=None, g=None, ln_w=None, ln_b=None, eps=1e-5,
                       want_state=True, y=None, sT=None, algo=None):
    """WKV-6 (bf16) fed the decay logit omega_t; the kernels form w_t = exp(-exp(omega_t)).

    r,k,v,omega (and g): [B,T,H,N] bf16; u (and ln_w, ln_b): [H,N] fp32; s0: [B,H,N,N] fp32.
    With g, ln_w and ln_b the fused head LayerNorm + SiLU gate is applied as in
    wkv6_forward_gated.  algo (plain output only): as in wkv6_forward.
    """
    lib = load()
    _cuda(r, "r", torch.bfloat16)
    B, T, H, N = r.shape
    for name, t in (("k", k), ("v", v), ("omega", omega), ("g", g)):
        _cuda(t, name, torch.bfloat16, (B, T, H, N))
    for name, t in (("u", u), ("ln_w", ln_w), ("ln_b", ln_b)):
        _cuda(t, name, torch.float32, (H, N))
    _cuda(s0, "s0", torch.float32, (B, H, N, N))
    if y is None:
        y = torch.empty_like(r)
    _cuda(y, "y", torch.bfloat16, (B, T, H, N))
    if sT is None and want_state:
        sT = torch.empty(B, H, N, N, device=r.device, dtype=torch.float32)
    _cuda(sT, "sT", torch.float32, (B, H, N, N))
    _use_current_stream(lib, r.device)
    prev = None
    if algo is not None:
        prev = lib.rwkv_get_wkv6_algo()
        _check(lib.rwkv_set_wkv6_algo(ALGOS[algo]))
    try:
        _check(lib.rwkv_wkv6_forward_omega_bf16(B, T, H, N, _ptr(r), _ptr(k), _ptr(v), _ptr(omega),
                                                 _ptr(u), _ptr(s0), _ptr(g), _ptr(ln_w), _ptr(ln_b),
                                                 float(eps), _ptr(y), _ptr(sT)))
    finally:
        if prev is not None:
            lib.rwkv_set_wkv6_algo(prev)
    return (y, sT) if want_state else y


def wkv6_backward_workspace_bytes(B, T, H, N=64) -> int:
    """Device scratch (bytes) that a WKV-6 backward call of this shape needs."""
    lib = load()
    out = ctypes.c_size_t(0)
    _check(lib.rwkv_wkv6_backward_workspace_bytes(int(B), int(T), int(H), int(N), ctypes.byref(out)))
    return int(out.value)


def wkv6_backward(r, k, v, w, u, dy, s0=None, dsT=None, omega=False, want_ds0=True, workspace=None,
                  algo=None):
    """WKV-6 backward: gradients of a loss with dL/dy = dy and dL/dsT = dsT (None = 0).

    r,k,v,w,dy: [B,T,H,N] fp32|bf16 (with omega=True, w holds omega_t and bf16 is required);
    u: [H,N] fp32; s0, dsT: [B,H,N,N] fp32.  Returns a dict of fp32 tensors dr, dk, dv,
    dw (or domega), du, and ds0 (when want_ds0).  workspace: optional uint8 CUDA tensor of at
    least wkv6_backward_workspace_bytes bytes; allocated here when not given.
    algo: None (library default: bf16 inputs take the chunked tensor-core path), "auto",
    "serial" (the exact fp32 walks) or "chunked" (this call only).
    """
    lib = load()
    _cuda(r, "r")
    B, T, H, N = r.shape
    dt = r.dtype
    if dt not in (torch.float32, torch.bfloat16):
        raise TypeError("r must be float32 or bfloat16")
    if omega and dt != torch.bfloat16:
        raise TypeError("the logit backward takes bf16 inputs")
    for name, t in (("k", k), ("v", v), ("w", w), ("dy", dy)):
        _cuda(t, name, dt, (B, T, H, N))
    _cuda(u, "u", torch.float32, (H, N))
    _cuda(s0, "s0", torch.float32, (B, H, N, N))
    _cuda(dsT, "dsT", torch.float32, (B, H, N, N))
    dev = r.device
    out = {n: torch.empty(B, T, H, N, device=dev, dtype=torch.float32) for n in ("dr", "dk", "dv")}
    dwn = "domega" if omega else "dw"
    out[dwn] = torch.empty(B, T, H, N, device=dev, dtype=torch.float32)
    out["du"] = torch.empty(H, N, device=dev, dtype=torch.float32)
    out["ds0"] = torch.empty(B, H, N, N, device=dev, dtype=torch.float32) if want_ds0 else None
    need = wkv6_backward_workspace_bytes(B, T, H, N)
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=dev, dtype=torch.uint8)
    _cuda(workspace, "workspace", torch.uint8)
    _use_current_stream(lib, dev)
    fn = (lib.rwkv_wkv6_backward_omega_bf16 if omega else
          lib.rwkv_wkv6_backward_bf16 if dt == torch.bfloat16 else lib.rwkv_wkv6_backward)
    prev = None
    if algo is not None:
        prev = lib.rwkv_get_wkv6_algo()
        _check(lib.rwkv_set_wkv6_algo(ALGOS[algo]))
    try:
        _check(fn(B, T, H, N, _ptr(r), _ptr(k), _ptr(v), _ptr(w), _ptr(u), _ptr(s0), _ptr(dy), _ptr(dsT),
                  _ptr(out["dr"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out[dwn]), _ptr(out["du"]),
                  _ptr(out["ds0"]), _ptr(workspace), ctypes.c_size_t(workspace.numel())))
    finally:
        if prev is not None:
            lib.rwkv_set_wkv6_algo(prev)
    if not want_ds0:
        del out["ds0"]
    return out


def device_status() -> int:
    """Synchronise the current stream and return/clear the device status word."""
    lib = load()
    _use_current_stream(lib, torch.cuda.current_device())
    return int(lib.rwkv_get_device_status())
