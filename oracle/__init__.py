"""fp64 CPU oracle for the WKV recurrences -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py (its CPU-baseline leg and its
reference arm) may import this package.  The CUDA product path never imports,
calls or links it, and nothing here imports the product package.

The arithmetic lives in wkv_oracle.c (plain C, fp64, serial per unit); this
module only marshals numpy arrays through ctypes.  Inputs are widened to
float64 exactly (bf16 and fp32 values convert without rounding).

Sources:
  * WKV-4: "RWKV: Reinventing RNNs for the Transformer Era" (Chinese
    translation), eq. 14 as referenced in the sections on temporal structure
    (decay e^{-w}, bonus e^{u}) and gradient stability (single-step
    time-dependent softmax).
  * WKV-6: "RWKV-5/6 (Eagle and Finch)" summary, sections 4 (row-vector
    convention), 4.1.2 (Eagle time mixing) and 4.2.2 (Finch per-token decay).
  * Head LayerNorm and SiLU gate on the WKV-6 output: the same summary, section 4
    (architecture overview: LayerNorm on the heads, SiLU attention gating) and 4.1.2
    (the LayerNorm acts on each head separately, i.e. GroupNorm over the heads).
  * Decay from its logit, w = exp(-exp(omega)): the same summary, section 4.1.2
    (Eagle: omega is the trainable per-head parameter) and 4.2.2 (Finch: w_t varies
    per token; section 4.2.1 gives the LoRA offset that makes omega_t per token).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_HERE = os.path.dirname(os.path.abspath(__file__))
_DP = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.c_int64


class Oracle:
    """ctypes handle on one compiled copy of the oracle library."""

    def __init__(self, lib_path: str):
        self.path = lib_path
        lib = ctypes.CDLL(lib_path)
        lib.oracle_wkv4.argtypes = [_I64, _I64, _I64, _DP, _DP, _DP, _DP, _DP, _DP, _DP]
        lib.oracle_wkv4.restype = None
        lib.oracle_wkv6.argtypes = [_I64, _I64, _I64, _I64, _DP, _DP, _DP, _DP, _DP,
                                    _DP, _DP, _DP, _DP]
        lib.oracle_head_norm_gate.argtypes = [_I64, _I64, _I64, _I64, _DP, _DP, _DP, _DP,
                                              ctypes.c_double, _DP]
        lib.oracle_head_norm_gate.restype = None
        lib.oracle_decay_from_logit.argtypes = [_I64, _DP, _DP]
        lib.oracle_decay_from_logit.restype = None
        lib.oracle_decay_from_logit_grad.argtypes = [_I64, _DP, _DP, _DP]
        lib.oracle_decay_from_logit_grad.restype = None
        lib.oracle_wkv6_backward.argtypes = [_I64, _I64, _I64, _I64] + [_DP] * 15
        lib.oracle_wkv6_backward.restype = None
        lib.oracle_wkv6.restype = None
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_set_threads.restype = ctypes.c_int
        self._lib = lib

    def set_threads(self, n: int = 0) -> int:
        """Set the OpenMP thread count (n <= 0 keeps it); returns the count in use."""
        return int(self._lib.oracle_set_threads(int(n)))

    @staticmethod
    def _f64(x):
        a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
        return a, a.ctypes.data_as(_DP)

    def wkv4(self, w, u, k, v, s0=None, want_state=False):
        """WKV-4 forward.  k, v: [B,T,C]; w, u: [C]; s0: [B,3,C] (a,b,p) or None.

        Returns y [B,T,C] (float64), and also sT [B,3,C] when want_state.
        """
        k, kp = self._f64(k)
        v, vp = self._f64(v)
        w, wp = self._f64(w)
        u, up = self._f64(u)
        B, T, C = k.shape
        assert v.shape == k.shape and w.shape == (C,) and u.shape == (C,)
        y = np.empty((B, T, C), np.float64)
        sT = np.empty((B, 3, C), np.float64) if want_state else None
        if s0 is not None:
            s0, s0p = self._f64(s0)
            assert s0.shape == (B, 3, C)
        else:
            s0p = None
        self._lib.oracle_wkv4(B, T, C, wp, up, kp, vp, s0p, y.ctypes.data_as(_DP),
                              sT.ctypes.data_as(_DP) if sT is not None else None)
        return (y, sT) if want_state else y

    def wkv6(self, r, k, v, w, u, s0=None):
        """WKV-6 forward.  r,k,v,w: [B,T,H,N]; u: [H,N]; s0: [B,H,N,N] or None.

        Returns (y [B,T,H,N], sT [B,H,N,N]) in float64.
        """
        r, rp = self._f64(r)
        k, kp = self._f64(k)
        v, vp = self._f64(v)
        w, wp = self._f64(w)
        u, up = self._f64(u)
        B, T, H, N = r.shape
        for x in (k, v, w):
            assert x.shape == (B, T, H, N)
        assert u.shape == (H, N)
        if s0 is not None:
            s0, s0p = self._f64(s0)
            assert s0.shape == (B, H, N, N)
        else:
            s0p = None
        y = np.empty((B, T, H, N), np.float64)
        sT = np.empty((B, H, N, N), np.float64)
        work = np.empty((B, H, N, N), np.float64)
        self._lib.oracle_wkv6(B, T, H, N, rp, kp, vp, wp, up, s0p, y.ctypes.data_as(_DP),
                              sT.ctypes.data_as(_DP), work.ctypes.data_as(_DP))
        return y, sT


    def head_norm_gate(self, o, g, ln_w, ln_b, eps):
        """y = SiLU(g) * (ln_w * (o - mean) / sqrt(var + eps) + ln_b) per (b, t, head).

        o, g: [B,T,H,N]; ln_w, ln_b: [H,N].  Returns y [B,T,H,N] in float64.
        """
        o, op = self._f64(o)
        g, gp = self._f64(g)
        ln_w, wp = self._f64(ln_w)
        ln_b, bp = self._f64(ln_b)
        B, T, H, N = o.shape
        assert g.shape == o.shape and ln_w.shape == (H, N) and ln_b.shape == (H, N)
        y = np.empty_like(o)
        self._lib.oracle_head_norm_gate(B, T, H, N, op, gp, wp, bp, float(eps), y.ctypes.data_as(_DP))
        return y

    def wkv6_gated(self, r, k, v, w, u, g, ln_w, ln_b, eps, s0=None):
        """WKV-6 forward followed by the head LayerNorm and SiLU gate: (y, sT)."""
        o, sT = self.wkv6(r, k, v, w, u, s0=s0)
        return self.head_norm_gate(o, g, ln_w, ln_b, eps), sT

    def decay_from_logit(self, omega):
        """w = exp(-exp(omega)) elementwise (any shape), in float64."""
        omega, op = self._f64(omega)
        w = np.empty_like(omega)
        self._lib.oracle_decay_from_logit(omega.size, op, w.ctypes.data_as(_DP))
        return w

    def decay_from_logit_grad(self, omega, dw):
        """dL/domega from dL/dw through w = exp(-exp(omega)), elementwise, in float64."""
        omega, op = self._f64(omega)
        dw, dp = self._f64(dw)
        assert dw.shape == omega.shape
        out = np.empty_like(omega)
        self._lib.oracle_decay_from_logit_grad(omega.size, op, dp, out.ctypes.data_as(_DP))
        return out

    def wkv6_backward(self, r, k, v, w, u, dy, s0=None, dsT=None):
        """WKV-6 backward: given dL/dy (and dL/dsT, None = 0), returns the dict of float64
        gradients dr, dk, dv, dw [B,T,H,N], du [H,N] and ds0 [B,H,N,N]."""
        r, rp = self._f64(r)
        k, kp = self._f64(k)
        v, vp = self._f64(v)
        w, wp = self._f64(w)
        u, up = self._f64(u)
        dy, gp = self._f64(dy)
        B, T, H, N = r.shape
        for x in (k, v, w, dy):
            assert x.shape == (B, T, H, N)
        assert u.shape == (H, N)
        s0p = dsp = None
        if s0 is not None:
            s0, s0p = self._f64(s0)
            assert s0.shape == (B, H, N, N)
        if dsT is not None:
            dsT, dsp = self._f64(dsT)
            assert dsT.shape == (B, H, N, N)
        out = {n: np.empty((B, T, H, N), np.float64) for n in ("dr", "dk", "dv", "dw")}
        out["du"] = np.empty((H, N), np.float64)
        out["ds0"] = np.empty((B, H, N, N), np.float64)
        work = np.empty(H * (T + 1) * N * N + H * N * N, np.float64)
        p = lambda a: a.ctypes.data_as(_DP)  # noqa: E731
        self._lib.oracle_wkv6_backward(B, T, H, N, rp, kp, vp, wp, up, s0p, gp, dsp, p(out["dr"]), p(out["dk"]),
                                       p(out["dv"]), p(out["dw"]), p(out["du"]), p(out["ds0"]), p(work))
        return out

    def wkv6_logit_backward(self, r, k, v, omega, u, dy, s0=None, dsT=None):
        """Backward of wkv6_logit (plain output): as wkv6_backward, with domega in place of dw."""
        out = self.wkv6_backward(r, k, v, self.decay_from_logit(omega), u, dy, s0=s0, dsT=dsT)
        out["domega"] = self.decay_from_logit_grad(omega, out.pop("dw"))
        return out

    def wkv6_logit(self, r, k, v, omega, u, s0=None, g=None, ln_w=None, ln_b=None, eps=1e-5):
        """WKV-6 with the decay given by its logit omega_t (w_t = exp(-exp(omega_t))): (y, sT).

        With g, ln_w and ln_b the head LayerNorm and SiLU gate follow, as in wkv6_gated.
        """
        w = self.decay_from_logit(omega)
        if g is None:
            return self.wkv6(r, k, v, w, u, s0=s0)
        return self.wkv6_gated(r, k, v, w, u, g, ln_w, ln_b, eps, s0=s0)


_DEFAULT = None


def get() -> Oracle:
    """The oracle built from oracle/wkv_oracle.c (compiled on first use if needed)."""
    global _DEFAULT
    if _DEFAULT is None:
        if not _build.up_to_date():
            _build.build()
        _DEFAULT = Oracle(_build.LIB)
    return _DEFAULT


def wkv4(w, u, k, v, s0=None, want_state=False):
    return get().wkv4(w, u, k, v, s0=s0, want_state=want_state)


def wkv6(r, k, v, w, u, s0=None):
    return get().wkv6(r, k, v, w, u, s0=s0)


def head_norm_gate(o, g, ln_w, ln_b, eps):
    return get().head_norm_gate(o, g, ln_w, ln_b, eps)


def wkv6_gated(r, k, v, w, u, g, ln_w, ln_b, eps, s0=None):
    return get().wkv6_gated(r, k, v, w, u, g, ln_w, ln_b, eps, s0=s0)


def decay_from_logit(omega):
    return get().decay_from_logit(omega)


def decay_from_logit_grad(omega, dw):
    return get().decay_from_logit_grad(omega, dw)


def wkv6_backward(r, k, v, w, u, dy, s0=None, dsT=None):
    return get().wkv6_backward(r, k, v, w, u, dy, s0=s0, dsT=dsT)


def wkv6_logit_backward(r, k, v, omega, u, dy, s0=None, dsT=None):
    return get().wkv6_logit_backward(r, k, v, omega, u, dy, s0=s0, dsT=dsT)


def wkv6_logit(r, k, v, omega, u, s0=None, g=None, ln_w=None, ln_b=None, eps=1e-5):
    return get().wkv6_logit(r, k, v, omega, u, s0=s0, g=g, ln_w=ln_w, ln_b=ln_b, eps=eps)


def set_threads(n: int = 0) -> int:
    return get().set_threads(n)
