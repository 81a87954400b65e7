"""Seeded synthetic inputs for the WKV recurrences (shared by tests, bench and smoke).

This module draws random numbers and shapes them into the workloads; it holds
none of the recurrences' arithmetic and imports nothing else from the package,
so both the CUDA path and the CPU oracle can be fed from it.

All draws use a CPU ``torch.Generator`` seeded with ``manual_seed``, in fp32,
in the order written below, and are cast to the requested dtype last.  The
decay inputs follow the pages' parametrisation (the caller, not the kernel,
applies it): RWKV-4 w = exp(omega) is a positive rate with per-step decay
e^{-w}; Eagle/Finch w = exp(-exp(omega)) lies in (0, 1) ("RWKV-5/6 (Eagle and
Finch)", section 4.1.2), with a per-token omega_t for Finch (section 4.2.2).
"""
import math
from dataclasses import dataclass

import torch

_DTYPES = {"fp32": torch.float32, "bf16": torch.bfloat16}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def wkv4_wu(C: int, seed: int):
    """Per-channel (w, u) for WKV-4: omega ~ U(-3, 1), w = exp(omega); u ~ N(0, 0.5).

    Draw order: omega [C], then u [C].  Both fp32.
    """
    g = _gen(seed)
    omega = torch.rand(C, generator=g) * 4.0 - 3.0
    u = torch.randn(C, generator=g) * 0.5
    return torch.exp(omega), u


def wkv4_kv(B: int, T: int, C: int, seed: int, dtype: str = "fp32"):
    """k, v ~ N(0, 1) of shape [B, T, C].  Draw order: k, then v; cast last."""
    g = _gen(seed)
    k = torch.randn(B, T, C, generator=g)
    v = torch.randn(B, T, C, generator=g)
    dt = _DTYPES[dtype]
    return k.to(dt), v.to(dt)


def wkv4_inputs(B: int, T: int, C: int, dtype: str = "fp32", seed: int = 0, wu_seed: int = None):
    """One WKV-4 call: k, v from `seed`; w, u from `wu_seed` (defaults to `seed`)."""
    w, u = wkv4_wu(C, seed if wu_seed is None else wu_seed)
    k, v = wkv4_kv(B, T, C, seed, dtype)
    return {"w": w, "u": u, "k": k, "v": v}


def wkv6_inputs(B: int, T: int, H: int, N: int = 64, dtype: str = "fp32", seed: int = 0,
                s0_std: float = None, decay: str = "w"):
    """One WKV-6 call, Finch-style per-token decay.

    Draw order (generator seeded with `seed`):
      omega_h ~ U(-6, -0.5)      [H, N]
      u       ~ N(0, 0.5)        [H, N]
      r, k, v ~ N(0, 1) / sqrt(N) [B, T, H, N] each, in that order
      xi      ~ N(0, 1)          [B, T, H, N];  omega_t = omega_h + 0.3 xi
      s0      ~ N(0, s0_std)     [B, H, N, N]  (only when s0_std is given)
    decay="w": w = exp(-exp(omega_t)) is formed in fp32 and then cast with r, k, v;
    decay="omega": the logit omega_t itself is returned (key "omega", cast like r, k, v)
    instead of w, for the entry points that take the logit.  u and s0 stay fp32.
    """
    if decay not in ("w", "omega"):
        raise ValueError(f"decay must be 'w' or 'omega', not {decay!r}")
    g = _gen(seed)
    omega_h = torch.rand(H, N, generator=g) * 5.5 - 6.0
    u = torch.randn(H, N, generator=g) * 0.5
    sc = 1.0 / math.sqrt(N)
    r = torch.randn(B, T, H, N, generator=g) * sc
    k = torch.randn(B, T, H, N, generator=g) * sc
    v = torch.randn(B, T, H, N, generator=g) * sc
    xi = torch.randn(B, T, H, N, generator=g)
    omega_t = omega_h + 0.3 * xi
    del xi
    dt = _DTYPES[dtype]
    if decay == "w":
        dec = {"w": torch.exp(-torch.exp(omega_t)).to(dt)}
    else:
        dec = {"omega": omega_t.to(dt)}
    del omega_t
    s0 = None
    if s0_std is not None:
        s0 = torch.randn(B, H, N, N, generator=g) * float(s0_std)
    return {"r": r.to(dt), "k": k.to(dt), "v": v.to(dt), **dec, "u": u, "s0": s0}


def norm_gate_inputs(B: int, T: int, H: int, N: int = 64, seed: int = 0):
    """Inputs of the WKV-6 output stage (head LayerNorm, SiLU gate).

    Draw order (generator seeded with `seed`):
      ln_w ~ U(0.5, 1.5)   [H, N] fp32 (per-channel scale)
      ln_b ~ N(0, 0.2)     [H, N] fp32 (per-channel shift)
      g    ~ N(0, 1.5)     [B, T, H, N], cast to bf16 (the gate before its SiLU)
    """
    gen = _gen(seed)
    ln_w = torch.rand(H, N, generator=gen) + 0.5
    ln_b = torch.randn(H, N, generator=gen) * 0.2
    g = (torch.randn(B, T, H, N, generator=gen) * 1.5).to(torch.bfloat16)
    return {"g": g, "ln_w": ln_w, "ln_b": ln_b}


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str          # "wkv4" | "wkv6"
    dtype: str
    B: int
    T: int
    C: int = 0         # WKV-4 channels
    H: int = 0         # WKV-6 heads
    N: int = 64        # WKV-6 head size
    calls: int = 1     # WKV-4: layers (independent w,u); WKV-6: chained calls splitting T
    s0_std: float = None


# The five workloads of the method's evaluation, by what they are.
WORKLOADS = {
    "wkv4_small_fp32": Workload("wkv4_small_fp32", "wkv4", "fp32", B=1, T=64, C=128),
    "wkv6_small_fp32": Workload("wkv6_small_fp32", "wkv6", "fp32", B=1, T=256, H=4),
    "wkv4_169m_bf16": Workload("wkv4_169m_bf16", "wkv4", "bf16", B=8, T=1024, C=768, calls=12),
    "wkv6_finch1b6_bf16": Workload("wkv6_finch1b6_bf16", "wkv6", "bf16", B=8, T=4096, H=32,
                                   s0_std=0.1),
    "wkv6_7b_long_bf16": Workload("wkv6_7b_long_bf16", "wkv6", "bf16", B=1, T=16384, H=64,
                                  calls=4),
    "wkv6_7b_decode": Workload("wkv6_7b_decode", "wkv6", "bf16", B=256, T=1, H=64, s0_std=0.1),
}
