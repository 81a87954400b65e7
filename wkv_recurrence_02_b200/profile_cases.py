"""Run single WKV launches on fixed synthetic shapes, for profilers (ncu) to capture.

    python -m wkv_recurrence_02_b200.profile_cases [--case NAME ...] [--reps N]

Every case first makes one untimed call (so a profiler can skip it with ``-s``), then
``--reps`` calls of the same launch.  Cases:

  wkv4          RWKV-4 scan, B8 T1024 C768 bf16: one layer of the 169M model's shape
  finch         WKV-6 chunked prefill, B8 T1024 H32 N64 bf16 with s0 (256 CTAs, 16 chunks
                each: the Finch-1.6B prefill shape at a quarter of its length)
  long          WKV-6 chunked prefill with sequence split, B1 T4096 H64 (first pass over
                half-segment pieces, then the chunked pass)
  decode        WKV-6 T=1 decode, B256 H64 with the state updated in place (268 MB of state)
  wkv4_decode   RWKV-4 T=1 decode, B2048 C4096 bf16, (a, b, p) state updated in place
  finch_gated   the finch case through rwkv_wkv6_forward_gated_bf16 (head LayerNorm and
                SiLU gate fused into the epilogue)
  finch_backward  the WKV-6 backward pass at the finch shape (B8 T4096 H32 bf16 inputs,
                fp32 gradients, random s0 and dsT): four launches per call
  small_backward  the same at B8 T1024 H32 (for ncu captures)

Inputs come from the seeded generators in ``inputs``; nothing here checks results.
"""
import argparse

import torch

from . import inputs, ops

CASES = ("wkv4", "finch", "long", "decode", "wkv4_decode", "finch_gated", "finch_backward", "small_backward")


def _wkv4(reps):
    x = inputs.wkv4_inputs(8, 1024, 768, "bf16", seed=0, wu_seed=1)
    a = [x[n].cuda() for n in ("w", "u", "k", "v")]
    y = torch.empty_like(a[2])
    for _ in range(1 + reps):
        ops.wkv4_forward(*a, y=y)


def _wkv4_decode(reps):
    x = inputs.wkv4_inputs(2048, 1, 4096, "bf16", seed=5, wu_seed=6)
    a = [x[n].cuda() for n in ("w", "u", "k", "v")]
    st = torch.zeros(2048, 3, 4096, dtype=torch.float32, device="cuda")
    st[:, 1] = 1.0
    y = torch.empty_like(a[2])
    for _ in range(1 + reps):
        ops.wkv4_forward(*a, s0=st, sT=st, y=y, want_state=True)


def _wkv6_gated(B, T, H, reps):
    x = inputs.wkv6_inputs(B, T, H, 64, "bf16", seed=0, s0_std=0.1)
    a = [x[n].cuda() for n in ("r", "k", "v", "w", "u")]
    ng = inputs.norm_gate_inputs(B, T, H, 64, seed=1)
    g, lw, lb = (ng[n].cuda() for n in ("g", "ln_w", "ln_b"))
    s0 = x["s0"].cuda()
    y = torch.empty_like(a[0])
    sT = torch.empty_like(s0)
    for _ in range(1 + reps):
        ops.wkv6_forward_gated(*a, g, lw, lb, eps=1e-5, s0=s0, y=y, sT=sT)


def _wkv6_backward(B, T, H, reps):
    x = inputs.wkv6_inputs(B, T, H, 64, "bf16", seed=0, s0_std=0.1)
    a = [x[n].cuda() for n in ("r", "k", "v", "w", "u")]
    g = torch.Generator(device="cuda")
    g.manual_seed(1)
    dy = torch.randn(B, T, H, 64, device="cuda", generator=g).to(torch.bfloat16)
    dsT = torch.randn(B, H, 64, 64, device="cuda", generator=g) * 0.1
    s0 = x["s0"].cuda()
    ws = torch.empty(ops.wkv6_backward_workspace_bytes(B, T, H), device="cuda", dtype=torch.uint8)
    for _ in range(1 + reps):
        ops.wkv6_backward(*a, dy, s0=s0, dsT=dsT, workspace=ws)


def _wkv6(B, T, H, reps, s0_std=0.1):
    x = inputs.wkv6_inputs(B, T, H, 64, "bf16", seed=0, s0_std=s0_std)
    a = [x[n].cuda() for n in ("r", "k", "v", "w", "u")]
    s0 = x["s0"].cuda()
    y = torch.empty_like(a[0])
    sT = s0 if T == 1 else torch.empty_like(s0)
    for _ in range(1 + reps):
        ops.wkv6_forward(*a, s0=s0, y=y, sT=sT)


def run(case, reps=1):
    if case == "wkv4":
        _wkv4(reps)
    elif case == "finch":
        _wkv6(8, 1024, 32, reps)
    elif case == "long":
        _wkv6(1, 4096, 64, reps)
    elif case == "decode":
        _wkv6(256, 1, 64, reps)
    elif case == "wkv4_decode":
        _wkv4_decode(reps)
    elif case == "finch_gated":
        _wkv6_gated(8, 1024, 32, reps)
    elif case == "finch_backward":
        _wkv6_backward(8, 4096, 32, reps)
    elif case == "small_backward":
        _wkv6_backward(8, 1024, 32, reps)
    else:
        raise ValueError(f"unknown case {case!r}; choose from {CASES}")


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--case", action="append", choices=CASES,
                    help="case to run (repeatable; default: all, in the order listed)")
    ap.add_argument("--reps", type=int, default=1)
    args = ap.parse_args()
    for case in args.case or CASES:
        run(case, args.reps)
    torch.cuda.synchronize()
    status = ops.device_status()
    print("device status", status)
    if status != 0:
        raise SystemExit(1)


if __name__ == "__main__":
    main()
