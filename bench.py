"""Throughput of the WKV hot path on B200: WKV tokens/s and fraction of the HBM roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the whole hot path over synthetic inputs resident in HBM:
  * WKV-4, 169M-model shape: B=8, T=1024, C=768, bf16 k/v, 12 layers (each layer its
    own k/v buffers and independently seeded w/u), fp32 accumulation;
  * WKV-6, Finch-1.6B shape: B=8, T=4096, H=32, N=64 bf16, random fp32 initial state;
  * WKV-6, 7B-scale long context: B=1, T=16384 as 4 chained calls of 4096 (sT -> s0), H=64;
  * WKV-6 decode: one T=1 step at B=256, H=64 with a random fp32 state, updated in place.
The metric counts B*T tokens of every call (each WKV-4 layer call counts its own B*T).
Inputs per step (~2.4 GB) exceed the 126 MB L2, so no L2 flush is needed between steps.
The K timed steps are captured as one CUDA graph (22 kernel launches per step, the calls
exactly as a user makes them) and replayed once between CUDA events, so host launch
overhead is not timed; each call's own duration is then measured by replaying a graph of
that call, and the end-to-end figure runs the same step eagerly through the public API.

Under torchrun each rank runs the same step on its own GPU (the path shards over
independent sequences/heads with no exchange step: weak scaling, no collective on the
data path); `value` is the tokens of all ranks over the max-over-ranks device time.

--impl reference times the fp64 CPU oracle (the only other implementation this method
has here) on whole steps of the same workload, on the host's cores.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)

METRIC = "WKV tokens/sec (B·T/s) and % of roofline at 1 B200, WKV-4 and WKV-6 prefill"
UNIT = "tokens/s"
WORKLOAD = ("wkv4 169M shape B8 T1024 C768 x12 layers + wkv6 Finch-1.6B B8 T4096 H32 prefill "
            "+ wkv6 7B long context B1 T16384 H64 (4x4096 chained) + wkv6 7B decode T1 B256 H64")
TOKENS_WKV4 = 12 * 8 * 1024
TOKENS_FINCH = 8 * 4096
TOKENS_LONG = 1 * 16384
TOKENS_DECODE = 256
STEP_TOKENS = TOKENS_WKV4 + TOKENS_FINCH + TOKENS_LONG + TOKENS_DECODE
N_HEAD = 64


def wkv4_bytes(B, T, C):
    return 3 * B * T * C * 2 + 2 * C * 4


def wkv6_bytes(B, T, H, s0=True, sT=True, esz=2):
    n = B * T * H * N_HEAD
    st = B * H * N_HEAD * N_HEAD * 4
    return 5 * n * esz + (st if s0 else 0) + (st if sT else 0) + H * N_HEAD * 4


# algorithmic bytes per launch, per kernel family
BYTES = {
    "wkv4_scan": wkv4_bytes(8, 1024, 768),
    "wkv6_chunked_finch": wkv6_bytes(8, 4096, 32),
    "wkv6_chunked_long_first": wkv6_bytes(1, 4096, 64, s0=False),
    "wkv6_chunked_long": wkv6_bytes(1, 4096, 64),
    "wkv6_decode": wkv6_bytes(256, 1, 64),
}


NOMINAL_HBM_GBS = 8000.0  # the 8 TB/s denominator the workload's roofline is stated against



def load_peaks():
    p = os.path.join(HERE, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling in the background (read-only)."""

    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.rows = []
        self.proc = None
        self.gpu = gpu_index

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "50"], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        threading.Thread(target=self._read, daemon=True).start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [x.strip() for x in line.split(",")]))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = [r for (t, r) in self.rows if t0 - 0.1 <= t <= t1 + 0.1] or [r for _, r in self.rows]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[4:8]) if v == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------------------- our arm

class Workload:
    """Device-resident inputs/outputs of one step, plus pinned host copies for e2e."""

    def __init__(self, torch, inputs, device):
        t = torch
        self.t = t
        dev = device
        kv = inputs.wkv4_kv(8, 1024, 768, 0, "bf16")
        self.w4 = []
        for layer in range(12):
            w, u = inputs.wkv4_wu(768, layer + 1)
            self.w4.append({"w": w.to(dev), "u": u.to(dev), "k": kv[0].to(dev).clone(),
                            "v": kv[1].to(dev).clone(),
                            "y": t.empty(8, 1024, 768, dtype=t.bfloat16, device=dev)})
        self.h_kv = (kv[0].pin_memory(), kv[1].pin_memory())
        x = inputs.wkv6_inputs(8, 4096, 32, 64, "bf16", seed=0, s0_std=0.1)
        self.h_finch = {k: v.pin_memory() for k, v in x.items()}
        self.finch = {k: v.to(dev) for k, v in x.items()}
        self.finch["y"] = t.empty_like(self.finch["r"])
        self.finch["sT"] = t.empty_like(self.finch["s0"])
        x = inputs.wkv6_inputs(1, 16384, 64, 64, "bf16", seed=0)
        self.h_long = {k: (v.pin_memory() if v is not None else None) for k, v in x.items()}
        self.long = {k: (v.to(dev) if v is not None else None) for k, v in x.items()}
        self.long["y"] = t.empty_like(self.long["r"])
        self.long["s"] = [t.empty(1, 64, 64, 64, device=dev) for _ in range(2)]
        x = inputs.wkv6_inputs(256, 1, 64, 64, "bf16", seed=7, s0_std=0.1)
        self.h_dec = {k: v.pin_memory() for k, v in x.items()}
        self.dec = {k: v.to(dev) for k, v in x.items()}
        self.dec["y"] = t.empty_like(self.dec["r"])

    def step(self, ops, rec=None):
        """One pass of the hot path; rec(name, fn) wraps each launch for timing."""
        run = rec or (lambda name, fn: fn())
        for L in self.w4:
            run("wkv4_scan", lambda L=L: ops.wkv4_forward(L["w"], L["u"], L["k"], L["v"], y=L["y"]))
        f = self.finch
        run("wkv6_chunked_finch", lambda: ops.wkv6_forward(
            f["r"], f["k"], f["v"], f["w"], f["u"], s0=f["s0"], y=f["y"], sT=f["sT"]))
        g = self.long
        for c in range(4):
            sl = slice(c * 4096, (c + 1) * 4096)
            s_in = None if c == 0 else g["s"][(c - 1) % 2]
            s_out = g["s"][c % 2]
            name = "wkv6_chunked_long_first" if c == 0 else "wkv6_chunked_long"
            run(name, lambda sl=sl, s_in=s_in, s_out=s_out: ops.wkv6_forward(
                g["r"][:, sl], g["k"][:, sl], g["v"][:, sl], g["w"][:, sl], g["u"], s0=s_in,
                y=g["y"][:, sl], sT=s_out))
        d = self.dec
        run("wkv6_decode", lambda: ops.wkv6_forward(d["r"], d["k"], d["v"], d["w"], d["u"],
                                                    s0=d["s0"], y=d["y"], sT=d["s0"]))

    # 12 WKV-4 layers, the Finch prefill, 4 long-context calls of two launches each (the
    # first pass and the chunked pass of the sequence split at 64 heads), the decode step; the
    # ncu launch list of this step counts the same
    launches_per_step = 12 + 1 + 4 * 2 + 1


def step_config(world):
    """The `config` object of the JSON line (the same for both arms)."""
    return {"workload": WORKLOAD, "tokens_per_step_per_gpu": STEP_TOKENS,
            "l2": "inputs larger than L2 (~2.4 GB per step per GPU); no flush",
            "parallelism": f"replicas x{world} (independent sequences, no collective)",
            "launch": "the K steps captured as one CUDA graph, replayed once"}


def max_over_ranks(values, dist, device=None):
    """Each value's maximum over all ranks (the job's time is its slowest rank's); the
    identity with one process.  Works with any process-group backend: CPU tensors for gloo,
    device tensors for nccl."""
    if dist is None:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_tokens_per_s(world, tokens_per_step_per_rank, steps, ms_max):
    """Whole-job throughput: every rank runs the same fixed work per step (weak scaling),
    so the job processes world x tokens per step in the slowest rank's time."""
    return world * tokens_per_step_per_rank * steps / (ms_max * 1e-3)


def run_ours(args, rank, world, dist):
    import torch
    from wkv_recurrence_02_b200 import inputs, ops

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ops.load()
    wl = Workload(torch, inputs, dev)
    stream = torch.cuda.Stream(dev)  # graphs are captured on a stream of their own
    torch.cuda.set_stream(stream)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    # warm-up (eager: sets up the library's per-device state, pools and kernel attributes)
    for _ in range(args.warmup):
        wl.step(ops)
    barrier()

    # timed: the K steps captured as one CUDA graph (22 launches per step, no host work
    # between them), replayed once between a barrier and events on the launching stream
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for _ in range(args.steps):
            wl.step(ops)
    graph.replay()  # untimed: the first replay uploads the graph
    barrier()

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    barrier()
    t_wall0 = time.time()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    graph.replay()
    e1.record(stream)
    barrier()
    t_wall1 = time.time()
    sampler.stop()
    ms = e0.elapsed_time(e1)
    del graph

    # the spread of single steps: one step captured as a graph, each of 100 replays between
    # its own events; the median is reported beside the K-step figure
    g1 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g1, stream=stream):
        wl.step(ops)
    g1.replay()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(100)]
    for a, b in ev:
        a.record(stream)
        g1.replay()
        b.record(stream)
    torch.cuda.synchronize(dev)
    single = sorted(a.elapsed_time(b) for a, b in ev)
    step_stats = {"median_ms": round(statistics.median(single), 4), "min_ms": round(single[0], 4),
                  "p90_ms": round(single[89], 4), "reps": len(single)}
    del g1

    # each call of the step on its own, for the per-kernel roofline: a CUDA graph of the call
    # replayed back to back between events (the same launches, inputs and outputs as the step)
    per = measure_calls(torch, ops, wl, stream, reps=20)

    # end to end through the public API with host buffers: H2D of every input, D2H of results
    e2e_ms, h2d, d2h = run_e2e(torch, ops, wl, stream, dev, max(3, min(args.steps, 10)), barrier)
    next_rows = measure_next_rows(torch, inputs, ops, dev, stream, wl)

    ms_max, e2e_max = max_over_ranks([ms, e2e_ms], dist, device=dev)
    status = ops.device_status()
    if rank != 0:
        return None

    hbm, peak_kind = load_peaks()
    fam = {}
    for name, ts in per.items():
        kern = "wkv6_chunked" if name.startswith("wkv6_chunked") else name
        f = fam.setdefault(kern, {"ms": 0.0, "bytes": 0.0, "launches": 0})
        f["ms"] += sum(ts)
        f["bytes"] += BYTES[name] * len(ts)
        f["launches"] += len(ts)
    total_kernel_ms = sum(f["ms"] for f in fam.values())
    dom = max(fam, key=lambda k: fam[k]["ms"])
    parts = {}
    for name, ts in sorted(per.items()):
        avg = sum(ts) / len(ts)
        gbs = BYTES[name] / (avg * 1e-3) / 1e9
        parts[name] = {"avg_us": round(avg * 1e3, 2), "launches": len(ts),
                       "GBps": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4),
                       "frac_8TBps": round(gbs / NOMINAL_HBM_GBS, 4)}
    for k, f in fam.items():
        parts.setdefault("share", {})[k] = round(f["ms"] / total_kernel_ms, 4)
    roofline = dominant_roofline(dom, fam[dom], per, hbm, peak_kind)
    cpu = cpu_baseline() if (world == 1 and not args.skip_cpu) else None
    line = {
        "metric": METRIC, "value": job_tokens_per_s(world, STEP_TOKENS, args.steps, ms_max),
        "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded torch CPU generator)",
        "config": step_config(world),
        "single_step_replays": step_stats,
        "roofline": roofline,
        "parts": parts,
        "cpu_baseline": cpu,
        "e2e": {"value": job_tokens_per_s(world, STEP_TOKENS, 1, e2e_max), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": Workload.launches_per_step * args.steps,
        "next_rows": next_rows,
        "clocks": sampler.summary(t_wall0, t_wall1),
        "device_status": status,
    }
    return line


def dominant_roofline(kern, fam, per, hbm, peak_kind):
    """Roofline of the dominant kernel over ALL its launches in the step: algorithmic bytes
    of every timed call of the kernel over their summed CUDA-event durations (the average
    launch).  Each call of the kernel is also listed on its own.  `traffic` is the DRAM
    read + write of the average call, from committed ncu captures (see load_traffic)."""
    names = sorted(n for n in per if (n.startswith(kern) if kern == "wkv6_chunked" else n == kern))
    achieved = fam["bytes"] / (fam["ms"] * 1e-3) / 1e9
    calls = {}
    for n in names:
        avg = sum(per[n]) / len(per[n])
        gbs = BYTES[n] / (avg * 1e-3) / 1e9
        calls[n] = {"algorithmic_bytes": BYTES[n], "avg_us": round(avg * 1e3, 2), "calls": len(per[n]),
                    "achieved": round(gbs, 1), "frac": round(gbs / hbm, 4),
                    "frac_8TBps": round(gbs / NOMINAL_HBM_GBS, 4)}
    traffic, note = load_traffic(names, per)
    return {"bound": "hbm", "kernel": kern, "scope": "every launch of the kernel in the timed steps",
            "algorithmic_bytes_per_launch": round(fam["bytes"] / fam["launches"]),
            "avg_us_per_launch": round(fam["ms"] / fam["launches"] * 1e3, 2),
            "achieved": round(achieved, 1), "peak": hbm, "peak_kind": peak_kind, "unit": "GB/s",
            "frac": round(achieved / hbm, 4), "frac_8TBps": round(achieved / NOMINAL_HBM_GBS, 4),
            "traffic": traffic, "traffic_note": note, "calls": calls}


def measure_calls(torch, ops, wl, stream, reps):
    """Per-call durations (ms) of the step's launches, keyed like Workload.step's names: each
    call captured as a CUDA graph and replayed `reps` times between CUDA events."""
    calls = []
    wl.step(ops, lambda name, fn: calls.append((name, fn)))
    torch.cuda.synchronize()
    per = {}
    for name, fn in calls:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        g.replay()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        per.setdefault(name, []).append(a.elapsed_time(b) / reps)
        del g
    return per


def _time_us(torch, stream, dev, fn, reps):
    """Average duration (us) of fn's launches: fn captured as a CUDA graph (after three eager
    calls) and the graph replayed `reps` times between CUDA events."""
    for _ in range(3):
        fn()
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    g.replay()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        g.replay()
    b.record(stream)
    torch.cuda.synchronize(dev)
    del g
    return a.elapsed_time(b) * 1e3 / reps


def measure_next_rows(torch, inputs, ops, dev, stream, wl, reps=50):
    """Rows beyond the step, timed on their own (not part of the step's metric):
      * the RWKV-4 decode step (T = 1) at the width of a 7B model, state updated in place;
      * the Finch prefill with the time-mixing output stage (head LayerNorm, SiLU gate)
        fused into the chunked kernel's epilogue, against the same call without it;
      * the Finch prefill fed the decay logit omega_t (w_t = exp(-exp(omega_t)) formed in
        the kernel), plain and with the fused output stage;
      * the WKV-6 backward pass at the Finch shape (the chunked tensor-core path, with the
        exact fp32 walks timed beside it)."""
    hbm, _ = load_peaks()
    rows = {}
    f = wl.finch
    ng = inputs.norm_gate_inputs(8, 4096, 32, 64, seed=3)
    g, lw, lb = (ng[n].to(dev) for n in ("g", "ln_w", "ln_b"))
    plain = _time_us(torch, stream, dev, lambda: ops.wkv6_forward(
        f["r"], f["k"], f["v"], f["w"], f["u"], s0=f["s0"], y=f["y"], sT=f["sT"]), 20)
    gated = _time_us(torch, stream, dev, lambda: ops.wkv6_forward_gated(
        f["r"], f["k"], f["v"], f["w"], f["u"], g, lw, lb, eps=1e-5, s0=f["s0"], y=f["y"], sT=f["sT"]), 20)
    nbytes = BYTES["wkv6_chunked_finch"] + g.numel() * 2 + 2 * 32 * 64 * 4
    separate = 3 * f["y"].numel() * 2  # an unfused stage reads y and g and writes y again
    rows["wkv6_finch_gated_B8_T4096_H32"] = {
        "avg_us": round(gated, 2), "ungated_avg_us": round(plain, 2), "algorithmic_bytes": nbytes,
        "GBps": round(nbytes / (gated * 1e-6) / 1e9, 1),
        "frac_hbm": round(nbytes / (gated * 1e-6) / 1e9 / hbm, 4),
        "separate_stage_floor_us": round(separate / (hbm * 1e9) * 1e6, 2)}
    # decay given by its logit: omega_t = omega_h + 0.3 xi, the recipe the step's w comes from
    gen = torch.Generator(device=dev)
    gen.manual_seed(7)
    om = ((torch.rand(32, 64, device=dev, generator=gen) * 5.5 - 6.0)
          + 0.3 * torch.randn(8, 4096, 32, 64, device=dev, generator=gen)).to(torch.bfloat16)
    omega = _time_us(torch, stream, dev, lambda: ops.wkv6_forward_omega(
        f["r"], f["k"], f["v"], om, f["u"], s0=f["s0"], y=f["y"], sT=f["sT"]), 20)
    omega_gated = _time_us(torch, stream, dev, lambda: ops.wkv6_forward_omega(
        f["r"], f["k"], f["v"], om, f["u"], s0=f["s0"], g=g, ln_w=lw, ln_b=lb, y=f["y"], sT=f["sT"]), 20)
    nb = BYTES["wkv6_chunked_finch"]
    rows["wkv6_finch_omega_B8_T4096_H32"] = {
        "avg_us": round(omega, 2), "w_input_avg_us": round(plain, 2), "gated_avg_us": round(omega_gated, 2),
        "algorithmic_bytes": nb, "GBps": round(nb / (omega * 1e-6) / 1e9, 1),
        "frac_hbm": round(nb / (omega * 1e-6) / 1e9 / hbm, 4),
        "separate_map_floor_us": round(2 * om.numel() * 2 / (hbm * 1e9) * 1e6, 2)}
    del om
    # WKV-6 backward at the Finch shape (fp32 gradients): the chunked tensor-core path (the
    # default for bf16 inputs), against the HBM roofline of its algorithmic bytes; the exact
    # fp32 walks timed beside it
    gen.manual_seed(8)
    dy = (torch.randn(8, 4096, 32, 64, device=dev, generator=gen)).to(torch.bfloat16)
    dsT = torch.randn(8, 32, 64, 64, device=dev, generator=gen) * 0.1
    ws = torch.empty(ops.wkv6_backward_workspace_bytes(8, 4096, 32), device=dev, dtype=torch.uint8)

    def bwd(algo):
        return lambda: ops.wkv6_backward(f["r"], f["k"], f["v"], f["w"], f["u"], dy, s0=f["s0"], dsT=dsT,
                                         workspace=ws, algo=algo)
    bwd_ms = _time_us(torch, stream, dev, bwd("chunked"), 10) / 1e3
    walks_ms = _time_us(torch, stream, dev, bwd("serial"), 2) / 1e3
    n_el, n_st = dy.numel(), dsT.numel()
    # r, k, v, w, dy in bf16; dr, dk, dv, dw in fp32; s0, dsT, ds0; u and du
    bwd_bytes = 5 * n_el * 2 + 4 * n_el * 4 + 3 * n_st * 4 + 2 * 32 * 64 * 4
    # tensor work: 24 products of 64 x 64 x 64 per chunk (A, dA, dR, dK, dV: 5 pairs of 4, dR/dK
    # second halves 2 x 4) and 4 per chunk in each state pass
    n_chunks = 8 * 32 * (4096 // 64)
    bwd_flops = (24 + 8) * 2 * 64 * 16 * 64 * n_chunks
    gbs = bwd_bytes / (bwd_ms * 1e-3) / 1e9
    rows["wkv6_finch_backward_B8_T4096_H32"] = {
        "avg_ms": round(bwd_ms, 3), "path": "chunked tensor-core (bf16 operands, fp32 accumulation)",
        "algorithmic_bytes": bwd_bytes, "GBps": round(gbs, 1), "bound": "hbm", "peak_gbs": hbm,
        "frac_hbm": round(gbs / hbm, 4), "frac_8TBps": round(gbs / NOMINAL_HBM_GBS, 4),
        "tensor_tflops": round(bwd_flops / (bwd_ms * 1e-3) / 1e12, 2),
        "exact_walks_avg_ms": round(walks_ms, 3),
        "workspace_bytes": ws.numel(), "launches_per_call": 7}
    del dy, dsT, ws
    B, C = 2048, 4096
    x = inputs.wkv4_inputs(B, 1, C, "bf16", seed=5, wu_seed=6)
    w, u, k, v = (x[n].to(dev) for n in ("w", "u", "k", "v"))
    st = torch.zeros(B, 3, C, dtype=torch.float32, device=dev)
    st[:, 0] = torch.randn(B, C, device=dev)
    st[:, 1] = 1.0 + torch.rand(B, C, device=dev)
    y = torch.empty_like(k)
    us = _time_us(torch, stream, dev, lambda: ops.wkv4_forward(w, u, k, v, s0=st, sT=st, y=y, want_state=True),
                  reps)
    nbytes = B * C * (2 * 2 + 2 + 2 * 3 * 4) + 2 * C * 4  # k, v, y bf16; state in and out; w, u
    gbs = nbytes / (us * 1e-6) / 1e9
    rows["wkv4_decode_B2048_C4096"] = {"avg_us": round(us, 2), "algorithmic_bytes": nbytes,
                                       "GBps": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4),
                                       "state_bytes": 2 * B * 3 * C * 4, "launches": reps}
    return rows


def run_e2e(torch, ops, wl, stream, dev, steps, barrier):
    """Same step through the public API with inputs/outputs in pinned host memory.  Each call's
    inputs go up on an upload stream and its outputs come back on a download stream, so the
    copies of one call overlap the compute of others and the two directions overlap each
    other; events order every reuse of a buffer (a call's inputs are not overwritten before
    the previous step's compute and download of that call are done, its outputs not before
    their previous download).  The timed region holds every copy of every timed step."""
    h_y4 = [torch.empty(8, 1024, 768, dtype=torch.bfloat16).pin_memory() for _ in range(12)]
    h_yf = torch.empty_like(wl.h_finch["r"]).pin_memory()
    h_sf = torch.empty_like(wl.h_finch["s0"]).pin_memory()
    h_yl = torch.empty_like(wl.h_long["r"]).pin_memory()
    h_sl = torch.empty(1, 64, 64, 64).pin_memory()
    h_yd = torch.empty_like(wl.h_dec["r"]).pin_memory()
    h_sd = torch.empty_like(wl.h_dec["s0"]).pin_memory()
    up_s = torch.cuda.Stream(device=dev)
    down_s = torch.cuda.Stream(device=dev)

    calls = []  # (inputs [(device, host)], compute, outputs [(host, device)])
    for i, L in enumerate(wl.w4):
        calls.append(([(L["k"], wl.h_kv[0]), (L["v"], wl.h_kv[1])],
                      lambda L=L: ops.wkv4_forward(L["w"], L["u"], L["k"], L["v"], y=L["y"]),
                      [(h_y4[i], L["y"])]))
    f, hf = wl.finch, wl.h_finch
    calls.append(([(f[n], hf[n]) for n in ("r", "k", "v", "w", "s0")],
                  lambda: ops.wkv6_forward(f["r"], f["k"], f["v"], f["w"], f["u"], s0=f["s0"], y=f["y"],
                                           sT=f["sT"]),
                  [(h_yf, f["y"]), (h_sf, f["sT"])]))
    g, hg = wl.long, wl.h_long

    def long_calls():
        for c in range(4):
            sl = slice(c * 4096, (c + 1) * 4096)
            ops.wkv6_forward(g["r"][:, sl], g["k"][:, sl], g["v"][:, sl], g["w"][:, sl], g["u"],
                             s0=None if c == 0 else g["s"][(c - 1) % 2], y=g["y"][:, sl], sT=g["s"][c % 2])
    calls.append(([(g[n], hg[n]) for n in ("r", "k", "v", "w")], long_calls,
                  [(h_yl, g["y"]), (h_sl, g["s"][1])]))
    d, hd = wl.dec, wl.h_dec
    calls.append(([(d[n], hd[n]) for n in ("r", "k", "v", "w", "s0")],
                  lambda: ops.wkv6_forward(d["r"], d["k"], d["v"], d["w"], d["u"], s0=d["s0"], y=d["y"],
                                           sT=d["s0"]),
                  [(h_yd, d["y"]), (h_sd, d["s0"])]))
    h2d = sum(h.numel() * h.element_size() for ins, _, _ in calls for _, h in ins)
    d2h = sum(dv.numel() * dv.element_size() for _, _, outs in calls for _, dv in outs)
    done = [None] * len(calls)  # download-done event of each call in the previous step

    def one():
        for i, (ins, fn, outs) in enumerate(calls):
            if done[i] is not None:
                up_s.wait_event(done[i])
            with torch.cuda.stream(up_s):
                for dst, src in ins:
                    dst.copy_(src, non_blocking=True)
            ev_up = torch.cuda.Event()
            ev_up.record(up_s)
            stream.wait_event(ev_up)
            with torch.cuda.stream(stream):
                fn()
            ev_c = torch.cuda.Event()
            ev_c.record(stream)
            down_s.wait_event(ev_c)
            with torch.cuda.stream(down_s):
                for dst, src in outs:
                    dst.copy_(src, non_blocking=True)
            done[i] = torch.cuda.Event()
            done[i].record(down_s)

    one()
    torch.cuda.synchronize(dev)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    up_s.wait_event(e0)
    down_s.wait_event(e0)
    for _ in range(steps):
        one()
    stream.wait_stream(up_s)
    stream.wait_stream(down_s)
    e1.record(stream)
    barrier()
    return e0.elapsed_time(e1) / steps, h2d, d2h


def load_traffic(names, per):
    """DRAM bytes (read + write) of the average launch of the calls `names`, weighted by how
    often each ran, from the committed ncu figures in profiles/traffic.json; None if any call
    has no figure.  Returns (bytes, the file's note on how the figures were taken)."""
    p = os.path.join(HERE, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None, None
    with open(p) as f:
        d = json.load(f)
    if any(d.get(n) is None for n in names):
        return None, d.get("_note")
    n_calls = sum(len(per[n]) for n in names)
    return round(sum(d[n] * len(per[n]) for n in names) / n_calls), d.get("_note")


# --------------------------------------------------------------------------- CPU oracle

def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


class OracleStep:
    """The fp64 CPU oracle on the inputs of one whole step (drawn once, widened to float64
    exactly; the draws are not timed).  full() runs the step as the GPU arm does: 12 WKV-4
    layers, the Finch prefill, the four chained long-context calls and the decode step."""

    def __init__(self):
        from wkv_recurrence_02_b200 import inputs
        f64 = lambda t: t.float().double().numpy()  # noqa: E731
        kv = inputs.wkv4_kv(8, 1024, 768, 0, "bf16")
        self.kv = (f64(kv[0]), f64(kv[1]))
        self.wu = [tuple(f64(t) for t in inputs.wkv4_wu(768, layer + 1)) for layer in range(12)]
        x = inputs.wkv6_inputs(8, 4096, 32, 64, "bf16", seed=0, s0_std=0.1)
        self.finch = [f64(x[n]) for n in ("r", "k", "v", "w", "u", "s0")]
        x = inputs.wkv6_inputs(1, 16384, 64, 64, "bf16", seed=0)
        self.long = [f64(x[n]) for n in ("r", "k", "v", "w", "u")]
        x = inputs.wkv6_inputs(256, 1, 64, 64, "bf16", seed=7, s0_std=0.1)
        self.dec = [f64(x[n]) for n in ("r", "k", "v", "w", "u", "s0")]
        del x

    def _long(self, T):
        r, k, v, w, u = self.long
        s = None
        for c in range(0, T, 4096):
            sl = slice(c, min(c + 4096, T))  # B = 1: a slice of T is contiguous
            _, s = oracle_mod().wkv6(r[:, sl], k[:, sl], v[:, sl], w[:, sl], u, s0=s)

    def full(self):
        """One whole step; returns its wall time in seconds."""
        o = oracle_mod()
        t0 = time.perf_counter()
        for w, u in self.wu:
            o.wkv4(w, u, *self.kv)
        r, k, v, w, u, s0 = self.finch
        o.wkv6(r, k, v, w, u, s0=s0)
        self._long(16384)
        r, k, v, w, u, s0 = self.dec
        o.wkv6(r, k, v, w, u, s0=s0)
        return time.perf_counter() - t0

    def sample(self):
        """A bounded part of each piece of the step: one WKV-4 layer, Finch batch row 0 (of 8),
        the first 512 tokens of the long context (of 16384) and the whole decode step.
        Returns (the step's time extrapolated from the pieces by tokens, description)."""
        o = oracle_mod()
        t0 = time.perf_counter()
        o.wkv4(*self.wu[0], *self.kv)
        t1 = time.perf_counter()
        r, k, v, w, u, s0 = self.finch
        o.wkv6(r[:1], k[:1], v[:1], w[:1], u, s0=s0[:1])
        t2 = time.perf_counter()
        self._long(512)
        t3 = time.perf_counter()
        r, k, v, w, u, s0 = self.dec
        o.wkv6(r, k, v, w, u, s0=s0)
        t4 = time.perf_counter()
        step = 12 * (t1 - t0) + 8 * (t2 - t1) + 32 * (t3 - t2) + (t4 - t3)
        desc = ("wkv4 one layer (x12), wkv6 Finch batch row 0 (x8), wkv6 7B long context first "
                "512 tokens (x32), the whole decode step; extrapolated to one step by tokens")
        return step, desc


def oracle_mod():
    import oracle
    return oracle


def cpu_figures(ostep, full_steps):
    """All-thread figure: `full_steps` whole steps of the oracle on every host thread (after
    one untimed step); single-thread figure: the bounded sample on one thread."""
    o = oracle_mod()
    threads = len(os.sched_getaffinity(0))
    o.set_threads(threads)
    times = [ostep.full() for _ in range(full_steps)]
    o.set_threads(1)
    one, desc1 = ostep.sample()
    o.set_threads(threads)
    return times, threads, {"value": STEP_TOKENS / one, "unit": UNIT, "cores": 1, "sample": desc1}


def cpu_baseline(full_steps=2):
    """The oracle timed on the host's cores: measured whole steps on every thread (the
    reported value), and the single-thread figure on a bounded sample."""
    ostep = OracleStep()
    o = oracle_mod()
    o.set_threads(len(os.sched_getaffinity(0)))
    ostep.full()  # untimed: pages in the outputs
    times, threads, single = cpu_figures(ostep, full_steps)
    step_s = statistics.median(times)
    return {"value": STEP_TOKENS / step_s, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"the whole step, measured ({full_steps} steps, median {step_s:.3f} s)",
            "cpu_model": cpu_model(), "single_thread": single}


def run_reference(args, rank, world):
    """The oracle as the reference arm: W untimed whole steps, then K whole steps timed with
    the host clock (every host thread), then the single-thread figure on the bounded sample."""
    if rank != 0:
        return None
    ostep = OracleStep()
    o = oracle_mod()
    threads = len(os.sched_getaffinity(0))
    o.set_threads(threads)
    for _ in range(args.warmup):
        ostep.full()
    t0 = time.perf_counter()
    times = [ostep.full() for _ in range(args.steps)]
    wall = time.perf_counter() - t0
    o.set_threads(1)
    one, desc1 = ostep.sample()
    o.set_threads(threads)
    ms = wall * 1e3 / args.steps
    value = STEP_TOKENS * args.steps / wall
    return {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded torch CPU generator)",
        "impl": "reference",
        "config": step_config(world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"the whole step, {args.steps} steps measured "
                                   f"(median {statistics.median(times) * 1e3:.1f} ms)",
                         "cpu_model": cpu_model(),
                         "single_thread": {"value": STEP_TOKENS / one, "unit": UNIT, "cores": 1,
                                           "sample": desc1}},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--skip-cpu", action="store_true", help="omit the CPU oracle baseline")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    try:
        line = run_ours(args, rank, world, dist)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
