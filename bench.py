"""Benchmark of the RG-LRU temporal core on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl own|reference] [--only PART]

Own arm. One step = one forward pass of the layer over one batch of the long-sequence
workload B=1, T=32768, D_RNN=4096, bf16 IO with float32 state (the largest single-GPU
RG-LRU forward configuration), inputs resident in HBM and larger than L2, L2 flushed
(256 MB write) before every timed step as well. The step is one rglru_forward call
through the C ABI: Conv1D(4) (which also zeroes the scan's workspace), the gate GEMM that
forms the recurrence coefficients, and the coefficient scan, the last two launched as
programmatic dependents of the kernel before. A second loop launches the same three
kernels one stage call at a time (the scan's call adds its workspace memset) so that each
kernel's duration is measured with CUDA events; a third times the scan that works from the
gate pre-activations (rglru_scan: Conv1D recompute, gates, log-space decay and the chunked
recurrence in one kernel).
Also reported, each as its own record: the Hawk-scale forward B=8, T=2048, D_RNN=2048
(same loops), the float32 forward B=1, T=256, D_RNN=256 as latency, decode steps/s on
B=256, D_RNN=4096, the recurrent block and the Hawk residual layer at B=4, T=4096, D=4096,
D_RNN=5632, the backward at the Hawk-scale workload, the headline metric end to end through
the public API with host buffers (pinned H2D of x, D2H of y and h_T inside the timed
region), the GPU clocks sampled during the timed region, and the CPU oracle on the host
cores.

Under torchrun (N > 1) every rank runs an independent replica on its own GPU (the
batches are independent; nothing is exchanged on the data path), timing is the max
over ranks, and rank 0 prints the JSON line.

Reference arm (--impl reference): the float64 CPU oracle, timed as it stands on the
host cores, each step a bounded sample of the same workload (4096 steps of the sequence,
64 of its 4096 channels, the Conv1D over all channels since the gate GEMM reads them all);
rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "RG-LRU fwd tokens/s and achieved HBM GB/s vs B200 peak; decode steps/s"
HEADLINE = dict(name="fwd_long_bf16", B=1, T=32768, R=4096, io="bf16",
                workload="Long-sequence RG-LRU forward: B=1 T=32768 D_RNN=4096, bf16 IO, fp32 state")
HAWK = dict(name="fwd_hawk_bf16", B=8, T=2048, R=2048, io="bf16",
            workload="RG-LRU forward, Hawk-scale layer: B=8 T=2048 D_RNN=2048, bf16 IO, fp32 state")
SMALL = dict(name="fwd_small_f32", B=1, T=256, R=256, io="f32",
             workload="RG-LRU forward B=1 T=256 D_RNN=256, float32 IO and state")
DECODE = dict(B=256, R=4096)
BLOCK = dict(B=4, T=4096, D=4096, R=5632)
ATTN = dict(B=256, D=4096, W=1024)
FLUSH_BYTES = 256 << 20
CPU_CHANNELS = 64        # oracle sample: channels of the headline workload (independent after u)
CPU_STEPS = 4096         # oracle sample: steps of the sequence

# DRAM bytes (read + write) per launch of the dominant kernel, from the ncu capture
# summarised under profiles/, keyed by workload and by the SHA-256 of the kernel's source
# at capture time. A source change invalidates the figure (reported as null).
_GEMM_TC_SHA = "2aa482e4322acf2fa6b97b30ca06a17fcd0db7c4ece33e2654a84e36b7cf2533"
NCU_TRAFFIC = {
    # ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum (1 pass) on
    # bench.py --only forward: 2.19 GB read + 313.4 MB written per launch of the fused gate
    # GEMM + scan, against 335 MB read and 268 MB written algorithmically (u and W read, y
    # written): operands are read from DRAM again where L2 does not hold them
    ("fwd_long_bf16", "gate_gemm_fused_scan"): {"bytes_per_launch": 2.19e9 + 313.4e6, "src_sha256": _GEMM_TC_SHA},
    # ncu --set full on bench.py --only forward_hawk: 84.4 MB read + 90.9 MB written
    ("fwd_hawk_bf16", "gate_gemm"): {"bytes_per_launch": 84.37e6 + 90.92e6, "src_sha256": _GEMM_TC_SHA},
}


def _sha(path):
    return hashlib.sha256(open(path, "rb").read()).hexdigest()


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained"), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# ----------------------------------------------------------------------------- clocks
_CLOCK_Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
            "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
            "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    def __init__(self, dev_index):
        self.proc = None
        self.dev = dev_index

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={_CLOCK_Q}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", str(self.dev)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(", ") for r in out.strip().splitlines() if r.strip()]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------ own arm
class Ctx:
    """What every measurement needs: the device, its stream, the flush buffer, the peaks and
    the replica plumbing (barrier, max over ranks)."""

    def __init__(self, torch, rglru, inputs, replicas, rk, dev):
        self.torch, self.rglru, self.inputs, self.replicas, self.rk = torch, rglru, inputs, replicas, rk
        self.dev = dev
        self.world = rk.world
        self.stream = torch.cuda.current_stream(dev)
        self.flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.flush_src = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.sink = torch.empty((), dtype=torch.float32, device=dev)
        self.pk = _peaks()

    def flush_l2(self):
        """Evicts the workload from L2 between timed steps: a 256 MB write (twice the L2),
        then a 256 MB read of another buffer, so that the lines the write left dirty are
        written back here and not inside the next timed region."""
        self.flush.zero_()
        self.torch.sum(self.flush_src, dim=0, out=self.sink)

    def barrier(self):
        self.replicas.barrier(self.rk)

    def max_over_ranks(self, v):
        return self.replicas.max_over_ranks(self.rk, v, device=self.dev)

    def events(self, n):
        return [self.torch.cuda.Event(enable_timing=True) for _ in range(n)]


def _roofline(kern, dom, pk, workload):
    src = os.path.join(ROOT, "gated_linear_rnn_conv1d_b200", "csrc",
                       {"gate_gemm": "gemm_tc.cu", "gate_gemm_fused_scan": "gemm_tc.cu", "scan": "scan.cu",
                        "conv1d": "conv.cu"}[dom])
    rec = NCU_TRAFFIC.get((workload, dom))
    traffic = rec["bytes_per_launch"] if rec and rec["src_sha256"] == _sha(src) else None
    if dom in ("gate_gemm", "gate_gemm_fused_scan"):
        roof = {"bound": "tensor", "achieved": kern[dom]["TFLOP/s"], "peak": pk["bf16_tflops"], "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": kern[dom]["GB/s"], "peak": pk["hbm_gbs"], "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = traffic
    roof["kernel"] = dom
    roof["algorithmic_per_launch"] = kern[dom]["flops" if roof["bound"] == "tensor" else "bytes"]
    roof["peak_source"] = ("measured: MEASURED_PEAKS.json burst figure" if pk["source"] == "measured"
                           else "fallback")
    if roof["bound"] == "tensor" and pk.get("bf16_tflops_sustained"):
        # the GEMM runs power-capped (sw_power_cap) inside the step loop; its fraction of the
        # measured sustained figure, for context (frac above stays against the burst peak)
        roof["frac_of_sustained"] = roof["achieved"] / pk["bf16_tflops_sustained"]
    return roof


def bench_forward(c, cfg, steps, warmup, seed=0, clocks=None):
    """rglru_forward on one workload: the step (one call, L2 flushed before each), then each
    kernel through its stage call, then the scan from pre-activations (rglru_scan)."""
    torch, rglru, inputs = c.torch, c.rglru, c.inputs
    B, T, R = cfg["B"], cfg["T"], cfg["R"]
    dt = torch.bfloat16 if cfg["io"] == "bf16" else torch.float32
    es = 2 if cfg["io"] == "bf16" else 4
    w = inputs.make_forward(B, T, R, dt, seed=seed)
    p = rglru.Params.from_host(w.params, c.dev)
    x = w.x.to(c.dev)
    y = torch.empty_like(x)
    h_T = torch.empty(B, R, dtype=torch.float32, device=c.dev)
    u = torch.empty_like(x)
    pitch = rglru.gate_pitch(R)
    zdt = torch.int16 if dt == torch.bfloat16 else torch.float32
    z = torch.empty(B * T, pitch, dtype=zdt, device=c.dev)   # coefficient words (bf16) / pre-activations (f32)
    ws_scan = torch.empty(rglru.scan_workspace_bytes(B, T, R, dt), dtype=torch.uint8, device=c.dev)
    ws_fwd = torch.empty(rglru.forward_workspace_bytes(B, T, R, dt), dtype=torch.uint8, device=c.dev)
    stream, flush = c.stream, c.flush_l2
    bf = dt == torch.bfloat16
    # rglru_forward's own kernels for this shape: Conv1D + the gate GEMM with the scan in its
    # epilogue (2), or Conv1D + coefficient GEMM + scan (3)
    n_kern = rglru.forward_kernels(B, T, R, dt)
    fused = n_kern == 2
    ws_f = torch.empty(rglru.gate_scan_workspace_bytes(B, T, R), dtype=torch.uint8, device=c.dev) \
        if bf and T % 128 == 0 else None

    def forward_step():
        rglru.forward(p, x, workspace=ws_fwd, y=y, h_T=h_T, want_conv_state=False)

    def stages(ev):
        # the separate path's three stage calls
        ev[0].record(stream)
        rglru.conv1d(p, x, u=u)
        ev[1].record(stream)
        if bf:
            rglru.gate_coeffs(p, u.view(B * T, R), g=z)
        else:
            rglru.gate_proj(p, u.view(B * T, R), z=z)
        ev[2].record(stream)
        if bf:
            rglru.scan_coeffs(z, B, T, R, workspace=ws_scan, y=y, h_T=h_T)
        else:
            rglru.scan(p, x, z, workspace=ws_scan, y=y, h_T=h_T)
        ev[3].record(stream)

    for _ in range(warmup):
        flush()
        forward_step()
        flush()
        stages(c.events(4))
    torch.cuda.synchronize()
    if rglru.workspace_status(ws_scan) != 0 or rglru.workspace_status(ws_fwd) != 0 \
            or rglru.workspace_status(None) != 0:
        raise SystemExit("a kernel reported a timeout during warm-up")
    fevs = [c.events(2) for _ in range(steps)]
    if clocks is not None:
        clocks.start()
    c.barrier()
    torch.cuda.synchronize()
    for k in range(steps):
        flush()                 # L2 flush between timed steps (outside the events)
        fevs[k][0].record(stream)
        forward_step()
        fevs[k][1].record(stream)
    torch.cuda.synchronize()
    c.barrier()
    clk = clocks.stop() if clocks is not None else None
    step_ms = c.max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in fevs) / steps)
    status = rglru.workspace_status(ws_fwd)
    ks = max(3, min(steps, 100))
    evs = [c.events(4) for _ in range(ks)]
    for k in range(ks):
        flush()
        stages(evs[k])
    torch.cuda.synchronize()
    conv_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / ks
    gemm_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / ks
    scan_ms = sum(e[2].elapsed_time(e[3]) for e in evs) / ks
    status = status or rglru.workspace_status(ws_scan)
    tokens = B * T
    conv_bytes = tokens * R * es * 2                           # read x, write u
    gemm_flops = 2.0 * tokens * (2 * R) * R
    kern = {
        "conv1d": {"ms": conv_ms, "GB/s": conv_bytes / conv_ms / 1e6, "bytes": conv_bytes},
        "gate_gemm": {"ms": gemm_ms, "TFLOP/s": gemm_flops / gemm_ms / 1e9, "flops": gemm_flops,
                      "kernel": "tcgen05 2-SM, coefficient epilogue" if bf else "FFMA, pre-activations"},
    }
    if bf:
        scan_bytes = tokens * R * (4 + 2)                      # read d (fp16) and b (bf16), write y
        kern["scan"] = {"ms": scan_ms, "GB/s": scan_bytes / scan_ms / 1e6, "bytes": scan_bytes,
                        "kernel": "rglru_scan_coeffs"}
        # the scan from pre-activations: Conv1D recompute, gates, log-space decay, chunked
        # recurrence; reads x and the packed z (bf16), writes y (8 B per token·channel)
        zp = torch.empty(B * T, pitch, dtype=torch.bfloat16, device=c.dev)
        rglru.gate_proj(p, u.view(B * T, R), z=zp)
        for _ in range(2):
            rglru.scan(p, x, zp, workspace=ws_scan, y=y, h_T=h_T)
        pev = [c.events(2) for _ in range(ks)]
        for k in range(ks):
            flush()
            pev[k][0].record(stream)
            rglru.scan(p, x, zp, workspace=ws_scan, y=y, h_T=h_T)
            pev[k][1].record(stream)
        torch.cuda.synchronize()
        pre_ms = sum(e[0].elapsed_time(e[1]) for e in pev) / ks
        pre_bytes = tokens * R * (2 + 4 + 2)
        kern["scan_from_preactivations"] = {"ms": pre_ms, "GB/s": pre_bytes / pre_ms / 1e6, "bytes": pre_bytes,
                                            "kernel": "rglru_scan (Conv1D recompute + gates + decay + scan)",
                                            "note": "timed apart; not part of the step"}
        status = status or rglru.workspace_status(ws_scan)
        del zp
        if ws_f is not None:
            # the gate GEMM with the scan fused into its epilogue (rglru_gate_scan, after the
            # Conv1D stage): the coefficients never reach HBM
            u3 = u.view(B, T, R)
            for _ in range(2):
                rglru.gate_scan(p, u3, workspace=ws_f, y=y, h_T=h_T)
            fev = [c.events(3) for _ in range(ks)]
            for k in range(ks):
                flush()
                fev[k][0].record(stream)
                rglru.conv1d(p, x, u=u)
                fev[k][1].record(stream)
                rglru.gate_scan(p, u3, workspace=ws_f, y=y, h_T=h_T)
                fev[k][2].record(stream)
            torch.cuda.synchronize()
            f_ms = sum(e[1].elapsed_time(e[2]) for e in fev) / ks
            f_step = sum(e[0].elapsed_time(e[2]) for e in fev) / ks
            kern["gate_gemm_fused_scan"] = {"ms": f_ms, "TFLOP/s": gemm_flops / f_ms / 1e9, "flops": gemm_flops,
                                            "step_ms_with_conv": f_step,
                                            "kernel": "rglru_gate_scan (tcgen05 2-SM, scan in the epilogue)",
                                            "note": ("the step's second kernel" if fused else
                                                     "timed apart; not the step's path at this shape") +
                                                    "; its stage call includes a carry memset"}
            status = status or rglru.workspace_status(ws_f)
    else:
        scan_bytes = tokens * R * 4 * 4                        # read x, z_a, z_x, write y (float32)
        kern["scan"] = {"ms": scan_ms, "GB/s": scan_bytes / scan_ms / 1e6, "bytes": scan_bytes,
                        "kernel": "rglru_scan (float32)"}
    for k in kern.values():
        if "GB/s" in k:
            k["frac_hbm"] = k["GB/s"] / c.pk["hbm_gbs"]
        if "TFLOP/s" in k and bf:
            k["frac_tensor"] = k["TFLOP/s"] / c.pk["bf16_tflops"]
    step_kernels = ("conv1d", "gate_gemm_fused_scan") if fused else ("conv1d", "gate_gemm", "scan")
    for k in kern:
        if k not in step_kernels and "note" not in kern[k]:
            kern[k]["note"] = "the separate path's stage; not the step's path at this shape"
    dom = max(step_kernels, key=lambda k: kern[k]["ms"])
    roof = _roofline(kern, dom, c.pk, cfg["name"])
    res = {"workload": cfg["workload"], "B": B, "T": T, "D_RNN": R, "ms_per_step": step_ms,
           "tokens_per_s": c.world * tokens / (step_ms / 1e3), "kernels": kern, "roofline": roof,
           "status": status, "gpu_launches_per_step": n_kern, "step_kernels": list(step_kernels), "clocks": clk,
           "timing": f"{steps} rglru_forward calls, L2 flushed before each; kernels: {ks} stage calls"}
    del x, y, u, z, ws_scan, ws_fwd
    return res, w


def bench_small_latency(c, cfg, reps=200):
    """The float32 workload is tiny (1 MB of input): its forward is launch-latency bound.
    Latency of one rglru_forward call (3 kernels), back to back on warm L2, and of each
    kernel alone."""
    torch, rglru, inputs = c.torch, c.rglru, c.inputs
    B, T, R = cfg["B"], cfg["T"], cfg["R"]
    w = inputs.make_forward(B, T, R, torch.float32, seed=0)
    p = rglru.Params.from_host(w.params, c.dev)
    x = w.x.to(c.dev)
    y = torch.empty_like(x)
    h_T = torch.empty(B, R, device=c.dev)
    ws = torch.empty(rglru.forward_workspace_bytes(B, T, R, torch.float32), dtype=torch.uint8, device=c.dev)
    for _ in range(20):
        rglru.forward(p, x, workspace=ws, y=y, h_T=h_T, want_conv_state=False)
    torch.cuda.synchronize()
    e0, e1 = c.events(2)
    e0.record(c.stream)
    for _ in range(reps):
        rglru.forward(p, x, workspace=ws, y=y, h_T=h_T, want_conv_state=False)
    e1.record(c.stream)
    torch.cuda.synchronize()
    us = c.max_over_ranks(1e3 * e0.elapsed_time(e1) / reps)
    st = rglru.workspace_status(ws)
    return {"workload": cfg["workload"], "us_per_call": us, "tokens_per_s": c.world * B * T / (us / 1e6),
            "status": st, "gpu_launches_per_call": 3,
            "timing": f"{reps} rglru_forward calls back to back (L2-warm: the inputs are 1 MB)",
            "bound": "launch latency (65 K token-channels; 67 MFLOP gate GEMM)"}


def run_own(args):
    import torch

    from gated_linear_rnn_conv1d_b200 import inputs, replicas, rglru

    rk = replicas.from_env()
    world, rank, local = rk.world, rk.rank, rk.local
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    replicas.init(rk, "nccl", device=dev)
    c = Ctx(torch, rglru, inputs, replicas, rk, dev)
    seed = replicas.seed_for(rk)

    def emit(obj):
        replicas.shutdown(rk)
        if rank == 0:
            print(json.dumps(obj))

    only = args.only
    if only == "decode":
        return emit({"only": "decode", "decode": run_decode(c)})
    if only == "block":
        return emit({"only": "block", "block": run_block(c, reps=2)})
    if only == "layer":
        return emit({"only": "layer", "layer": run_layer(c)})
    if only == "backward":
        return emit({"only": "backward", "backward": run_backward(c, reps=3)})
    if only == "attention":
        return emit({"only": "attention", "attention_decode": run_attention(c)})
    if only == "forward_small":
        return emit({"only": "forward_small", "forward_small_f32": bench_small_latency(c, SMALL)})
    if only == "forward_hawk":
        r, _ = bench_forward(c, HAWK, args.steps, args.warmup, seed)
        return emit({"only": "forward_hawk", "forward_hawk_bf16": r})

    clocks = ClockSampler(local)
    head, w = bench_forward(c, HEADLINE, args.steps, args.warmup, seed, clocks=clocks)
    B, T, R = HEADLINE["B"], HEADLINE["T"], HEADLINE["R"]
    value = world * B * T / (head["ms_per_step"] / 1e3)
    if only == "forward":
        return emit({"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                     "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "kernels": head["kernels"],
                     "roofline": head["roofline"], "gpu_launches": head["gpu_launches_per_step"] * args.steps,
                     "clocks": head["clocks"],
                     "only": "forward"})

    # ---- end to end through the public API, host buffers -----------------------------
    # rglru.forward_host: the sequence cut into time chunks pipelined through pinned host
    # copies in both directions and rglru_forward on three streams (the call a user with
    # host data makes), each chunk started from the state the previous one returned
    p = rglru.Params.from_host(w.params, dev)
    x_host = w.x.pin_memory()
    del w
    y_host = torch.empty(B, T, R, dtype=torch.bfloat16).pin_memory()
    h_host = torch.empty(B, R, dtype=torch.float32).pin_memory()
    plan = rglru.HostForwardPlan(B, T, R, torch.bfloat16, groups=E2E_GROUPS, slots=3, device=dev)
    e2e_steps = max(3, min(args.steps, 20))
    for _ in range(2):
        rglru.forward_host(p, x_host, y_host, h_host, plan, stream=c.stream)
    torch.cuda.synchronize()
    e0, e1 = c.events(2)
    c.barrier()
    torch.cuda.synchronize()
    e0.record(c.stream)
    for _ in range(e2e_steps):
        rglru.forward_host(p, x_host, y_host, h_host, plan, stream=c.stream)
    e1.record(c.stream)
    torch.cuda.synchronize()
    c.barrier()
    e2e_ms = c.max_over_ranks(e0.elapsed_time(e1) / e2e_steps)
    e2e = {"value": world * B * T / (e2e_ms / 1e3), "unit": "tokens/s", "ms_per_step": e2e_ms,
           "h2d_bytes_per_step": B * T * R * 2, "d2h_bytes_per_step": B * T * R * 2 + B * R * 4,
           "api": f"rglru.forward_host: {E2E_GROUPS} time chunks; host->device copy, rglru_forward (from the "
                  "previous chunk's state) and device->host copy of neighbouring chunks overlapped on three streams"}
    status = head["status"] or plan.status()
    del plan, x_host, y_host, h_host

    hawk, _ = bench_forward(c, HAWK, args.steps, args.warmup, seed)
    small = bench_small_latency(c, SMALL)
    dec = run_decode(c)
    att = run_attention(c)
    blk = run_block(c)
    lay = run_layer(c)
    bwd = run_backward(c)

    replicas.shutdown(rk)
    if rank != 0:
        return
    cpu = cpu_baseline(inputs) if world == 1 else None
    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) inputs, LeCun-normal gate weights, a^8~U[0.9,0.999])",
        "config": {"workload": HEADLINE["workload"], "B": B, "T": T, "D_RNN": R, "global_batch": B * world,
                   "seq_len": T,
                   "parallelism": f"replicas x{world} (independent batches, no collective on the data path)",
                   "l2": "inputs larger than L2 (x 268 MB) and L2 flushed before every timed step (256 MB write, then 256 MB read of another buffer so no dirty line is left; "
                         "outside the step events)"},
        "roofline": head["roofline"],
        "kernels": head["kernels"],
        "hbm_gb_per_s": {"scan": head["kernels"]["scan"]["GB/s"], "conv1d": head["kernels"]["conv1d"]["GB/s"],
                         "peak": c.pk["hbm_gbs"], "peak_source": c.pk["source"]},
        "forward_hawk_bf16": hawk,
        "forward_small_f32": small,
        "decode": dec,
        "attention_decode": att,
        "block": blk,
        "layer": lay,
        "backward": bwd,
        "e2e": e2e,
        "gpu_launches": head["gpu_launches_per_step"] * args.steps,
        "clocks": head["clocks"],
        "status": "ok" if status == 0 else "timeout reported",
        "cpu_baseline": cpu,
    }
    print(json.dumps(out))


def run_decode(c):
    torch, rglru, inputs, dev, stream, flush, pk = c.torch, c.rglru, c.inputs, c.dev, c.stream, c.flush_l2, c.pk
    barrier, max_over_ranks, world = c.barrier, c.max_over_ranks, c.world
    B, R = DECODE["B"], DECODE["R"]
    w = inputs.make_decode(B, R, torch.bfloat16, seed=0)
    p = rglru.Params.from_host(w.params, dev)
    n_tok = 48
    toks = torch.stack([inputs.decode_token(k, B, R) for k in range(n_tok)]).to(dev)
    ring = torch.zeros(B, 3, R, dtype=torch.bfloat16, device=dev)
    h = torch.zeros(B, R, device=dev)
    y = torch.empty(B, R, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(rglru.step_workspace_bytes(B, R), dtype=torch.uint8, device=dev)
    for k in range(6):
        rglru.step(p, toks[k], ring, h, k, workspace=ws, y_t=y)
    torch.cuda.synchronize()
    # graph of n_tok consecutive steps (weights stay L2-warm across steps, as in serving)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for k in range(n_tok):
            rglru.step(p, toks[k], ring, h, k, workspace=ws, y_t=y)
    g.replay()
    torch.cuda.synchronize()
    reps = 8
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    warm_ms = max_over_ranks(e0.elapsed_time(e1) / (reps * n_tok))
    # one step at a time with L2 flushed before each step (weights come from HBM)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(24)]
    for k, (a, b) in enumerate(evs):
        flush()
        a.record(stream)
        rglru.step(p, toks[k % n_tok], ring, h, k, workspace=ws, y_t=y)
        b.record(stream)
    torch.cuda.synchronize()
    cold_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / len(evs))
    del g
    step_bytes = 2 * R * R * 2 + B * R * (4 + 4) + B * 3 * R * 2 + B * R * 2 * 3   # W, h r/w, ring r, x/ring w/y
    return {"workload": "RG-LRU decode B=256 D_RNN=4096 bf16 x_t/y, fp32 h, bf16 3-slot conv ring",
            "steps_per_s": world / (warm_ms / 1e3), "ms_per_step": warm_ms,
            "steps_per_s_l2_flushed": world / (cold_ms / 1e3), "ms_per_step_l2_flushed": cold_ms,
            "bytes_per_step": step_bytes,
            "GB/s_l2_flushed": step_bytes / cold_ms / 1e6,
            "frac_hbm_l2_flushed": step_bytes / cold_ms / 1e6 / pk["hbm_gbs"],
            # at B=256 the step is at the compute/bandwidth ridge: with the weights L2-warm it is
            # bound by the gate GEMM's 2·B·2R·R FLOP
            "flops_per_step": 2.0 * B * (2 * R) * R,
            "TFLOP/s_warm": 2.0 * B * (2 * R) * R / warm_ms / 1e9,
            "frac_tensor_warm": 2.0 * B * (2 * R) * R / warm_ms / 1e9 / pk["bf16_tflops"],
            "gpu_launches_per_step": 2,
            "timing": "CUDA graph of 48 steps replayed 8x (L2-warm); and 24 single steps with L2 flushed"}


def run_block(c, reps=5):
    """The recurrent block (two input linears, conv, gates, scan with the GeLU branch, output
    linear) as one rglru_block_forward call, L2 flushed before each timed call."""
    torch, rglru, inputs, dev, stream, flush, pk = c.torch, c.rglru, c.inputs, c.dev, c.stream, c.flush_l2, c.pk
    max_over_ranks, world = c.max_over_ranks, c.world
    B, T, D, R = BLOCK["B"], BLOCK["T"], BLOCK["D"], BLOCK["R"]
    w = inputs.make_block(B, T, D, R, torch.bfloat16, seed=0)
    p = rglru.Params.from_host(w.params, dev)
    W_1, W_2, W_o = w.W_1.to(dev), w.W_2.to(dev), w.W_o.to(dev)
    x = w.x.to(dev)
    out = torch.empty_like(x)
    h_T = torch.empty(B, R, dtype=torch.float32, device=dev)
    ws = torch.empty(rglru.block_workspace_bytes(B, T, D, R), dtype=torch.uint8, device=dev)
    for _ in range(2):
        rglru.block_forward(p, W_1, W_2, W_o, x, workspace=ws, out=out, h_T=h_T)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in evs:
        flush()
        a.record(stream)
        rglru.block_forward(p, W_1, W_2, W_o, x, workspace=ws, out=out, h_T=h_T)
        b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / reps)
    n_tok = B * T
    flops = 2.0 * n_tok * (2 * D * R + 2 * R * R + R * D)
    peak = pk["bf16_tflops_sustained"] or pk["bf16_tflops"]
    status = rglru.workspace_status(ws)
    del ws, out, x, W_1, W_2, W_o
    return {"workload": f"recurrent block B={B} T={T} D={D} D_RNN={R} bf16", "ms_per_call": ms,
            "tokens_per_s": world * n_tok / (ms / 1e3), "flops_per_call": flops, "TFLOP/s": flops / ms / 1e9,
            "peak_TFLOP/s": peak, "frac_tensor": flops / ms / 1e9 / peak,
            "peak_source": "measured sustained bf16 (a multi-ms call)", "status": status,
            "gpu_launches_per_call": 6, "timing": f"{reps} calls, L2 flushed before each"}


def run_layer(c, reps=3):
    """One Hawk residual layer at the recurrent block's sizes with the gated MLP (M = 3):
    RMSNorm, the recurrent block, residual add fused with the second RMSNorm, the MLP's
    three linears and GeLU product, residual add — one rglru_layer_forward call, L2
    flushed before each timed call."""
    torch, rglru, inputs, dev, stream, flush, pk = c.torch, c.rglru, c.inputs, c.dev, c.stream, c.flush_l2, c.pk
    max_over_ranks, world = c.max_over_ranks, c.world
    B, T, D, R, M = BLOCK["B"], BLOCK["T"], BLOCK["D"], BLOCK["R"], 3
    H = M * D
    w = inputs.make_layer(B, T, D, R, M, torch.bfloat16, seed=0)
    p = rglru.Params.from_host(w.params, dev)
    lw = rglru.LayerWeights.from_host(w, dev)
    x = w.x.to(dev)
    out = torch.empty_like(x)
    h_T = torch.empty(B, R, dtype=torch.float32, device=dev)
    ws = torch.empty(rglru.layer_workspace_bytes(B, T, D, R, H), dtype=torch.uint8, device=dev)
    for _ in range(2):
        rglru.layer_forward(p, lw, x, workspace=ws, out=out, h_T=h_T)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in evs:
        flush()
        a.record(stream)
        rglru.layer_forward(p, lw, x, workspace=ws, out=out, h_T=h_T)
        b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / reps)
    n_tok = B * T
    flops = 2.0 * n_tok * (2 * D * R + 2 * R * R + R * D) + 2.0 * n_tok * 3 * D * H
    peak = pk["bf16_tflops_sustained"] or pk["bf16_tflops"]
    status = rglru.workspace_status(ws)
    del ws, out, x, lw
    return {"workload": f"Hawk residual layer B={B} T={T} D={D} D_RNN={R} MLP {H} bf16", "ms_per_call": ms,
            "tokens_per_s": world * n_tok / (ms / 1e3), "flops_per_call": flops, "TFLOP/s": flops / ms / 1e9,
            "peak_TFLOP/s": peak, "frac_tensor": flops / ms / 1e9 / peak,
            "peak_source": "measured sustained bf16 (a multi-ms call)", "status": status,
            "gpu_launches_per_call": 13, "timing": f"{reps} calls, L2 flushed before each"}


def run_backward(c, reps=5):
    """The backward of the forward step (rglru_backward at the forward workload: recompute
    of u and z, the chunked reverse recurrence with the gate gradients, the ∂u and weight
    gradient GEMMs reading ∂z and u in place, the Conv1D backward), L2 flushed before each call."""
    torch, rglru, inputs, dev, stream, flush = c.torch, c.rglru, c.inputs, c.dev, c.stream, c.flush_l2
    max_over_ranks, world = c.max_over_ranks, c.world
    B, T, R = HAWK["B"], HAWK["T"], HAWK["R"]
    w = inputs.make_forward(B, T, R, torch.bfloat16, seed=0)
    p = rglru.Params.from_host(w.params, dev)
    x = w.x.to(dev)
    y, _, _ = rglru.forward(p, x)
    g = torch.Generator("cpu").manual_seed(1)
    dy = torch.randn(B, T, R, generator=g).to(torch.bfloat16).to(dev)
    ws = torch.empty(rglru.backward_workspace_bytes(B, T, R), dtype=torch.uint8, device=dev)
    fws = torch.empty(rglru.forward_workspace_bytes(B, T, R, torch.bfloat16), dtype=torch.uint8, device=dev)
    saved = torch.empty(rglru.saved_bytes(B, T, R), dtype=torch.uint8, device=dev)

    def timed(fn):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for a, b in evs:
            flush()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / reps)

    ms = timed(lambda: rglru.backward(p, x, y, dy, workspace=ws))
    # the training pair: the forward also saves the gate pre-activations, the backward
    # reads them instead of recomputing them
    fwd_ms = timed(lambda: rglru.forward(p, x, workspace=fws))
    fwd_train_ms = timed(lambda: rglru.forward_train(p, x, workspace=fws, saved=saved))
    ms_saved = timed(lambda: rglru.backward(p, x, y, dy, workspace=ws, saved=saved))
    n_tok = B * T
    # tensor-core work: z recomputed (2·N·2R·R), ∂u (2·N·2R·R), ∂W_a and ∂W_x (2·2R·R·N)
    flops = 3 * 2.0 * n_tok * (2 * R) * R
    status = rglru.workspace_status(ws) | rglru.workspace_status(fws)
    del ws, fws, saved, x, y, dy
    return {"workload": f"RG-LRU backward B={B} T={T} D_RNN={R} bf16 (dL/dy given)", "ms_per_call": ms,
            "training_pair": {"forward_ms": fwd_ms, "forward_train_ms": fwd_train_ms, "backward_saved_ms": ms_saved,
                              "saved_bytes": rglru.saved_bytes(B, T, R),
                              "note": "rglru_forward_train also writes the gate pre-activations; "
                                      "rglru_backward_saved reads them instead of its z GEMM (9 launches)"},
            "tokens_per_s": world * n_tok / (ms / 1e3), "gemm_flops_per_call": flops,
            # launches: conv, z GEMM, maps, carries, replay, ∂Λ, ∂u GEMM, 2 ∂W GEMMs, conv backward
            "gemm_TFLOP/s_over_the_call": flops / ms / 1e9, "status": status, "gpu_launches_per_call": 10,
            "timing": f"{reps} calls, L2 flushed before each"}


def run_attention(c, reps=24):
    """Griffin's local-attention block, one decode step (rglru_attention_step: the fused
    q/k/v projection, RoPE and ring update, the windowed attention over 1024 ring slots, the
    output projection) for 256 sequences of D = 4096 (32 query heads, one key/value head),
    at positions past the first window so that every slot is live. The rings (134 MB) are
    larger than L2; L2 is flushed before each timed step as well."""
    torch, rglru, inputs, dev, stream, flush = c.torch, c.rglru, c.inputs, c.dev, c.stream, c.flush_l2
    B, D, W = ATTN["B"], ATTN["D"], ATTN["W"]
    H = D // 128
    w = inputs.make_attention(D, seed=0)
    aw = rglru.AttentionWeights.from_host(w, dev)
    g = torch.Generator("cpu").manual_seed(1)
    k_ring = torch.randn(B, W, 128, generator=g).to(torch.bfloat16).to(dev)
    v_ring = torch.randn(B, W, 128, generator=g).to(torch.bfloat16).to(dev)
    toks = torch.stack([inputs.decode_token(k, B, D) for k in range(8)]).to(dev)
    out = torch.empty(B, D, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(rglru.attention_step_workspace_bytes(B, D, W), dtype=torch.uint8, device=dev)
    pos0 = 4 * W
    for k in range(4):
        rglru.attention_step(aw, toks[k % 8], k_ring, v_ring, pos0 + k, workspace=ws, out_t=out)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for k, (a, b) in enumerate(evs):
        flush()
        a.record(stream)
        rglru.attention_step(aw, toks[k % 8], k_ring, v_ring, pos0 + 4 + k, workspace=ws, out_t=out)
        b.record(stream)
    torch.cuda.synchronize()
    ms = c.max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / reps)
    status = rglru.workspace_status(ws)
    ring_bytes = B * W * 128 * 2 * 2                                  # keys and values of the window
    weight_bytes = ((H + 2) * 128 * D + D * H * 128) * 2              # W_qkv and W_o
    act_bytes = B * D * 2 * 2 + B * 256 * 2                           # x_t, out_t; k, v written
    step_bytes = ring_bytes + weight_bytes + act_bytes
    flops = 2.0 * B * D * (H + 2) * 128 + 2.0 * B * H * W * 128 * 2 + 2.0 * B * H * 128 * D
    del k_ring, v_ring, ws
    return {"workload": f"Griffin local MQA decode step B={B} D={D} ({H} heads of 128, 1 KV head) window {W} bf16",
            "ms_per_step": ms, "steps_per_s": c.world / (ms / 1e3), "bytes_per_step": step_bytes,
            "ring_bytes_per_step": ring_bytes, "GB/s": step_bytes / ms / 1e6,
            "frac_hbm": step_bytes / ms / 1e6 / c.pk["hbm_gbs"], "flops_per_step": flops,
            "status": status, "gpu_launches_per_step": 6,  # 2 split-K GEMMs + 2 reduces, prep, chunk
            "timing": f"{reps} single steps at positions past the first window, L2 flushed before each"}


# ------------------------------------------------------------------------------ CPU side
def _host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


_HOST_WORKLOAD = {}


def _host_workload(inputs):
    """The headline workload's inputs on the host (generated once per process)."""
    import torch
    if "w" not in _HOST_WORKLOAD:
        _HOST_WORKLOAD["w"] = inputs.make_forward(HEADLINE["B"], HEADLINE["T"], HEADLINE["R"], torch.bfloat16, seed=0)
    return _HOST_WORKLOAD["w"]


def _oracle_sample(inputs, k=0):
    """The oracle on a bounded sample of the headline workload: CPU_STEPS steps of the
    sequence (the k-th block of them, cycling), CPU_CHANNELS evenly spaced channels (each
    channel of the RG-LRU is independent once the Conv1D output is known; the Conv1D runs
    over all channels because the gate GEMM reads them all). Returns the work done in
    tokens of the full-width workload (steps × channels / D_RNN) and the seconds taken."""
    import numpy as np
    import oracle
    w = _host_workload(inputs)
    pr = w.params
    R = HEADLINE["R"]
    n_blocks = HEADLINE["T"] // CPU_STEPS
    t0 = (k % n_blocks) * CPU_STEPS
    x = w.x[:, t0:t0 + CPU_STEPS]
    ch = np.arange(0, R, R // CPU_CHANNELS)
    t = time.perf_counter()
    oracle.rglru_forward(x, pr.conv_w, pr.conv_b, pr.W_a, pr.b_a, pr.W_x, pr.b_x, pr.Lambda, channels=ch)
    dt = time.perf_counter() - t
    return CPU_STEPS * len(ch) / R, dt


CPU_SAMPLE_SECONDS = 10.0
E2E_GROUPS = 8   # time chunks that forward_host pipelines in the e2e measurement
SAMPLE_TEXT = (f"{CPU_STEPS} steps x {CPU_CHANNELS} of {HEADLINE['R']} channels of the B=1 T={HEADLINE['T']} "
               "sequence per sample (Conv1D over all channels), counted as steps x channels / D_RNN tokens; "
               "float64 numpy, BLAS matmul on the host cores, recurrence vectorised over channels")


def cpu_baseline(inputs):
    from threadpoolctl import threadpool_limits
    _oracle_sample(inputs, 0)                         # untimed: first touch of host memory
    tok, dt, n = 0.0, 0.0, 0
    while dt < CPU_SAMPLE_SECONDS:
        t, d = _oracle_sample(inputs, n)
        tok += t
        dt += d
        n += 1
    # the same oracle with its BLAS held to one thread (the recurrence is single-threaded numpy)
    tok1, dt1, n1 = 0.0, 0.0, 0
    with threadpool_limits(limits=1):
        while dt1 < CPU_SAMPLE_SECONDS / 2:
            t, d = _oracle_sample(inputs, n1)
            tok1 += t
            dt1 += d
            n1 += 1
    return {"value": tok / dt, "unit": "tokens/s", "cores": _host_cores(), "kind": "oracle",
            "sample": f"{n} samples, {dt:.1f} s: " + SAMPLE_TEXT,
            "single_core": {"value": tok1 / dt1, "unit": "tokens/s", "cores": 1,
                            "sample": f"{n1} samples, {dt1:.1f} s, BLAS limited to one thread"}}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    from gated_linear_rnn_conv1d_b200 import inputs
    for i in range(args.warmup):
        _oracle_sample(inputs, i)
    tot_tok, tot_dt = 0.0, 0.0
    for i in range(args.steps):
        tok, dt = _oracle_sample(inputs, args.warmup + i)
        tot_tok += tok
        tot_dt += dt
    value = tot_tok / tot_dt
    cores = _host_cores()
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": HEADLINE["workload"], "B": HEADLINE["B"], "T": HEADLINE["T"], "D_RNN": HEADLINE["R"]},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": "per step: " + SAMPLE_TEXT},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["own", "reference"], default="own")
    ap.add_argument("--only", choices=["all", "forward", "forward_hawk", "forward_small", "decode", "attention", "block",
                                       "backward", "layer"], default="all",
                    help="time that part only (small commands for profiler captures): forward = the headline "
                         "long-sequence forward, forward_hawk = B=8 T=2048 D_RNN=2048, forward_small = the float32 "
                         "B=1 T=256 D_RNN=256 latency")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_own(args)


if __name__ == "__main__":
    main()
