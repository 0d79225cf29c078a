"""Benchmark of the RG-LRU temporal core on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl own|reference]

Own arm. One step = one forward pass of the layer over one batch of the Hawk-scale
workload B=8, T=2048, D_RNN=2048, bf16 IO with float32 state, inputs resident in HBM, L2
flushed (256 MB write) before every timed step. The step is one rglru_forward call
through the C ABI: Conv1D(4) (which also zeroes the scan's workspace), the gate GEMM that
forms the recurrence coefficients, and the coefficient scan, the last two launched as
programmatic dependents of the kernel before. A second loop launches the same three
kernels one stage call at a time (the scan's call adds its workspace memset) so that each
kernel's duration is measured with CUDA events. The alternative second stage (gate GEMM
with the scan in its epilogue, rglru_gate_scan) is timed in a third loop and is not part
of the step.
Reported: tokens/s (all ranks), per-kernel achieved bandwidth / throughput and their
fractions of the measured B200 peaks, the roofline of the dominant kernel, the same
metric end to end through the public API with host buffers (pinned H2D of x, D2H of y
and h_T inside the timed region), decode steps/s on B=256, D_RNN=4096, the GPU clocks
sampled during the timed region, and the CPU oracle on the host cores.

Under torchrun (N > 1) every rank runs an independent replica on its own GPU (the
batches are independent; nothing is exchanged on the data path), timing is the max
over ranks, and rank 0 prints the JSON line.

Reference arm (--impl reference): the float64 CPU oracle, timed as it stands on the
host cores, each step a bounded sample of the same workload (one batch row, 512 steps,
all 2048 channels); rank 0 only.
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
WORKLOAD = dict(B=8, T=2048, R=2048)
DECODE = dict(B=256, R=4096)
BLOCK = dict(B=4, T=4096, D=4096, R=5632)
FLUSH_BYTES = 256 << 20

# DRAM bytes (read + write) per launch of the dominant kernel, from the ncu capture
# summarised under profiles/, keyed by the SHA-256 of the kernel's source at capture
# time. A source change invalidates the figure (reported as null).
NCU_TRAFFIC = {
    # dram__bytes_read.sum + dram__bytes_write.sum of one ncu capture of each kernel at this
    # workload (profiles/), valid while the kernel's source file is unchanged
    "gate_gemm": {"src_sha256": "9d882880ce820ce56ec82f063441547a439137e8927679d06e43181c666aec01",
                  "bytes_per_launch": 84198144 + 90386944},
    "scan": {"src_sha256": "38a92a145b986134deb9fdbc8589dc579e93ba17b42ebc9b8a8d13e4f1288d8d",
             "bytes_per_launch": 135208704 + 31897344},
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

    def barrier():
        replicas.barrier(rk)

    def max_over_ranks(v):
        return replicas.max_over_ranks(rk, v, device=dev)

    B, T, R = WORKLOAD["B"], WORKLOAD["T"], WORKLOAD["R"]
    w = inputs.make_forward(B, T, R, torch.bfloat16, seed=replicas.seed_for(rk))
    p = rglru.Params.from_host(w.params, dev)
    x = w.x.to(dev)
    y = torch.empty_like(x)
    h_T = torch.empty(B, R, dtype=torch.float32, device=dev)
    u = torch.empty_like(x)
    z = torch.empty(B * T, rglru.gate_pitch(R), dtype=torch.float16, device=dev)  # packed coefficients
    ws_gs = torch.empty(rglru.gate_scan_workspace_bytes(B, T, R), dtype=torch.uint8, device=dev)
    ws_scan = torch.empty(rglru.scan_workspace_bytes(B, T, R, torch.bfloat16), dtype=torch.uint8, device=dev)
    ws_fwd = torch.empty(rglru.forward_workspace_bytes(B, T, R, torch.bfloat16), dtype=torch.uint8, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    if args.only == "decode":
        dec = run_decode(torch, rglru, inputs, dev, stream, flush, _peaks(), barrier, max_over_ranks, world)
        replicas.shutdown(rk)
        if rank == 0:
            print(json.dumps({"only": "decode", "decode": dec}))
        return
    if args.only == "block":
        blk = run_block(torch, rglru, inputs, dev, stream, flush, _peaks(), max_over_ranks, world, reps=2)
        replicas.shutdown(rk)
        if rank == 0:
            print(json.dumps({"only": "block", "block": blk}))
        return
    if args.only == "layer":
        lay = run_layer(torch, rglru, inputs, dev, stream, flush, _peaks(), max_over_ranks, world)
        replicas.shutdown(rk)
        if rank == 0:
            print(json.dumps({"only": "layer", "layer": lay}))
        return
    if args.only == "backward":
        bwd = run_backward(torch, rglru, inputs, dev, stream, flush, _peaks(), max_over_ranks, world, reps=3)
        replicas.shutdown(rk)
        if rank == 0:
            print(json.dumps({"only": "backward", "backward": bwd}))
        return

    def forward_step():
        # the timed step: one rglru_forward call (conv, gate GEMM forming the recurrence
        # coefficients, coefficient scan; the last two launched as programmatic dependents)
        rglru.forward(p, x, workspace=ws_fwd, y=y, h_T=h_T, want_conv_state=False)

    def step(ev=None):
        # the same three kernels through the stage entry points, for the per-kernel times
        # (the scan's interval also holds its workspace memset, which rglru_forward leaves
        # to the conv kernel)
        if ev is not None:
            ev[0].record(stream)
        rglru.conv1d(p, x, u=u)
        if ev is not None:
            ev[1].record(stream)
        rglru.gate_coeffs(p, u.view(B * T, R), g=z)
        if ev is not None:
            ev[2].record(stream)
        rglru.scan_coeffs(z, B, T, R, workspace=ws_scan, y=y, h_T=h_T)
        if ev is not None:
            ev[3].record(stream)

    def fused(ev):
        # the alternative second stage: gate GEMM with the scan in its epilogue
        ev[0].record(stream)
        rglru.gate_scan(p, x, u, workspace=ws_gs, y=y, h_T=h_T)
        ev[1].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        forward_step()
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if (rglru.workspace_status(ws_scan) != 0 or rglru.workspace_status(ws_fwd) != 0
            or rglru.workspace_status(None) != 0):
        raise SystemExit("a kernel reported a timeout during warm-up")

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    fevs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    for k in range(K):
        flush.zero_()                 # L2 flush between timed steps (outside the events)
        fevs[k][0].record(stream)
        forward_step()
        fevs[k][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    step_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in fevs) / K)
    status = rglru.workspace_status(ws_fwd)
    # per-kernel times: the same kernels launched one stage call at a time
    for k in range(K):
        flush.zero_()
        step(evs[k])
    torch.cuda.synchronize()
    conv_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / K
    gemm_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / K
    scan_ms = sum(e[2].elapsed_time(e[3]) for e in evs) / K
    status = status or rglru.workspace_status(ws_scan)

    # the fused gate GEMM + scan stage (not part of the timed forward step)
    for _ in range(3):
        flush.zero_()
        fused([torch.cuda.Event(enable_timing=True) for _ in range(2)])
    Ku = max(3, min(K, 30))
    uev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(Ku)]
    for k in range(Ku):
        flush.zero_()
        fused(uev[k])
    torch.cuda.synchronize()
    gs_ms = sum(e[0].elapsed_time(e[1]) for e in uev) / Ku
    if rglru.workspace_status(ws_gs) != 0:
        status = -7

    tokens = B * T
    value = world * tokens / (step_ms / 1e3)
    pk = _peaks()
    # algorithmic bytes / flops per launch (bf16 = 2 B; packed coefficients = 2 × 2 B per channel)
    conv_bytes = tokens * R * 2 * 2                     # read x, write u
    scan_bytes = tokens * R * (4 + 2)                   # read d and b (fp16), write y
    gemm_flops = 2.0 * tokens * (2 * R) * R
    kern = {
        "conv1d": {"ms": conv_ms, "GB/s": conv_bytes / conv_ms / 1e6, "bytes": conv_bytes},
        "gate_gemm": {"ms": gemm_ms, "TFLOP/s": gemm_flops / gemm_ms / 1e9, "flops": gemm_flops},
        "scan": {"ms": scan_ms, "GB/s": scan_bytes / scan_ms / 1e6, "bytes": scan_bytes},
        "gate_scan_fused_alternative": {"ms": gs_ms, "TFLOP/s": gemm_flops / gs_ms / 1e9, "flops": gemm_flops,
                                        "note": "rglru_gate_scan, timed apart; not part of the step"},
    }
    kern["conv1d"]["frac_hbm"] = kern["conv1d"]["GB/s"] / pk["hbm_gbs"]
    kern["scan"]["frac_hbm"] = kern["scan"]["GB/s"] / pk["hbm_gbs"]
    kern["gate_gemm"]["frac_tensor"] = kern["gate_gemm"]["TFLOP/s"] / pk["bf16_tflops"]
    kern["gate_scan_fused_alternative"]["frac_tensor"] = (kern["gate_scan_fused_alternative"]["TFLOP/s"]
                                                          / pk["bf16_tflops"])
    dom = max(("conv1d", "gate_gemm", "scan"), key=lambda k: kern[k]["ms"])
    traffic = None
    src = os.path.join(ROOT, "gated_linear_rnn_conv1d_b200", "csrc",
                       {"gate_gemm": "gemm_tc.cu", "scan": "scan.cu", "conv1d": "conv.cu"}[dom])
    rec = NCU_TRAFFIC.get(dom)
    if rec and rec["src_sha256"] == _sha(src):
        traffic = rec["bytes_per_launch"]
    if dom == "gate_gemm":
        roof = {"bound": "tensor", "achieved": kern[dom]["TFLOP/s"], "peak": pk["bf16_tflops"], "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": kern[dom]["GB/s"], "peak": pk["hbm_gbs"], "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = traffic
    roof["kernel"] = dom
    roof["peak_source"] = ("measured: MEASURED_PEAKS.json burst figure" if pk["source"] == "measured"
                           else "fallback")
    if dom == "gate_gemm" and pk.get("bf16_tflops_sustained"):
        # the GEMM runs power-capped (sw_power_cap) inside the step loop; its fraction of the
        # measured sustained figure, for context (frac above stays against the burst peak)
        roof["frac_of_sustained"] = roof["achieved"] / pk["bf16_tflops_sustained"]

    if args.only == "forward":
        replicas.shutdown(rk)
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
                              "warmup": args.warmup, "ms_per_step": step_ms, "kernels": kern, "roofline": roof,
                              "gpu_launches": 3 * K, "clocks": clk, "only": "forward"}))
        return

    # ---- end to end through the public API, host buffers -----------------------------
    # rglru.forward_host: row groups of the batch pipelined through pinned host copies in
    # both directions and rglru_forward on three streams (the call a user with host data makes)
    x_host = w.x.pin_memory()
    y_host = torch.empty(B, T, R, dtype=torch.bfloat16).pin_memory()
    h_host = torch.empty(B, R, dtype=torch.float32).pin_memory()
    plan = rglru.HostForwardPlan(B, T, R, torch.bfloat16, groups=E2E_GROUPS, slots=3, device=dev)
    e2e_steps = max(3, min(K, 50))
    for _ in range(2):
        rglru.forward_host(p, x_host, y_host, h_host, plan, stream=stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(e2e_steps):
        rglru.forward_host(p, x_host, y_host, h_host, plan, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps)
    e2e = {"value": world * tokens / (e2e_ms / 1e3), "unit": "tokens/s", "ms_per_step": e2e_ms,
           "h2d_bytes_per_step": x.numel() * 2, "d2h_bytes_per_step": y.numel() * 2 + h_T.numel() * 4,
           "api": f"rglru.forward_host: {E2E_GROUPS} row groups, host->device copy, rglru_forward and "
                  "device->host copy of neighbouring groups overlapped on three streams"}
    if plan.status() != 0:
        status = -7

    # ---- decode steps/s ---------------------------------------------------------------
    dec = run_decode(torch, rglru, inputs, dev, stream, flush, pk, barrier, max_over_ranks, world)

    # ---- recurrent block ------------------------------------------------------------------
    blk = run_block(torch, rglru, inputs, dev, stream, flush, pk, max_over_ranks, world)
    # ---- backward of the forward step ---------------------------------------------------
    bwd = run_backward(torch, rglru, inputs, dev, stream, flush, pk, max_over_ranks, world)

    replicas.shutdown(rk)
    if rank != 0:
        return
    cpu = cpu_baseline(inputs) if world == 1 else None
    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) inputs, LeCun-normal gate weights, a^8~U[0.9,0.999])",
        "config": {"workload": "RG-LRU forward, Hawk-scale layer: B=8 T=2048 D_RNN=2048, bf16 IO, fp32 state",
                   "B": B, "T": T, "D_RNN": R, "global_batch": B * world, "seq_len": T,
                   "parallelism": f"replicas x{world} (independent batches, no collective on the data path)",
                   "l2": "flushed before every timed step (256 MB write, outside the step events)"},
        "roofline": roof,
        "kernels": kern,
        "hbm_gb_per_s": {"scan": kern["scan"]["GB/s"], "conv1d": kern["conv1d"]["GB/s"],
                         "peak": pk["hbm_gbs"], "peak_source": pk["source"]},
        "decode": dec,
        "block": blk,
        "backward": bwd,
        "e2e": e2e,
        "gpu_launches": 3 * K,
        "clocks": clk,
        "status": "ok" if status == 0 else "timeout reported",
        "cpu_baseline": cpu,
    }
    print(json.dumps(out))


def run_decode(torch, rglru, inputs, dev, stream, flush, pk, barrier, max_over_ranks, world):
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
        flush.zero_()
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


def run_block(torch, rglru, inputs, dev, stream, flush, pk, max_over_ranks, world, reps=5):
    """The recurrent block (two input linears, conv, gates, scan with the GeLU branch, output
    linear) as one rglru_block_forward call, L2 flushed before each timed call."""
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
        flush.zero_()
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


def run_layer(torch, rglru, inputs, dev, stream, flush, pk, max_over_ranks, world, reps=3):
    """One Hawk residual layer at the recurrent block's sizes with the gated MLP (M = 3):
    RMSNorm, the recurrent block, residual add fused with the second RMSNorm, the MLP's
    three linears and GeLU product, residual add — one rglru_layer_forward call, L2
    flushed before each timed call."""
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
        flush.zero_()
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


def run_backward(torch, rglru, inputs, dev, stream, flush, pk, max_over_ranks, world, reps=5):
    """The backward of the forward step (rglru_backward at the forward workload: recompute
    of u and z, the chunked reverse recurrence with the gate gradients, the ∂u and weight
    gradient GEMMs on transposed copies, the Conv1D backward), L2 flushed before each call."""
    B, T, R = WORKLOAD["B"], WORKLOAD["T"], WORKLOAD["R"]
    w = inputs.make_forward(B, T, R, torch.bfloat16, seed=0)
    p = rglru.Params.from_host(w.params, dev)
    x = w.x.to(dev)
    y, _, _ = rglru.forward(p, x)
    g = torch.Generator("cpu").manual_seed(1)
    dy = torch.randn(B, T, R, generator=g).to(torch.bfloat16).to(dev)
    ws = torch.empty(rglru.backward_workspace_bytes(B, T, R), dtype=torch.uint8, device=dev)
    for _ in range(2):
        rglru.backward(p, x, y, dy, workspace=ws)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in evs:
        flush.zero_()
        a.record(stream)
        rglru.backward(p, x, y, dy, workspace=ws)
        b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / reps)
    n_tok = B * T
    # tensor-core work: z recomputed (2·N·2R·R), ∂u (2·N·2R·R), ∂W_a and ∂W_x (2·2R·R·N)
    flops = 3 * 2.0 * n_tok * (2 * R) * R
    status = rglru.workspace_status(ws)
    del ws, x, y, dy
    return {"workload": f"RG-LRU backward B={B} T={T} D_RNN={R} bf16 (dL/dy given)", "ms_per_call": ms,
            "tokens_per_s": world * n_tok / (ms / 1e3), "gemm_flops_per_call": flops,
            "gemm_TFLOP/s_over_the_call": flops / ms / 1e9, "status": status, "gpu_launches_per_call": 14,
            "timing": f"{reps} calls, L2 flushed before each"}


# ------------------------------------------------------------------------------ CPU side
def _host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


_HOST_WORKLOAD = {}


def _host_workload(inputs):
    """The bench workload's inputs on the host (generated once per process)."""
    import torch
    if "w" not in _HOST_WORKLOAD:
        _HOST_WORKLOAD["w"] = inputs.make_forward(WORKLOAD["B"], WORKLOAD["T"], WORKLOAD["R"], torch.bfloat16, seed=0)
    return _HOST_WORKLOAD["w"]


def _oracle_sample(inputs, row=0, steps=512):
    """The oracle on batch row `row`, its first `steps` steps, all channels of the workload."""
    import oracle
    w = _host_workload(inputs)
    pr = w.params
    x = w.x[row:row + 1, :steps]
    t0 = time.perf_counter()
    oracle.rglru_forward(x, pr.conv_w, pr.conv_b, pr.W_a, pr.b_a, pr.W_x, pr.b_x, pr.Lambda)
    dt = time.perf_counter() - t0
    return steps, dt


CPU_SAMPLE_SECONDS = 10.0
E2E_GROUPS = 4   # row groups of the batch that forward_host pipelines in the e2e measurement


def cpu_baseline(inputs):
    from threadpoolctl import threadpool_limits
    _oracle_sample(inputs, row=0, steps=512)          # untimed: first touch of host memory
    tok, dt, n = 0, 0.0, 0
    while dt < CPU_SAMPLE_SECONDS:
        t, d = _oracle_sample(inputs, row=n % WORKLOAD["B"], steps=WORKLOAD["T"])
        tok += t
        dt += d
        n += 1
    # the same oracle with its BLAS held to one thread (the recurrence is single-threaded numpy)
    tok1, dt1, n1 = 0, 0.0, 0
    with threadpool_limits(limits=1):
        while dt1 < CPU_SAMPLE_SECONDS / 2:
            t, d = _oracle_sample(inputs, row=n1 % WORKLOAD["B"], steps=WORKLOAD["T"])
            tok1 += t
            dt1 += d
            n1 += 1
    return {"value": tok / dt, "unit": "tokens/s", "cores": _host_cores(), "kind": "oracle",
            "sample": f"{n} batch rows (cycling over the {WORKLOAD['B']} rows) x {WORKLOAD['T']} steps x "
                      f"{WORKLOAD['R']} channels of the workload, {dt:.1f} s; float64 numpy, BLAS matmul on the "
                      "host cores, recurrence vectorised over channels",
            "single_core": {"value": tok1 / dt1, "unit": "tokens/s", "cores": 1,
                            "sample": f"{n1} batch rows, {dt1:.1f} s, BLAS limited to one thread"}}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    from gated_linear_rnn_conv1d_b200 import inputs
    for i in range(args.warmup):
        _oracle_sample(inputs, row=i % WORKLOAD["B"])
    tot_tok, tot_dt = 0, 0.0
    for i in range(args.steps):
        tok, dt = _oracle_sample(inputs, row=i % WORKLOAD["B"])
        tot_tok += tok
        tot_dt += dt
    value = tot_tok / tot_dt
    cores = _host_cores()
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "RG-LRU forward, Hawk-scale layer: B=8 T=2048 D_RNN=2048, bf16 IO, fp32 state",
                   "B": WORKLOAD["B"], "T": WORKLOAD["T"], "D_RNN": WORKLOAD["R"]},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": "per step: 1 batch row x 512 steps x 2048 channels of the workload"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["own", "reference"], default="own")
    ap.add_argument("--only", choices=["all", "forward", "decode", "block", "backward", "layer"], default="all",
                    help="forward / decode / block / backward / layer: time that part only (small commands for profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_own(args)


if __name__ == "__main__":
    main()
