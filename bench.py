#!/usr/bin/env python
"""Benchmark of the NVFP4 MoE layer hot path on B200.

One step = one moe_forward call over one batch: grouped top-8 routing, token
permutation, NVFP4 activation quantisation (unit global), gate/up grouped GEMM
+ SwiGLU (+ requantisation), down grouped GEMM x routing weight, weighted
un-permute.  Default workload: the 8192-token W4A4 prefill layer (H=4096,
I=2048, 256 experts in 8 groups, keep 4, top-8, scaling 2.827).  At N=1 the
run also measures, as nested objects, the W4A16 decode layer (T=16, also with
compact scales), the W4A8 prefill layer, the 65536-token skewed W4A4 layer on
128 experts, the MXFP4->NVFP4 transcode of one layer of expert weights and the
fused router.  Every timed step runs between its own CUDA events after an L2
flush (256 MB written outside the events).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

For N > 1 it is launched by torchrun, one rank per GPU; every rank runs the
same-shaped workload on its own batch (independent problems, no collective on
the data path), timings are the max over ranks and `value` is the total tokens
of all ranks per second ("scaling": "weak").  `--impl reference` times the CPU
oracle (the parity reference) on a bounded token sample per step instead.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from nvfp4_mixture_experts_grouped_b200 import inputs  # noqa: E402

N_TRACE = 7
STAGES = ["route", "permute", "quantize", "gateup_gemm", "down_gemm", "combine"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["prefill", "skewed", "decode", "decode_pow2", "prefill_pow2"],
                    default="prefill")
    ap.add_argument("--no-extras", action="store_true", help="skip the decode and transcode sub-measurements")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-tokens", type=int, default=0, help="oracle tokens per step (0 = host threads)")
    ap.add_argument("--tokens", type=int, default=0, help="override T (smaller cases for profiling)")
    ap.add_argument("--experts", type=int, default=0, help="override E (smaller cases for profiling)")
    ap.add_argument("--transcode-only", action="store_true",
                    help="run only the transcode sub-measurement and print its JSON (profiling)")
    ap.add_argument("--transcode-experts", type=int, default=256,
                    help="experts of the transcode sub-measurement's layer (smaller cases for profiling)")
    ap.add_argument("--router-only", action="store_true",
                    help="run only the router sub-measurement and print its JSON (profiling)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "src": "fallback"}


# nominal dense FP4 : BF16 and FP8 : BF16 tensor-core throughput on B200 (9 : 4.5 : 2.25 PFLOP/s)
FP4_OVER_BF16 = 4.0
FP8_OVER_BF16 = 2.0
# B200 specification figures, for the second set of fractions
SPEC_FP4_TFLOPS = 9000.0
SPEC_FP8_TFLOPS = 4500.0
SPEC_HBM_GBS = 8000.0
# Rate of the block-scaled FP4 pair MMA (cta_group::2, M=256, N=256, K=64) that one
# thread issuing back to back on resident operands reaches: one every 128 SM
# cycles per CTA pair, i.e. 32,768 FLOP per cycle per SM (9.53 PFLOP/s at the
# 1965 MHz maximum clock over 148 SMs).  Scaled by the SM clock sampled during
# the timed region.
MMA_FP4_FLOP_PER_CYCLE_PER_SM = 2 * 256 * 256 * 64 / 128 / 2
N_SMS = 148
# between timed steps this much memory is written, more than the 126 MB L2
L2_FLUSH_BYTES = 256 << 20

MODE_NAMES = {0: "W4A16", 1: "W4A4", 2: "W4A16 compact scales", 3: "W4A8 (MXFP8 x FP4)"}
MODE_DTYPES = {0: "bf16 activations x fp4 e2m1 weights (e4m3 block scales), fp16 mma -> f32",
               1: "fp4 e2m1 (e4m3 block scales) x fp4 -> f32",
               2: "bf16 activations x fp4 e2m1 weights (compact power-of-two scales), fp16 mma -> f32",
               3: "fp8 e4m3 (e8m0 block scales) x fp4 e2m1 (e8m0 block scales) -> f32"}

# DRAM bytes (read + write) per launch from ncu captures of smaller cases of
# the same kernels (profiles/), valid for these kernel versions and workloads only:
#  - k_w4a4_gemm gate/up, W4A4, single-CTA form (k_w4a4_gemm_traffic_prefill2k_e64.txt:
#    653.8 MB read + 19.9 MB written at T=2048, E=64), scaled x4 to T=8192, E=256
#    (weights and activations both grow 4x);
#  - the same for W4A8 (same file: 656.7 MB + 33.4 MB);
#  - k_w16_gateup + k_w16_down of one 16-token decode step at E=256 (the bench's
#    own workload, captured at full size: k_w16_decode16.txt).
GATEUP_TRAFFIC_T8192_E256 = 4 * (653826816 + 19891200)
GATEUP_W4A8_TRAFFIC_T8192_E256 = 4 * (656710656 + 33436160)
DECODE_TRAFFIC_T16_E256 = 1010.475e6 + 4.71296e6 + 505.455e6 + 5.101568e6
#  - k_transcode out of place (k_transcode_layer96.txt: 427.9 MB read + 404.6 MB
#    written for a 96-tensor layer), scaled x8 to the 768-tensor layer timed here.
TRANSCODE_TRAFFIC_768 = 8 * (427850240 + 404599296)


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    def __init__(self, index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={index}", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                       "-lms", "20"], stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def wait_ready(self, timeout_s: float = 10.0):
        """Block until nvidia-smi has written its first sample (its start-up takes
        longer than a short timed region)."""
        t0 = time.time()
        while self.p is not None and time.time() - t0 < timeout_s:
            if os.path.getsize(self.f.name) > 0:
                return
            time.sleep(0.02)

    def mark(self):
        """Samples before this point (start-up, warm-up) are not reported."""
        self.offset = os.path.getsize(self.f.name) if self.p is not None else 0

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.seek(0)
        text = self.f.read()
        during = text[getattr(self, "offset", 0):]
        # a timed region shorter than the sampling interval may hold no sample:
        # then the last one taken before its end stands for it
        lines = [r for r in during.strip().splitlines() if r.strip()] or text.strip().splitlines()[-1:]
        rows = [r.split(",") for r in lines if r.strip()]
        os.unlink(self.f.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if len(r) > 5 + i and r[5 + i].strip() == "Active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def workload(args):
    import dataclasses

    wl = inputs.WORKLOADS[args.workload]
    if args.tokens:
        wl = dataclasses.replace(wl, T=args.tokens)
    if args.experts:
        wl = dataclasses.replace(wl, E=args.experts)
    return wl


def launches_per_step(mode, T, wl):
    """Kernels one moe_forward launches (the library's dispatch): routing 1; the
    permutation 1 fused kernel up to 8192 pairs with E <= 256, else 3; then W4A4 /
    W4A8: quantise 1 + gate/up 1 + down 1; W4A16 (either scale form): two FP16
    conversions + gate/up 1 + down 1; the combine 1."""
    permute = 1 if (wl.E <= 256 and T * wl.top_k <= 8192) else 3
    layer = 3 if mode in (1, 3) else 4
    return 1 + permute + layer + 1


def config_of(wl, T, world):
    """The workload description both arms print."""
    weights_gb = wl.E * 3 * wl.H * wl.I * (0.5 + 1.0 / 16) / 1e9  # NVFP4 codes + E4M3 scales
    return {"workload": f"{wl.name}: T={T} H={wl.H} I={wl.I} E={wl.E} groups={wl.n_group} keep={wl.topk_group} "
                        f"top_k={wl.top_k} rsf={wl.rsf} {MODE_NAMES[wl.mode]}",
            "global_batch": T * world, "tokens_per_gpu": T, "parallelism": f"replicas{world}",
            "l2": f"L2 flushed between timed steps ({L2_FLUSH_BYTES >> 20} MB written, outside the step's events); "
                  f"inputs larger than L2 too ({weights_gb:.2f} GB of expert weights per step)"}


def layer_flops(T, H, I, k):
    return 6.0 * T * k * H * I


def gemm_roofline(moe, mode, wl, T, gateup_ms, P, clocks, traffic):
    """Roofline of the gate/up GEMM launch (the step's dominant kernel).  Peak:
    the measured burst bf16 GEMM rate scaled by the nominal dense FP4:BF16 (FP8
    for W4A8) ratio -- the kernel is timed in a region of tens of milliseconds,
    too short for the power cap to lower the clock (the clocks sampled during it
    are reported beside it).  Also: the fraction of the B200 specification
    figure, of the pair MMA's own issue rate at the sampled clock, and the HBM
    view (algorithmic bytes: the expert weights once, the input codes and scales
    of every pair, the intermediate codes and scales written)."""
    fp4 = mode == moe.W4A4
    flops = 4.0 * T * wl.top_k * wl.H * wl.I  # padding excluded
    t_kernel = gateup_ms / 1e3
    achieved = flops / t_kernel / 1e12
    ratio = FP4_OVER_BF16 if fp4 else FP8_OVER_BF16
    peak = P["bf16_tflops"] * ratio
    spec = SPEC_FP4_TFLOPS if fp4 else SPEC_FP8_TFLOPS
    P_pairs = T * wl.top_k
    act_b = 0.5 + 1.0 / 16 if fp4 else 1.0 + 1.0 / 32  # bytes per activation element with its scale
    nbytes = wl.E * 2 * wl.I * wl.H * (0.5 + 1.0 / 16) + P_pairs * (wl.H + wl.I) * act_b
    gbs = nbytes / t_kernel / 1e9
    r = {"bound": "tensor", "kernel": "k_w4a4_gemm<gate/up>" + ("" if fp4 else ", FP8 x FP4"),
         "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
         "traffic": traffic, "traffic_unit": "bytes per launch (ncu dram read+write)",
         "peak_src": f"{P['src']} bf16 burst x {ratio:g} (nominal dense {'FP4' if fp4 else 'FP8'}:BF16)",
         "algorithmic_flops_per_launch": flops,
         "frac_of_spec": round(achieved / spec, 4), "spec_tflops": spec,
         "hbm": {"algorithmic_bytes_per_launch": int(nbytes), "achieved_gbs": round(gbs, 1),
                 "frac_of_measured": round(gbs / P["hbm_gbs"], 4), "frac_of_spec": round(gbs / SPEC_HBM_GBS, 4)}}
    mhz = (clocks or {}).get("sm_mhz")
    if fp4 and mhz:
        pace = MMA_FP4_FLOP_PER_CYCLE_PER_SM * N_SMS * mhz * 1e6 / 1e12
        r["frac_of_mma_pace"] = round(achieved / pace, 4)
        r["mma_pace_tflops"] = round(pace, 1)
    return r


def max_over_ranks(torch, dist, ms, device):
    """The slowest rank's time: the job is done only when every rank is."""
    if dist is None:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank, world, ms):
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * world / (ms / 1e3)


def rank_batch(wl, d, rank):
    """Rank r > 0 gets its own seeded batch (activations, logits); the layer's
    weights are the same on every rank."""
    if rank == 0:
        return d["x"], d["logits"]
    rng = np.random.default_rng(wl.seed * 1000 + rank)
    return inputs.activations(rng, wl.T, wl.H, wl.outliers), inputs.router_logits(rng, wl.T, wl.E, wl.zipf)


def make_layer(torch, moe, mode, w, T, wl):
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    E, I, hh = w["gate_codes"].shape
    H = hh * 2
    packed = torch.empty(moe.moe_packed_weights_size(mode, E, H, I), dtype=torch.uint8, device="cuda")
    tw = {k: dev(v) for k, v in w.items()}
    moe.moe_pack_weights(mode, tw["gate_codes"], tw["gate_sf"], tw["up_codes"], tw["up_sf"], tw["down_codes"],
                         tw["down_sf"], tw["w_global"], packed)
    torch.cuda.synchronize()
    del tw
    ws = torch.empty(moe.moe_forward_workspace_size(mode, T, H, I, E, wl.top_k), dtype=torch.uint8, device="cuda")
    return packed, ws


class L2Flush:
    """Writes L2_FLUSH_BYTES (more than the L2) on the current stream, between
    timed steps and outside their events, so no step finds the previous step's
    data in L2."""

    def __init__(self, torch):
        self.buf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.int32, device="cuda")
        self.n = 0

    def __call__(self):
        self.n += 1
        self.buf.fill_(self.n)


def time_layer(torch, moe, mode, packed, ws, x, logits, out, wl, T, steps, warmup, trace=True, on_start=None,
               on_end=None):
    """Returns (ms per step, per-stage ms means), both timed with CUDA events on the current
    stream, each step between its own pair of events with an L2 flush before it.  The step
    time comes from a pass without stage events (recording 7 events per step costs a few
    microseconds, visible at decode sizes); the stage times from a second, traced pass of
    the same steps."""
    H, I, E = wl.H, wl.I, wl.E
    flush = L2Flush(torch)

    def step():
        moe.moe_forward(mode, x, logits, None, packed, 1.0, T, H, I, E, wl.n_group, wl.topk_group, wl.top_k, wl.rsf,
                        True, ws, out)

    for _ in range(warmup):
        flush()
        step()
    torch.cuda.synchronize()
    if on_start:
        on_start()
    marks = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in marks:
        flush()
        a.record()
        step()
        b.record()
    torch.cuda.synchronize()
    moe.nvfp4moe_check_device_status()
    ms = float(np.sum([a.elapsed_time(b) for a, b in marks])) / steps
    if on_end:
        on_end()
    stage = None
    if trace:
        evs = []
        for _ in range(steps):
            row = [torch.cuda.Event(enable_timing=True) for _ in range(N_TRACE)]
            for e in row:
                e.record()
            evs.append(row)
        torch.cuda.synchronize()
        for i in range(steps):
            flush()
            moe.nvfp4moe_set_trace_events(evs[i])
            step()
        torch.cuda.synchronize()
        moe.nvfp4moe_set_trace_events(None)
        moe.nvfp4moe_check_device_status()
        stage = {}
        for s, name in enumerate(STAGES):
            stage[name] = float(np.mean([evs[i][s].elapsed_time(evs[i][s + 1]) for i in range(steps)]))
    return ms, stage


def time_e2e(torch, moe, mode, packed, ws, d, wl, T, steps, warmup):
    """ms per step of the pipelined host-buffer loop (see run_ours)."""
    xh = torch.from_numpy(d["x"].view(np.int16)).pin_memory()
    lh = torch.from_numpy(d["logits"]).pin_memory()
    oh = [torch.empty((T, wl.H), dtype=torch.int16).pin_memory() for _ in range(2)]
    xd = [torch.empty((T, wl.H), dtype=torch.int16, device="cuda") for _ in range(2)]
    ld = [torch.empty((T, wl.E), dtype=torch.float32, device="cuda") for _ in range(2)]
    od = [torch.empty((T, wl.H), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    up, ran, down = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    used = [False, False]

    def step(i):
        b = i & 1
        with torch.cuda.stream(s_in):
            if used[b]:
                s_in.wait_event(ran[b])  # the layer of step i-2 has read these inputs
            xd[b].copy_(xh, non_blocking=True)
            ld[b].copy_(lh, non_blocking=True)
            up[b].record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(up[b])
            if used[b]:
                s_run.wait_event(down[b])  # step i-2's output has left the device
            moe.moe_forward(mode, xd[b].view(torch.bfloat16), ld[b], None, packed, 1.0, T, wl.H, wl.I, wl.E,
                            wl.n_group, wl.topk_group, wl.top_k, wl.rsf, True, ws, od[b], stream=s_run)
            ran[b].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ran[b])
            oh[b].copy_(od[b].view(torch.int16), non_blocking=True)
            down[b].record(s_out)
        used[b] = True

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for i in range(steps):
        step(warmup + i)
    # the last step's download ends the region
    s_out.wait_event(down[(warmup + steps - 1) & 1])
    z.record(s_out)
    torch.cuda.synchronize()
    # every step really produced its output on the host
    ref = od[(warmup + steps - 1) & 1].view(torch.int16).cpu()
    assert torch.equal(oh[(warmup + steps - 1) & 1], ref)
    return a.elapsed_time(z) / steps


def run_ours(args, rank, world, local_rank):
    import torch

    import nvfp4_mixture_experts_grouped_b200 as moe

    torch.cuda.set_device(local_rank)
    P = peaks()
    if args.transcode_only or args.router_only:
        if rank == 0:
            sub = bench_transcode if args.transcode_only else bench_router
            print(json.dumps(sub(torch, moe, args, P)), flush=True)
        return
    wl = workload(args)
    T = wl.T
    # host-side input generation (about a minute at the 8K prefill) runs before
    # the process group exists, so no collective waits on it
    d = inputs.moe_inputs(wl)
    w = {k: d[k] for k in ("gate_codes", "gate_sf", "up_codes", "up_sf", "down_codes", "down_sf", "w_global")}
    d["x"], d["logits"] = rank_batch(wl, d, rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local_rank))
    mode = wl.mode
    packed, ws = make_layer(torch, moe, mode, w, T, wl)
    x = torch.from_numpy(d["x"].view(np.int16)).cuda().view(torch.bfloat16)
    logits = torch.from_numpy(d["logits"]).cuda()
    out = torch.empty((T, wl.H), dtype=torch.bfloat16, device="cuda")

    # ----------------------------------------------------------------- timed region
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank) if rank == 0 else None
    if sampler:
        sampler.wait_ready()
    held = {}

    def end_of_region():
        if sampler:
            held["clocks"] = sampler.stop()

    ms, stage = time_layer(torch, moe, mode, packed, ws, x, logits, out, wl, T, args.steps, args.warmup,
                           on_start=sampler.mark if sampler else None, on_end=end_of_region)
    clocks = held.get("clocks")
    ms = max_over_ranks(torch, dist, ms, "cuda")
    if dist:
        dist.barrier()
    value = job_tokens_per_s(T, world, ms)

    # ----------------------------------------------------------------- end to end
    # A stream of batches through the public API with host buffers: every step
    # uploads its x and logits from pinned host memory, runs moe_forward and
    # downloads its output to pinned host memory, all inside the timed region.
    # Uploads, layer and downloads run on three streams with double-buffered
    # device inputs and outputs, so step i+1's upload and step i-1's download
    # overlap step i's layer (PCIe is full duplex); the layer calls are ordered on
    # one stream and share one workspace.
    e2e_ms = time_e2e(torch, moe, mode, packed, ws, d, wl, T, args.steps, args.warmup)
    e2e_ms = max_over_ranks(torch, dist, e2e_ms, "cuda")

    # ----------------------------------------------------------------- roofline
    if mode in (moe.W4A4, moe.W4A8):
        full = (T, wl.E, wl.H, wl.I) == (8192, 256, 4096, 2048)
        traffic = (GATEUP_TRAFFIC_T8192_E256 if mode == moe.W4A4 else GATEUP_W4A8_TRAFFIC_T8192_E256) if full else None
        roofline = gemm_roofline(moe, mode, wl, T, stage["gateup_gemm"], P, clocks, traffic)
    else:
        # W4A16 weight stream: every active expert's codes + E4M3 scales read once
        ids_t = torch.empty((T, wl.top_k), dtype=torch.int32, device="cuda")
        w_t = torch.empty((T, wl.top_k), dtype=torch.float32, device="cuda")
        moe.moe_route(logits, None, wl.n_group, wl.topk_group, wl.top_k, wl.rsf, True, ids_t, w_t)
        active = int(torch.unique(ids_t).numel())
        if mode == moe.W4A16C:  # codes + a 4-bit field per 32 weights + an exponent byte per row
            wbytes = active * ((2 * wl.I * wl.H + wl.H * wl.I) * (0.5 + 1.0 / 64) + (2 * wl.I + wl.H))
        else:
            wbytes = active * (2 * wl.I * wl.H + wl.H * wl.I) * (0.5 + 1.0 / 16)
        t_kernel = (stage["gateup_gemm"] + stage["down_gemm"]) / 1e3
        achieved = wbytes / t_kernel / 1e9
        roofline = {"bound": "hbm", "kernel": "k_w16_gateup + k_w16_down", "achieved": round(achieved, 1),
                    "peak": P["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / P["hbm_gbs"], 4),
                    "frac_of_spec": round(achieved / SPEC_HBM_GBS, 4),
                    "traffic": (DECODE_TRAFFIC_T16_E256 if mode == moe.W4A16 and wl.name == "decode" and T == 16
                                and wl.E == 256 else None),
                    "traffic_unit": "bytes per step of both GEMM launches (ncu dram read+write)",
                    "peak_src": f"{P['src']} copy bandwidth", "algorithmic_bytes_per_step": int(wbytes),
                    "active_experts": active}

    res = {
        "metric": "MoE-layer tokens/s", "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": MODE_DTYPES[mode],
        "data": "synthetic",
        "config": config_of(wl, T, world),
        "roofline": roofline,
        "stages_ms": {k: round(v, 4) for k, v in stage.items()},
        "e2e": {"value": round(job_tokens_per_s(T, world, e2e_ms), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": int(d["x"].nbytes + d["logits"].nbytes), "d2h_bytes_per_step": int(T * wl.H * 2)},
        "gpu_launches": launches_per_step(mode, T, wl) * args.steps,
        "clocks": clocks,
        "tflops": round(layer_flops(T, wl.H, wl.I, wl.top_k) / (ms / 1e3) / 1e12, 2),
    }
    del packed, ws
    torch.cuda.empty_cache()

    if world == 1 and not args.no_extras and rank == 0:
        res["decode"] = bench_decode(torch, moe, w, args, P)
        del w
        res["decode_compact"] = bench_decode(torch, moe, None, args, P, compact=True)
        res["prefill_w4a8"] = bench_w4a8(torch, moe, args, P)
        res["skewed"] = bench_skewed(torch, moe, args, P)
        res["transcode"] = bench_transcode(torch, moe, args, P)
        res["router"] = bench_router(torch, moe, args, P)
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(wl, d, args)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def bench_decode(torch, moe, w, args, P, compact=False):
    """W4A16 decode layer (T=16): tokens/s and weight-stream HBM GB/s.  compact:
    the same layer on weights with the transcode's scale structure, stored with
    compact scales (mode W4A16C, 4.125 bits per weight)."""
    mode = moe.W4A16C if compact else moe.W4A16
    if compact:
        wl = inputs.WORKLOADS["decode_pow2"]
        d = inputs.moe_inputs(wl)
        w = {k: d[k] for k in ("gate_codes", "gate_sf", "up_codes", "up_sf", "down_codes", "down_sf", "w_global")}
        x, lg = d["x"], d["logits"]
        del d
    else:
        wl = inputs.WORKLOADS["decode"]
        rng = np.random.default_rng(wl.seed)
        x = inputs.activations(rng, wl.T, wl.H)
        lg = inputs.router_logits(rng, wl.T, wl.E)
    xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    ld = torch.from_numpy(lg).cuda()
    out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    same_weights = None
    if compact:
        # the plain W4A16 form of the same weights, for comparison (same outputs bit for bit)
        packed, ws = make_layer(torch, moe, moe.W4A16, w, wl.T, wl)
        ms16, _ = time_layer(torch, moe, moe.W4A16, packed, ws, xd, ld, out, wl, wl.T, max(args.steps, 20),
                             args.warmup, trace=False)
        same_weights = {"mode": "W4A16", "ms_per_step": round(ms16, 4)}
        del packed, ws
        torch.cuda.empty_cache()
    packed, ws = make_layer(torch, moe, mode, w, wl.T, wl)
    del w
    ms, stage = time_layer(torch, moe, mode, packed, ws, xd, ld, out, wl, wl.T, max(args.steps, 20), args.warmup)
    ids = torch.empty((wl.T, wl.top_k), dtype=torch.int32, device="cuda")
    wts = torch.empty((wl.T, wl.top_k), dtype=torch.float32, device="cuda")
    moe.moe_route(ld, None, wl.n_group, wl.topk_group, wl.top_k, wl.rsf, True, ids, wts)
    active = int(torch.unique(ids).numel())
    if compact:  # codes + a 4-bit field per 32 weights + an exponent byte per row
        per_expert = (2 * wl.I * wl.H + wl.H * wl.I) * (0.5 + 1.0 / 64) + (2 * wl.I + wl.H)
    else:  # codes + E4M3 scales
        per_expert = (2 * wl.I * wl.H + wl.H * wl.I) * (0.5 + 1.0 / 16)
    gemm_ms = stage["gateup_gemm"] + stage["down_gemm"]
    wbytes = active * per_expert
    achieved = wbytes / (gemm_ms / 1e3) / 1e9
    del packed, ws
    torch.cuda.empty_cache()
    name = "W4A16 compact scales (4.125 bits per weight)" if compact else "W4A16"
    return {"workload": f"{wl.name}: T={wl.T} H={wl.H} I={wl.I} E={wl.E} top_k={wl.top_k} {name}",
            "value": round(wl.T / (ms / 1e3), 1), "unit": "tokens/s", "ms_per_step": round(ms, 4),
            "active_experts": active, "stages_ms": {k: round(v, 4) for k, v in stage.items()},
            **({"same_weights": same_weights} if same_weights else {}),
            "roofline": {"bound": "hbm", "kernel": "k_w16_gateup + k_w16_down", "achieved": round(achieved, 1),
                         "peak": P["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / P["hbm_gbs"], 4),
                         "frac_of_spec": round(achieved / SPEC_HBM_GBS, 4),
                         "step_frac_of_spec": round(wbytes / (ms / 1e3) / 1e9 / SPEC_HBM_GBS, 4),
                         "traffic": None if compact else DECODE_TRAFFIC_T16_E256,
                         "traffic_unit": "bytes per step of both GEMM launches (ncu dram read+write)",
                         "algorithmic_bytes_per_step": int(wbytes)}}


def bench_w4a8(torch, moe, args, P):
    """W4A8 prefill layer (MXFP8 activations x FP4 weights, T=8192) on weights with
    the transcode's scale structure; the W4A4 layer on the same weights beside it.
    The FP8 x FP4 MMA runs at the FP8 rate, so the denominator is the FP8 peak."""
    wl = inputs.WORKLOADS["prefill_pow2"]
    d = inputs.moe_inputs(wl)
    w = {k: d[k] for k in ("gate_codes", "gate_sf", "up_codes", "up_sf", "down_codes", "down_sf", "w_global")}
    xd = torch.from_numpy(d["x"].view(np.int16)).cuda().view(torch.bfloat16)
    ld = torch.from_numpy(d["logits"]).cuda()
    del d
    out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    packed, ws = make_layer(torch, moe, moe.W4A4, w, wl.T, wl)
    ms4, _ = time_layer(torch, moe, moe.W4A4, packed, ws, xd, ld, out, wl, wl.T, args.steps, args.warmup, trace=False)
    del packed, ws
    torch.cuda.empty_cache()
    packed, ws = make_layer(torch, moe, moe.W4A8, w, wl.T, wl)
    del w
    ms, stage = time_layer(torch, moe, moe.W4A8, packed, ws, xd, ld, out, wl, wl.T, args.steps, args.warmup)
    del packed, ws
    torch.cuda.empty_cache()
    return {"workload": f"{wl.name}: T={wl.T} H={wl.H} I={wl.I} E={wl.E} top_k={wl.top_k} W4A8 (MXFP8 x FP4)",
            "value": round(wl.T / (ms / 1e3), 1), "unit": "tokens/s", "ms_per_step": round(ms, 4),
            "stages_ms": {k: round(v, 4) for k, v in stage.items()},
            "same_weights": {"mode": "W4A4", "ms_per_step": round(ms4, 4)},
            "roofline": gemm_roofline(moe, moe.W4A8, wl, wl.T, stage["gateup_gemm"], P, None,
                                      GATEUP_W4A8_TRAFFIC_T8192_E256)}


def bench_skewed(torch, moe, args, P):
    """The long skewed prefill: T=65536 on the 128-expert pruned layer (8 groups of
    16), router logits with a Zipf(1.1) per-expert bias, W4A4.  Reports the
    per-expert load (pairs routed to each expert) beside the stage times."""
    wl = inputs.WORKLOADS["skewed"]
    d = inputs.moe_inputs(wl)
    w = {k: d[k] for k in ("gate_codes", "gate_sf", "up_codes", "up_sf", "down_codes", "down_sf", "w_global")}
    xd = torch.from_numpy(d["x"].view(np.int16)).cuda().view(torch.bfloat16)
    ld = torch.from_numpy(d["logits"]).cuda()
    del d
    out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    packed, ws = make_layer(torch, moe, moe.W4A4, w, wl.T, wl)
    del w
    ms, stage = time_layer(torch, moe, moe.W4A4, packed, ws, xd, ld, out, wl, wl.T, args.steps, args.warmup)
    ids = torch.empty((wl.T, wl.top_k), dtype=torch.int32, device="cuda")
    wts = torch.empty((wl.T, wl.top_k), dtype=torch.float32, device="cuda")
    moe.moe_route(ld, None, wl.n_group, wl.topk_group, wl.top_k, wl.rsf, True, ids, wts)
    load = torch.bincount(ids.reshape(-1).long(), minlength=wl.E).cpu().numpy()
    del packed, ws, xd, ld, out, ids, wts
    torch.cuda.empty_cache()
    return {"workload": f"{wl.name}: T={wl.T} H={wl.H} I={wl.I} E={wl.E} groups={wl.n_group} keep={wl.topk_group} "
                        f"top_k={wl.top_k} rsf={wl.rsf} W4A4, logits + Zipf(1.1) expert bias",
            "value": round(wl.T / (ms / 1e3), 1), "unit": "tokens/s", "ms_per_step": round(ms, 4),
            "tflops": round(layer_flops(wl.T, wl.H, wl.I, wl.top_k) / (ms / 1e3) / 1e12, 2),
            "stages_ms": {k: round(v, 4) for k, v in stage.items()},
            "expert_load": {"pairs_per_expert": [int(v) for v in load], "max": int(load.max()),
                            "min": int(load.min()), "mean": round(float(load.mean()), 1)},
            "roofline": gemm_roofline(moe, moe.W4A4, wl, wl.T, stage["gateup_gemm"], P, None, None)}


def bench_router(torch, moe, args, P):
    """Router projection + grouped top-k (moe_router_topk) at the decode shape:
    T=16 BF16 hidden rows x an FP32 router [256, 4096].  Successive calls use the
    routers of 47 distinct layers (188 MB > L2), as a model stepping through its
    MoE layers does, so every call reads its router from HBM."""
    wl = inputs.WORKLOADS["decode"]
    T, H, E, layers = wl.T, wl.H, wl.E, 47
    rng = np.random.default_rng(wl.seed + 100)
    x = torch.from_numpy(inputs.bf16_bits(rng.standard_normal((T, H), dtype=np.float32)).view(np.int16)).cuda()
    w = torch.empty((layers, E, H), dtype=torch.float32, device="cuda")
    for l in range(layers):
        w[l].copy_(torch.from_numpy(inputs.router_weights(rng, E, H)))
    logits = torch.empty((T, E), dtype=torch.float32, device="cuda")
    ids = torch.empty((T, wl.top_k), dtype=torch.int32, device="cuda")
    wts = torch.empty((T, wl.top_k), dtype=torch.float32, device="cuda")
    ws = torch.zeros(max(16, moe.moe_router_topk_workspace_size(T)), dtype=torch.uint8, device="cuda")

    def call(l):
        moe.moe_router_topk(x, w[l], None, wl.n_group, wl.topk_group, wl.top_k, wl.rsf, True, logits, ids, wts, ws)

    for l in range(layers):
        call(l)
    torch.cuda.synchronize()
    reps = max(args.steps, 20)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # eager: one library call per layer from Python (host-bound at this size)
    a.record()
    for i in range(reps * layers):
        call(i % layers)
    b.record()
    torch.cuda.synchronize()
    eager_us = a.elapsed_time(b) / (reps * layers) * 1e3
    # device time: the 47 calls captured once in a CUDA graph, as a decode step is
    g = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream()
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=cs):
        for l in range(layers):
            call(l)
    g.replay()
    torch.cuda.synchronize()
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    moe.nvfp4moe_check_device_status()
    us = a.elapsed_time(b) / (reps * layers) * 1e3
    del g
    nbytes = E * H * 4 + T * H * 2 + T * E * 4 + T * wl.top_k * 8
    gbs = nbytes / (us / 1e6) / 1e9
    del w
    torch.cuda.empty_cache()
    prefill = bench_router_prefill(torch, moe, args)
    return {"prefill": prefill,
            "workload": f"router: T={T} H={H} E={E} groups={wl.n_group} keep={wl.topk_group} top_k={wl.top_k}, "
                        f"FP32 router, {layers} layers' routers rotated (> L2)",
            "value": round(us, 2), "unit": "us per layer (CUDA graph of 47 layers' calls)",
            "higher_is_better": False, "eager_us_per_call": round(eager_us, 2),
            "roofline": {"bound": "hbm", "kernel": "k_router_logits + k_route_rows", "achieved": round(gbs, 1),
                         "peak": P["hbm_gbs"],
                         "unit": "GB/s", "frac": round(gbs / P["hbm_gbs"], 4), "traffic": None,
                         "frac_of_spec": round(gbs / SPEC_HBM_GBS, 4),
                         "algorithmic_bytes_per_launch": int(nbytes)}}


# FP32 FMA peak of the CUDA cores, derived from unit counts and the clock: SMs x
# 128 FP32 lanes x 2 FLOP x 1.965 GHz (the maximum SM clock), 74.4 TFLOP/s on 148 SMs
FP32_LANES_PER_SM = 128
MAX_SM_GHZ = 1.965


def bench_router_prefill(torch, moe, args):
    """Router projection + grouped top-k at the prefill shape, T=8192 (the
    tiled FP32 projection).  Calls alternate between two hidden batches (134 MB
    together, > L2) and four layers' routers."""
    wl = inputs.WORKLOADS["prefill"]
    T, H, E = wl.T, wl.H, wl.E
    rng = np.random.default_rng(wl.seed + 101)
    xs = [torch.from_numpy(inputs.bf16_bits(rng.standard_normal((T, H), dtype=np.float32)).view(np.int16)).cuda()
          for _ in range(2)]
    w = torch.empty((4, E, H), dtype=torch.float32, device="cuda")
    for l in range(4):
        w[l].copy_(torch.from_numpy(inputs.router_weights(rng, E, H)))
    logits = torch.empty((T, E), dtype=torch.float32, device="cuda")
    ids = torch.empty((T, wl.top_k), dtype=torch.int32, device="cuda")
    wts = torch.empty((T, wl.top_k), dtype=torch.float32, device="cuda")
    ws = torch.zeros(max(16, moe.moe_router_topk_workspace_size(T)), dtype=torch.uint8, device="cuda")

    def call(i):
        moe.moe_router_topk(xs[i % 2], w[i % 4], None, wl.n_group, wl.topk_group, wl.top_k, wl.rsf, True, logits,
                            ids, wts, ws)

    for i in range(max(args.warmup, 3)):
        call(i)
    torch.cuda.synchronize()
    reps = max(args.steps, 20)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(reps):
        call(i)
    b.record()
    torch.cuda.synchronize()
    moe.nvfp4moe_check_device_status()
    us = a.elapsed_time(b) / reps * 1e3
    flops = 2.0 * T * H * E
    tf = flops / (us / 1e6) / 1e12
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    peak = sms * FP32_LANES_PER_SM * 2 * MAX_SM_GHZ / 1e3
    del xs, w
    torch.cuda.empty_cache()
    return {"workload": f"router: T={T} H={H} E={E} groups={wl.n_group} keep={wl.topk_group} top_k={wl.top_k}, "
                        "FP32 router, two hidden batches x four routers rotated (> L2)",
            "value": round(us, 2), "unit": "us per call (projection + routing)", "higher_is_better": False,
            "roofline": {"bound": "alu", "kernel": "k_router_logits_tiled + k_route_rows", "achieved": round(tf, 2),
                         "peak": round(peak, 1), "unit": "TFLOP/s", "frac": round(tf / peak, 4), "traffic": None,
                         "peak_src": f"derived: {sms} SMs x {FP32_LANES_PER_SM} FP32 lanes x 2 FLOP x "
                                     f"{MAX_SM_GHZ} GHz",
                         "algorithmic_flops_per_call": int(flops)}}


def bench_transcode(torch, moe, args, P):
    """MXFP4 -> NVFP4 transcode of one layer (3 x E expert tensors, E = 256: 768), out of place."""
    rng = np.random.default_rng(inputs.TRANSCODE_SEED)
    E = args.transcode_experts
    layer = inputs.transcode_layer(rng, E=E)
    codes = np.concatenate([layer["gate"][0], layer["up"][0], layer["down"][0].reshape(E, 2048, 2048)])
    e8 = np.concatenate([layer["gate"][1], layer["up"][1], layer["down"][1].reshape(E, 2048, 128)])
    nt, N, K = codes.shape[0], 2048, 4096  # the down tensors [4096, 2048] have the same block count
    c = torch.from_numpy(codes).cuda()
    s = torch.from_numpy(e8).cuda()
    del codes, e8, layer
    co = torch.empty_like(c)
    e4 = torch.empty((nt, N, K // 16), dtype=torch.uint8, device="cuda")
    g = torch.empty(nt, dtype=torch.float32, device="cuda")
    st = torch.empty(nt, dtype=torch.int32, device="cuda")
    ws = torch.empty(moe.nvfp4moe_transcode_workspace_size(nt), dtype=torch.uint8, device="cuda")
    status, rep = moe.transcode_mxfp4_to_nvfp4(c, s, nt, N, K, co, e4, g, st, ws, report=True)
    for _ in range(args.warmup):
        moe.transcode_mxfp4_to_nvfp4(c, s, nt, N, K, co, e4, g, st, ws, report=False)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    steps = max(args.steps, 10)
    a.record()
    for _ in range(steps):
        moe.transcode_mxfp4_to_nvfp4(c, s, nt, N, K, co, e4, g, st, ws, report=False)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    nbytes = c.numel() * 2 + s.numel() + e4.numel()  # read codes + e8m0, write codes + e4m3
    gbs = nbytes / (ms / 1e3) / 1e9
    res = {"workload": f"transcode: {nt} MXFP4 expert tensors ({E} experts x gate/up [2048,4096], down [4096,2048]), "
                       "out of place", "value": round(gbs, 1), "unit": "GB/s", "ms_per_step": round(ms, 4),
           "tensors_per_s": round(nt / (ms / 1e3), 1), "status": int(status), "report": rep,
           "roofline": {"bound": "hbm", "kernel": "k_transcode", "achieved": round(gbs, 1), "peak": P["hbm_gbs"],
                        "unit": "GB/s", "frac": round(gbs / P["hbm_gbs"], 4),
                        "traffic": TRANSCODE_TRAFFIC_768 if nt == 768 else None,
                        "traffic_unit": "bytes per launch (ncu dram read+write)",
                        "frac_of_spec": round(gbs / SPEC_HBM_GBS, 4),
                        "algorithmic_bytes_per_launch": int(nbytes)}}
    # in place (codes aliased): scales only
    a.record()
    for _ in range(steps):
        moe.transcode_mxfp4_to_nvfp4(c, s, nt, N, K, c, e4, g, st, ws, report=False)
    b.record()
    torch.cuda.synchronize()
    ms2 = a.elapsed_time(b) / steps
    nb2 = c.numel() + s.numel() + e4.numel()
    res["in_place"] = {"ms": round(ms2, 4), "GB/s": round(nb2 / (ms2 / 1e3) / 1e9, 1)}
    del c, s, co, e4
    torch.cuda.empty_cache()
    return res


def cpu_baseline(wl, d, args, steps=1, per_thread=4):
    """The oracle as it stands, on a bounded token sample of the same workload:
    per_thread tokens for each host thread (4: ~10 s of oracle work)."""
    import oracle

    threads = oracle.num_threads()
    n = args.cpu_sample_tokens or per_thread * threads
    toks = np.arange(n, dtype=np.int32)
    w = {k: d[k] for k in ("gate_codes", "gate_sf", "up_codes", "up_sf", "down_codes", "down_sf", "w_global")}
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle.moe_layer(wl.mode, d["x"], d["logits"], None, w["gate_codes"], w["gate_sf"], w["up_codes"], w["up_sf"],
                         w["down_codes"], w["down_sf"], w["w_global"], 1.0, wl.n_group, wl.topk_group, wl.top_k,
                         wl.rsf, True, toks)
    dt = (time.perf_counter() - t0) / steps
    return {"value": round(n / dt, 3), "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} tokens of the {wl.name} workload per step (float64 C oracle, OpenMP over tokens)",
            "seconds_per_step": round(dt, 3)}


def run_reference(args, rank, world):
    if rank != 0:
        return
    wl = workload(args)
    d = inputs.moe_inputs(wl)
    import oracle

    oracle.build()
    # exactly W warm-up and K timed steps; past 6 steps in all each step samples
    # one token per host thread (a few seconds), so the run stays within minutes
    per_thread = 4 if args.warmup + args.steps <= 6 else 1
    for _ in range(args.warmup):
        cpu_baseline(wl, d, args, per_thread=per_thread)
    vals = [cpu_baseline(wl, d, args, per_thread=per_thread) for _ in range(max(1, args.steps))]
    v = float(np.mean([r["value"] for r in vals]))
    dt = float(np.mean([r["seconds_per_step"] for r in vals]))
    out = {"impl": "reference", "metric": "MoE-layer tokens/s", "value": round(v, 3), "unit": "tokens/s",
           "n_gpus": world, "steps": len(vals), "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 1),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": config_of(wl, wl.T, world),
           "cpu_baseline": {"value": round(v, 3), "unit": "tokens/s", "kind": "oracle", "cores": vals[0]["cores"],
                            "sample": vals[0]["sample"]},
           "e2e": {"value": round(v, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus)))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if "WORLD_SIZE" not in os.environ:
        world = 1  # without torchrun there is one process
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
