#!/usr/bin/env python
"""Throughput of VDA forward (both scan directions + gated readout) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]

One step = one whole VDA forward (Gram, factor-and-solve, bidirectional scan,
readout) over one 768p full-clip problem: B=1, H=32, T=45 frames, n=1008
tokens (24 x 42), d_k=d_v=128, 256 text tokens, bfloat16, lambda=1, seeded
synthetic inputs resident in HBM.  Metric: (frame, head) units per second.

N > 1 (torchrun, one process per GPU): every rank runs its own problem (heads
and batches are independent, so there is no data-path collective); the value
is the units of all ranks over the max-over-ranks device time (weak scaling).

The number comes from K calls of vda_forward timed with CUDA events on the
launching stream.  A second timed region of K vda_forward_timed calls gives
each kernel's time (CUDA events between the kernels, on the same stream);
the JSON line carries the roofline of the dominant kernel from those times,
the path's roofline fraction, an end-to-end figure through the host-buffer
entry point,
clocks sampled during the timed region, and (rank 0, N=1) the float64 CPU
oracle timed on a bounded sample of the same workload.
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

METRIC = "VDA frames*heads/sec (fwd+bwd) at 768p shape; % of B200 roofline"
UNIT = "frames*heads/s"
WORKLOAD = "768p"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
# FP32 SIMT peak from unit counts and clock: 148 SMs x 128 FMA/clk x 2 flop x 1.965 GHz.
FP32_SIMT_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12

# Kernel of each reported stage and the source file that defines it (for ncu
# traffic lookups), by input dtype.  With bf16 inputs the Gram and the factor
# are one kernel.
STAGE_SOURCES = {
    1: {"gram+factor": "frame_wise_linear_b200/csrc/vda_gramfactor_tc.cu",
        "scan": "frame_wise_linear_b200/csrc/vda_scan_tc.cu",
        "readout": "frame_wise_linear_b200/csrc/vda_readout_tc.cu"},
    2: {"gram+factor": "frame_wise_linear_b200/csrc/vda_gramfactor_tc.cu",
        "scan": "frame_wise_linear_b200/csrc/vda_scan_tc.cu",
        "readout": "frame_wise_linear_b200/csrc/vda_readout_tc.cu"},
    0: {"gram": "frame_wise_linear_b200/csrc/vda_simt.cu",
        "factor": "frame_wise_linear_b200/csrc/vda_factor.cu",
        "scan": "frame_wise_linear_b200/csrc/vda_simt.cu",
        "readout": "frame_wise_linear_b200/csrc/vda_simt.cu"},
}


def parse():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("b200", "reference"), default="b200")
    ap.add_argument("--workload", default=WORKLOAD, help="a name from frame_wise_linear_b200.synth.WORKLOADS")
    ap.add_argument("--e2e-steps", type=int, default=None, help="steps of the end-to-end leg (default min(K, 10))")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="CPU oracle sample budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layout", choices=("bhtnd", "btnhd"), default="bhtnd",
                    help="token tensors as [B, H, T, n, d] (default) or token-major [B, T*n, H, d]")
    ap.add_argument("--direction", choices=("forward", "backward", "merge", "softmax"), default="forward",
                    help="backward: time vda_backward (the gradients); merge: time vda_merge_project (both "
                         "branches' output projections, summed); softmax: time vda_local_softmax (the local "
                         "softmax branch); separate lines, not the headline")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# Work counts: algorithmic bytes / flops per launch.
# ---------------------------------------------------------------------------

def elem_bytes(w):
    """Bytes of one input element and of one element of O (bf16 O for 8-bit inputs)."""
    return {0: (4, 4), 1: (2, 2), 2: (1, 2)}[w.dtype]


DTYPE_NAMES = {0: "f32", 1: "bf16", 2: "e4m3"}


def stage_work(w):
    es, eo = elem_bytes(w)
    bh = w.B * w.H
    frames = bh * w.T
    slots = bh * (w.T + 1)
    d_k, d_v = w.d_k, w.d_v
    gram = dict(bound="hbm", bytes=(frames * w.n + bh * w.n_txt) * (d_k + d_v) * es,
                flops=2.0 * (frames * w.n + bh * w.n_txt) * d_k * (d_k + d_v))
    return {
        # reads K_t, V_t of every frame and the text once
        "gram": gram,
        # the same, with the factor in the same kernel (no algorithmic bytes of its own)
        "gram+factor": dict(bound="hbm", bytes=gram["bytes"], flops=gram["flops"] + slots * float(d_k) ** 3),
        # lambda A^{-1} by the symmetric sweep: d^3/2 FMA = d^3 flops per slot
        "factor": dict(bound="alu", bytes=0, flops=slots * float(d_k) ** 3),
        # two directions, one d_k x d_k by d_k x d_v product per frame
        "scan": dict(bound="alu", bytes=0, flops=2.0 * frames * 2.0 * d_k * d_k * d_v),
        # reads Q_t, G_t, writes O_t
        "readout": dict(bound="hbm", bytes=frames * w.n * ((d_k + d_v) * es + d_v * eo),
                        flops=2.0 * frames * w.n * d_k * d_v),
    }


def path_roofline(w, peaks):
    es, eo = elem_bytes(w)
    bh = w.B * w.H
    frames = bh * w.T
    nbytes = frames * w.n * ((2 * w.d_k + 2 * w.d_v) * es + w.d_v * eo) + bh * w.n_txt * (w.d_k + w.d_v) * es
    flops = 2.0 * frames * w.n * (w.d_k * (w.d_k + w.d_v) + w.d_k * w.d_v) \
        + 2.0 * bh * w.n_txt * w.d_k * (w.d_k + w.d_v)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    return dict(bytes=nbytes, tensor_flops=flops, t_roof_s=max(t_hbm, t_tc),
                bound="hbm" if t_hbm >= t_tc else "tensor")


# The other lines' kernels (bf16 only).
KERNEL_SOURCES = {"merge": "frame_wise_linear_b200/csrc/vda_merge_tc.cu",
                  "softmax": "frame_wise_linear_b200/csrc/vda_local_softmax_tc.cu"}


def traffic_lookup(stage, w):
    """DRAM bytes per launch of a stage's kernel on workload `w`, from the committed ncu summary,
    if the kernel's source is unchanged since the capture."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    srcs = dict(STAGE_SOURCES[w.dtype], **KERNEL_SOURCES)
    if not os.path.exists(path) or stage not in srcs:
        return None
    src = os.path.join(ROOT, srcs[stage])
    digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    with open(path) as fh:
        for line in fh:
            p = line.split()
            if len(p) >= 4 and not line.startswith("#") and p[0] == stage and p[1] == w.name and p[2] == digest:
                return float(p[3])
    return None


# ---------------------------------------------------------------------------
# Clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def start(self):
        import tempfile
        try:
            fd, self.path = tempfile.mkstemp(prefix="vda_clocks_", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.6)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"unavailable": "nvidia-smi could not be started"}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as fh:
            for line in fh:
                p = [x.strip() for x in line.split(",")]
                if len(p) < 9:
                    continue
                if self.uuid and p[0] != self.uuid:
                    continue
                rows.append(p)
        os.unlink(self.path)
        if not rows:
            return {"unavailable": "no nvidia-smi samples for this GPU"}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# CPU oracle timing (bounded sample)
# ---------------------------------------------------------------------------

def cpu_threads():
    """Threads the CPU legs give the oracle's BLAS: every host core."""
    return os.cpu_count() or 1


def cpu_model():
    """The host CPU's model name (from /proc/cpuinfo), for the CPU legs' lines."""
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def blas_limits():
    """Fixes the BLAS thread count for the oracle's timing (both CPU legs use the same)."""
    from threadpoolctl import threadpool_limits
    return threadpool_limits(limits=cpu_threads(), user_api="blas")


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return cpu_threads()


def cpu_sample_inputs(w, frames=None):
    """The CPU legs' sample: head (0, 0) of the workload, its first `frames` frames (all by default)."""
    from frame_wise_linear_b200 import synth
    x = synth.head_widened(w, 0, 0, seed=0)
    T = w.T if frames is None else max(1, min(w.T, frames))
    return [x["Q"][:T], x["K"][:T], x["V"][:T], x["G"][:T], x["K_txt"], x["V_txt"], w.lam], T


def cpu_oracle_sample(w, budget_s):
    """Times the float64 oracle on the CPU sample, repeated until the budget is used.

    Returns (frames*heads per second, threads, description).  The same sample
    and thread count as the reference arm's steps; input generation and
    widening are outside the timed part.
    """
    from oracle import vda_oracle as vo
    args, T = cpu_sample_inputs(w)
    with blas_limits():
        vo.vda_head(*args)           # warm-up (BLAS thread pool start-up)
        spent, reps = 0.0, 0
        while spent < budget_s:
            t0 = time.perf_counter()
            vo.vda_head(*args)
            spent += time.perf_counter() - t0
            reps += 1
        threads = blas_threads()
    desc = (f"head (0,0), frames 1..{T} of the {w.name} workload, repeated {reps} times "
            f"(float64 oracle, {threads} BLAS threads)")
    return reps * T / spent, threads, desc


# ---------------------------------------------------------------------------
# Arms
# ---------------------------------------------------------------------------

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def run_reference(args, w):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    from oracle import vda_oracle as vo
    # Each step is the CPU sample (head (0,0), all frames), cut to fewer
    # frames only if the whole run would take more than about two minutes.
    with blas_limits():
        args2, _ = cpu_sample_inputs(w, 2)
        vo.vda_head(*args2)
        t0 = time.perf_counter()
        vo.vda_head(*args2)
        per_frame = (time.perf_counter() - t0) / 2
        budget = 120.0 / max(args.steps + args.warmup, 1)
        args_h, frames = cpu_sample_inputs(w, int(max(1, budget / max(per_frame, 1e-6))))
        for _ in range(args.warmup):
            vo.vda_head(*args_h)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            vo.vda_head(*args_h)
        dt = time.perf_counter() - t0
        threads = blas_threads()
    value = args.steps * frames / dt
    sample = (f"each step: head (0,0), frames 1..{frames} of the {w.name} workload "
              f"(float64 oracle, {threads} BLAS threads)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample, "cpu": cpu_model()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


L2_BYTES = 126e6
LAYOUTS = {"bhtnd": 0, "btnhd": 1}
LAYOUT_NAMES = {0: "[B,H,T,n,d]", 1: "[B,T*n,H,d]"}


def config_of(w, n, layout=0):
    return {"workload": f"{w.name}: B={w.B} H={w.H} T={w.T} n={w.n} d_k={w.d_k} d_v={w.d_v} "
                        f"n_txt={w.n_txt} lambda={w.lam} {DTYPE_NAMES[w.dtype]}"
                        + (" (per-tensor scales, bf16 O)" if w.dtype == 2 else ""),
            "B": w.B, "H": w.H, "T": w.T, "n": w.n, "n_txt": w.n_txt, "d": w.d_k,
            "layout": LAYOUT_NAMES[layout],
            "parallelism": f"independent problems on {n} GPU(s), no collective",
            "l2": (f"inputs larger than L2 ({input_bytes(w) / 1e9:.2f} GB read per step vs 126 MB); no flush"
                   if input_bytes(w) > L2_BYTES else
                   f"inputs smaller than L2 ({input_bytes(w) / 1e6:.1f} MB vs 126 MB), not flushed: "
                   "a latency-bound workload, not the headline")}


def max_over_ranks(ms, dist, device):
    """The job's device time: the slowest rank's (ms on every rank afterwards)."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([float(ms)], device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(units_per_rank, n_ranks, ms_per_step):
    """Whole-job throughput: every rank's units over the job's time per step."""
    return n_ranks * units_per_rank / (ms_per_step / 1e3)


def input_bytes(w):
    es = elem_bytes(w)[0]
    return (w.B * w.H * (w.T * w.n * 2 * (w.d_k + w.d_v) + w.n_txt * (w.d_k + w.d_v))) * es


def run_b200(args, w):
    import torch
    from frame_wise_linear_b200 import build as _build
    from frame_wise_linear_b200 import synth, vda

    ws_n, rank, local = dist_env()
    if args.gpus != ws_n:
        if ws_n == 1 and args.gpus > 1:
            raise SystemExit("--gpus N > 1 needs torchrun (one process per GPU)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if ws_n > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist
    _build.build()
    vda.load()

    peaks, peaks_kind = load_peaks()
    layout = LAYOUTS[args.layout]
    d = synth.make_inputs_torch(w, seed=rank, device=dev)
    if layout:
        d = {k: synth.token_major(v) for k, v in d.items()}
    prob = vda.make_problem(**w.problem(), layout=layout)
    wsb = vda.vda_workspace_size(prob)
    wsp = torch.empty(wsb, dtype=torch.uint8, device=dev)
    O = torch.empty(d["G"].shape, dtype=torch.float32 if w.dtype == 0 else torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    kt = d["K_txt"] if w.n_txt else None
    vt = d["V_txt"] if w.n_txt else None

    def step(events=None):
        if events is None:
            vda.vda_forward(prob, d["Q"], d["K"], d["V"], d["G"], kt, vt, O, wsp, stream=stream)
        else:
            vda.vda_forward_timed(prob, d["Q"], d["K"], d["V"], d["G"], kt, vt, O, wsp, events, stream=stream)

    for _ in range(max(args.warmup, 3)):
        step()
    vda.vda_sync_status(wsp, stream=stream)

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    sampler.start()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(vda.VDA_TIMED_EVENTS)]
          for _ in range(args.steps)]
    for e_step in ev:          # torch creates the CUDA event on its first record
        for e in e_step:
            e.record(stream)
    torch.cuda.synchronize(dev)

    def timed_region(events):
        """K steps between a barrier + synchronize on both sides; device ms."""
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        if pg:
            pg.barrier()
        torch.cuda.synchronize(dev)
        start.record(stream)
        for k in range(args.steps):
            step(events[k] if events else None)
        end.record(stream)
        torch.cuda.synchronize(dev)
        if pg:
            pg.barrier()
        return start.elapsed_time(end)

    # Region 1, the number: K calls of vda_forward as a user makes them.
    # Region 2, the stage times: K calls of vda_forward_timed, whose events
    # between the kernels also stop the next kernel from starting early
    # (programmatic dependent launch), so it runs a little slower.
    ms = timed_region(None)
    ms_instrumented = timed_region(ev)
    clocks = sampler.stop()
    vda.vda_sync_status(wsp, stream=stream)
    stage_ms = {s: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in ev) for i, s in enumerate(vda.STAGES)}
    if w.dtype != 0:   # one kernel for the Gram and the factor: report them as one stage
        stage_ms = {"gram+factor": stage_ms["gram"] + stage_ms["factor"], "scan": stage_ms["scan"],
                    "readout": stage_ms["readout"]}
    ms = max_over_ranks(ms, pg, dev)
    ms_step = ms / args.steps
    value = job_value(w.units, ws_n, ms_step)

    # dominant kernel roofline
    work = stage_work(w)
    dom = max(stage_ms, key=stage_ms.get)
    wk = work[dom]
    t_s = stage_ms[dom] / 1e3
    if wk["bound"] == "hbm":
        roof = {"kernel": dom, "bound": "hbm", "achieved": wk["bytes"] / t_s / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "peak_source": f"{peaks_kind} (MEASURED_PEAKS.json hbm_gbs)"}
    else:
        roof = {"kernel": dom, "bound": "alu", "achieved": wk["flops"] / t_s / 1e12, "peak": FP32_SIMT_TFLOPS,
                "unit": "TFLOP/s", "peak_source": "derived: 148 SMs x 128 FP32 FMA/clk x 2 x 1.965 GHz"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    tr = traffic_lookup(dom, w)
    roof["traffic"] = tr
    pr = path_roofline(w, peaks)
    path = {"t_roof_us": pr["t_roof_s"] * 1e6, "bound": pr["bound"], "bytes": pr["bytes"],
            "frac": pr["t_roof_s"] / (ms_step / 1e3), "stage_ms": stage_ms,
            "stage_timing": "a second timed region of K vda_forward_timed calls (CUDA events between the "
                            "kernels), %.4f ms per step" % (max_over_ranks(ms_instrumented, pg, dev) / args.steps)}

    # The training direction beside the headline (bf16 only): the backward on the state one forward
    # left in a backward-sized workspace, and forward + backward steps, K each, CUDA events on the stream.
    path["backward"] = backward_extras(args, w, d, prob, kt, vt, stream, dev, pg) if w.dtype == 1 else None

    # end-to-end through host buffers (pinned), copies inside the timed region
    e2e_steps = args.e2e_steps if args.e2e_steps is not None else min(args.steps, 10)
    if e2e_steps <= 0:
        return finish(args, w, ws_n, rank, pg, value, ms_step, roof, path, None, clocks)
    host = {k: v.cpu().pin_memory() for k, v in d.items()}
    Oh = torch.empty(O.shape, dtype=O.dtype).pin_memory()
    del d
    wsh = torch.empty(vda.vda_host_workspace_size(prob), dtype=torch.uint8, device=dev)
    hkt = host["K_txt"] if w.n_txt else None
    hvt = host["V_txt"] if w.n_txt else None
    vda.vda_forward_host(prob, host["Q"], host["K"], host["V"], host["G"], hkt, hvt, Oh, wsh, stream=stream)
    if pg:
        pg.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(e2e_steps):
        vda.vda_forward_host(prob, host["Q"], host["K"], host["V"], host["G"], hkt, hvt, Oh, wsh, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, pg, dev)
    h2d = sum(v.numel() * v.element_size() for k, v in host.items() if (w.n_txt or k not in ("K_txt", "V_txt")))
    d2h = Oh.numel() * Oh.element_size()
    e2e = {"value": job_value(w.units, ws_n, e2e_ms / e2e_steps), "unit": UNIT, "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "steps": e2e_steps,
           "api": "vda_forward_host (C ABI, pinned host buffers)"}
    return finish(args, w, ws_n, rank, pg, value, ms_step, roof, path, e2e, clocks)


def backward_extras(args, w, d, prob, kt, vt, stream, dev, pg):
    """ms per vda_backward_from_forward call after one vda_forward, and per training step (vda_forward +
    vda_backward_from_forward), over K calls each (max over ranks); the backward's roofline fraction."""
    import torch
    from frame_wise_linear_b200 import synth, vda
    rank = dist_env()[1]
    dO = synth.grad_out_torch(w, seed=rank, device=dev)
    if prob.layout:
        dO = synth.token_major(dO)
    wsb = torch.empty(vda.vda_backward_workspace_size(prob), dtype=torch.uint8, device=dev)
    outs = [torch.empty_like(d[k]) for k in ("Q", "K", "V", "G")]
    touts = [torch.empty_like(d["K_txt"]), torch.empty_like(d["V_txt"])] if w.n_txt else [None, None]
    O2 = torch.empty_like(d["G"])
    ins = (prob, d["Q"], d["K"], d["V"], d["G"], kt, vt)

    def fwd():
        vda.vda_forward(*ins, O2, wsb, stream=stream)

    def bwd():
        vda.vda_backward_from_forward(*ins, dO, *outs, *touts, wsb, stream=stream)

    def timed(fn):
        for _ in range(max(args.warmup, 3)):
            fn()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        if pg:
            pg.barrier()
        torch.cuda.synchronize(dev)
        a.record(stream)
        for _ in range(args.steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return max_over_ranks(a.elapsed_time(b) / args.steps, pg, dev)

    fwd()
    ms_bwd = timed(bwd)

    def train():
        fwd()
        bwd()

    ms_train = timed(train)
    vda.vda_sync_status(wsb, stream=stream)
    peaks, _ = load_peaks()
    rf = backward_roofline(w, peaks)
    del wsb, outs, touts, dO, O2
    torch.cuda.empty_cache()
    return {"from_forward_ms": ms_bwd, "from_forward_frac": rf["t_roof_s"] / (ms_bwd / 1e3),
            "train_step_ms": ms_train,
            "train_step_value": job_value(w.units, dist_env()[0], ms_train),
            "calls": "vda_backward_from_forward after one vda_forward; train step = vda_forward + "
                     "vda_backward_from_forward; K calls each, CUDA events on the launching stream"}


def finish(args, w, ws_n, rank, pg, value, ms_step, roof, path, e2e, clocks):
    from frame_wise_linear_b200 import vda
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws_n, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": DTYPE_NAMES[w.dtype], "data": "synthetic",
        "config": config_of(w, ws_n, LAYOUTS[args.layout]), "roofline": roof, "roofline_path": path, "e2e": e2e,
        "clocks": clocks, "gpu_launches": vda.LAUNCHES_PER_FORWARD[w.dtype] * args.steps,
    }
    bwd = path.pop("backward", None) if isinstance(path, dict) else None
    if bwd is not None:
        line["backward"] = bwd
    if rank == 0 and ws_n == 1 and not args.no_cpu_baseline:
        v, threads, desc = cpu_oracle_sample(w, args.cpu_seconds)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": desc, "cpu": cpu_model()}
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


BWD_METRIC = "VDA backward frames*heads/sec (gradients of Q, K, V, G and the text) at 768p shape; % of B200 roofline"


def backward_roofline(w, peaks):
    """Algorithmic work of one backward: Q, K, V, G, dO read; dQ, dK, dV, dG written (and the text's);
    tensor flops of the Gram, P = Q S, dQ, E and the two products of dK and one of dV per token."""
    es = 2 if w.dtype == 1 else 4
    bh = w.B * w.H
    frames = bh * w.T
    tok = frames * w.n
    # per token: Q, K, dQ, dK (d_k each); V, G, dO, dV, dG (d_v each); the text: K_txt, V_txt, dK_txt, dV_txt
    nbytes = tok * (4 * w.d_k + 5 * w.d_v) * es + bh * w.n_txt * 2 * (w.d_k + w.d_v) * es
    flops = 2.0 * tok * w.d_k * (w.d_k + w.d_v) + 2.0 * tok * 3 * w.d_k * w.d_v + 2.0 * tok * w.d_k * (w.d_k + 2 * w.d_v)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    return dict(bytes=nbytes, tensor_flops=flops, t_roof_s=max(t_hbm, t_tc), bound="hbm" if t_hbm >= t_tc else "tensor")


def run_backward(args, w):
    """K timed vda_backward calls on one GPU: whole-call throughput and its roofline."""
    import torch
    from frame_wise_linear_b200 import build as _build
    from frame_wise_linear_b200 import synth, vda
    if args.gpus != 1:
        raise SystemExit("--direction backward runs on one GPU")
    dev = torch.device("cuda", 0)
    _build.build()
    vda.load()
    peaks, peaks_kind = load_peaks()
    layout = LAYOUTS[args.layout]
    d = synth.make_inputs_torch(w, seed=0, device=dev)
    dO = synth.grad_out_torch(w, seed=0, device=dev)
    if layout:
        d = {k: synth.token_major(v) for k, v in d.items()}
        dO = synth.token_major(dO)
    prob = vda.make_problem(**w.problem(), layout=layout)
    wsp = torch.empty(vda.vda_backward_workspace_size(prob), dtype=torch.uint8, device=dev)
    txt = w.n_txt > 0
    outs = [torch.empty_like(d[k]) for k in ("Q", "K", "V", "G")]
    touts = [torch.empty_like(d["K_txt"]), torch.empty_like(d["V_txt"])] if txt else [None, None]
    stream = torch.cuda.current_stream(dev)

    ins = (prob, d["Q"], d["K"], d["V"], d["G"], d["K_txt"] if txt else None, d["V_txt"] if txt else None)
    O = torch.empty_like(d["G"])

    def step():
        vda.vda_backward(*ins, dO, *outs, *touts, wsp, stream=stream)

    def fwd():
        vda.vda_forward(*ins, O, wsp, stream=stream)

    def step_ff():
        vda.vda_backward_from_forward(*ins, dO, *outs, *touts, wsp, stream=stream)

    def timed(fn, k):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        a.record(stream)
        for _ in range(k):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / k

    for _ in range(max(args.warmup, 3)):
        step()
    vda.vda_sync_status(wsp, stream=stream)
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    sampler.start()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    start.record(stream)
    for _ in range(args.steps):
        step()
    end.record(stream)
    torch.cuda.synchronize(dev)
    ms_step = start.elapsed_time(end) / args.steps
    # The backward on the state a forward call left in the workspace (a
    # training step's form), and the whole forward + backward step.
    fwd()
    for _ in range(max(args.warmup, 3)):
        step_ff()
    ms_ff = timed(step_ff, args.steps)

    def train():
        fwd()
        step_ff()

    for _ in range(max(args.warmup, 3)):
        train()
    ms_train = timed(train, args.steps)
    clocks = sampler.stop()
    vda.vda_sync_status(wsp, stream=stream)
    rf = backward_roofline(w, peaks)
    line = {
        "metric": BWD_METRIC, "direction": "backward", "value": job_value(w.units, 1, ms_step), "unit": UNIT,
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == 1 else "f32", "data": "synthetic",
        "config": config_of(w, 1, LAYOUTS[args.layout]),
        "roofline": {"kernel": "whole vda_backward call", "bound": rf["bound"],
                     "achieved": rf["bytes"] / (ms_step / 1e3) / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "peak_source": f"{peaks_kind} (MEASURED_PEAKS.json hbm_gbs)",
                     "frac": rf["t_roof_s"] / (ms_step / 1e3), "traffic": None},
        "roofline_path": {"t_roof_us": rf["t_roof_s"] * 1e6, "bound": rf["bound"], "bytes": rf["bytes"],
                          "frac": rf["t_roof_s"] / (ms_step / 1e3)},
        "from_forward": {"call": "vda_backward_from_forward after vda_forward (no recompute)", "ms_per_call": ms_ff,
                         "value": job_value(w.units, 1, ms_ff), "frac": rf["t_roof_s"] / (ms_ff / 1e3)},
        "train_step": {"calls": "vda_forward + vda_backward_from_forward", "ms_per_step": ms_train,
                       "value": job_value(w.units, 1, ms_train)},
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


MERGE_METRIC = "branch merge (output projections of both branches, summed) tokens/sec at 768p shape; % of B200 bf16 peak"


def run_merge(args, w):
    """K timed vda_merge_project calls on one GPU: Y = O_lin W_lin + O_sm W_sm over the workload's tokens,
    K = H * d_v features per branch, D = H * d_v outputs (the attention block's width)."""
    import torch
    from frame_wise_linear_b200 import build as _build
    from frame_wise_linear_b200 import vda
    if args.gpus != 1:
        raise SystemExit("--direction merge runs on one GPU")
    dev = torch.device("cuda", 0)
    _build.build()
    vda.load()
    peaks, peaks_kind = load_peaks()
    tokens, K = w.B * w.T * w.n, w.H * w.d_v
    D = K
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    O = torch.randn(tokens, K, device=dev, generator=g).to(torch.bfloat16)
    P = torch.randn(tokens, K, device=dev, generator=g).to(torch.bfloat16)
    Wl = (torch.randn(K, D, device=dev, generator=g) / K ** 0.5).to(torch.bfloat16)
    Ws = (torch.randn(K, D, device=dev, generator=g) / K ** 0.5).to(torch.bfloat16)
    Y = torch.empty(tokens, D, device=dev, dtype=torch.bfloat16)
    ws = torch.empty(256, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        vda.vda_merge_project(tokens, K, D, O, Wl, P, Ws, Y, ws, stream=stream)

    for _ in range(max(args.warmup, 3)):
        step()
    vda.vda_sync_status(ws, stream=stream)
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    sampler.start()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    a.record(stream)
    for _ in range(args.steps):
        step()
    b.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    vda.vda_sync_status(ws, stream=stream)
    ms = a.elapsed_time(b) / args.steps
    flops = 2.0 * tokens * (2 * K) * D
    bytes_ = 2 * (2 * tokens * K + 2 * K * D + tokens * D)
    tf = flops / (ms / 1e3) / 1e12
    line = {
        "metric": MERGE_METRIC, "direction": "merge", "value": tokens / (ms / 1e3), "unit": "tokens/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{w.name} tokens ({w.B}x{w.T}x{w.n}), K = D = {K}, two branches, bf16",
                   "tokens": tokens, "K": K, "D": D, "l2": "inputs larger than L2; no flush"},
        "roofline": {"kernel": "merge_tc_kernel", "bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": tf / peaks["bf16_tflops"],
                     "peak_source": f"{peaks_kind} (MEASURED_PEAKS.json bf16_tflops)",
                     "traffic": traffic_lookup("merge", w), "algorithmic_bytes": bytes_},
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


SOFTMAX_METRIC = "local softmax branch frames*heads/sec at 768p shape; % of B200 bf16 peak"


def softmax_work(w):
    """Tensor flops of the local softmax branch over the workload: per (b, h, t) query frame, Q K^T and P V over
    its keys (the tokens of its key frames and the text): 4 n keys d."""
    def key_frame_count(t, T, block=5):   # the window's frames and the anchors 0 and T - 1
        b = t // block
        lo, hi = max(0, (b - 1) * block), min(T, (b + 2) * block)
        return (hi - lo) + (lo > 0) + (hi < T)
    keys = sum(w.n * key_frame_count(t, w.T) + w.n_txt for t in range(w.T))
    return 4.0 * w.B * w.H * w.n * keys * w.d_k


def run_softmax(args, w):
    """K timed vda_local_softmax calls on one GPU over the workload's shapes (the branch's own Q, K, V, G)."""
    import torch
    from frame_wise_linear_b200 import build as _build
    from frame_wise_linear_b200 import synth, vda
    if args.gpus != 1:
        raise SystemExit("--direction softmax runs on one GPU")
    dev = torch.device("cuda", 0)
    _build.build()
    vda.load()
    peaks, peaks_kind = load_peaks()
    d = synth.make_inputs_torch(w, seed=0, device=dev)
    prob = vda.make_problem(**w.problem())
    O = torch.empty_like(d["G"])
    ws = torch.empty(256, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    kt, vt = (d["K_txt"], d["V_txt"]) if w.n_txt else (None, None)

    def step():
        vda.vda_local_softmax(prob, d["Q"], d["K"], d["V"], d["G"], kt, vt, O, ws, stream=stream)

    for _ in range(max(args.warmup, 3)):
        step()
    vda.vda_sync_status(ws, stream=stream)
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    sampler.start()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    a.record(stream)
    for _ in range(args.steps):
        step()
    b.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    vda.vda_sync_status(ws, stream=stream)
    ms = a.elapsed_time(b) / args.steps
    tf = softmax_work(w) / (ms / 1e3) / 1e12
    line = {
        "metric": SOFTMAX_METRIC, "direction": "softmax", "value": job_value(w.units, 1, ms), "unit": UNIT,
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_of(w, 1),
        "roofline": {"kernel": "local_softmax_tc_kernel", "bound": "tensor", "achieved": tf,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": tf / peaks["bf16_tflops"],
                     "peak_source": f"{peaks_kind} (MEASURED_PEAKS.json bf16_tflops)",
                     "traffic": traffic_lookup("softmax", w), "flops": softmax_work(w)},
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    from frame_wise_linear_b200 import synth
    w = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if args.direction == "backward":
        return run_backward(args, w)
    if args.direction == "merge":
        return run_merge(args, w)
    if args.direction == "softmax":
        return run_softmax(args, w)
    return run_b200(args, w)


if __name__ == "__main__":
    sys.exit(main())
