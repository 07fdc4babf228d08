#!/usr/bin/env python
"""Benchmark of the Windowed-MTP decode step on B200: microseconds per decode step and KV-read
GB/s against the measured HBM peak, windowed vs native full-context draft, at 1M context.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload ctx1m] [--gamma 3]
    python bench.py --impl reference ...      # the fp64 CPU oracle as the reference arm

One step = the whole hot path once (Pith verdict on arXiv 2607.21535, Eq. 1): the draft's
context pass and gamma draft forwards (ring append + windowed attention in one call, or full
paged attention in the native arm), verify attention over every target attention layer, greedy
acceptance.  Inputs are synthetic and resident in HBM before timing; each step streams ~26 GiB
of KV (more than the 126 MB L2), so no L2 flush is needed between steps.  After the headline
workload the other workloads (128K context, the ragged batch of 8 with a draft tree, the NoPE
1M window sweep) get compact records of their own.  Rank 0 prints one JSON line.  With N GPUs
every rank runs an independent replica (the path has no exchange step).
"""
import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "µs per decode step & KV-read GB/s vs HBM peak at 1M ctx (windowed vs full draft)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="wmtp", choices=["wmtp", "reference"])
    p.add_argument("--workload", default="ctx1m")
    p.add_argument("--gamma", type=int, default=3)
    p.add_argument("--window", type=int, default=0, help="recent window W (default: the workload's first)")
    p.add_argument("--no-sweep", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-loop", action="store_true", help="skip the decode-loop measurement")
    p.add_argument("--no-fp8", action="store_true", help="skip the fp8-KV measurement")
    p.add_argument("--agree", type=float, default=0.8,
                   help="decode loop: probability a synthetic draft proposal is the target's token")
    p.add_argument("--context", type=int, default=0, help="override the committed context (profiling cases)")
    p.add_argument("--layers", type=int, default=0, help="override the verify layer count (profiling cases)")
    p.add_argument("--eager", action="store_true", help="time eager launches instead of CUDA-graph replays")
    p.add_argument("--no-others", action="store_true", help="skip the records of the other workloads")
    p.add_argument("--sub-steps", type=int, default=10, help="timed steps per other workload")
    return p.parse_args()


# ----------------------------------------------------------------------------- environment
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest of the ranks' values (every rank gets it); the identity on one rank."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def per_replica_us_per_step(ms_max: float, steps: int) -> float:
    """Decode-step latency of a replica: the slowest rank's timed region over its steps (every
    rank runs the same steps on its own GPU; no exchange between replicas)."""
    return ms_max * 1e3 / steps


def aggregate_steps_per_s(ms_max: float, steps: int, world: int) -> float:
    """Whole-job throughput: N replicas ran steps x N decode steps in the slowest rank's time."""
    return steps * world / (ms_max * 1e-3)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError, TypeError):
        return dict(FALLBACK_PEAKS, bf16_tflops_sustained=1400.0, source="fallback")


# The sources that define the dominant kernel of the default workload (the mma.sync verify
# kernel) and its launch configuration: a committed traffic figure stays valid while they do.
DOMINANT_KERNEL_SOURCES = ("attn_kernels.cuh", "device_common.cuh", "capi.cu")


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "long_context_speculative_kv_b200", "csrc")
    for f in DOMINANT_KERNEL_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def committed_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on this source."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    src = kernel_source_hash()
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) == 4 and not line.startswith("#") and parts[0] == kernel \
                    and parts[1] == workload and parts[3] == src:
                return float(parts[2])
    return None


class ClockSampler:
    """nvidia-smi samples of one GPU while the timed region runs (started before, stopped after)."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.seek(0)
        text = self.file.read()
        os.unlink(self.file.name)
        return parse_clock_samples(text)


def parse_clock_samples(text: str):
    """nvidia-smi CSV rows (ClockSampler.FIELDS, no header, no units) -> median SM clock under
    load, the largest max clock, and every throttle reason seen Active; None without samples."""
    rows = [r.split(",") for r in text.strip().splitlines() if r.count(",") >= 6]
    if not rows:
        return None
    sm = [float(r[0]) for r in rows if r[0].strip().replace(".", "").isdigit()]
    mx = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    reasons = sorted({names[i] for r in rows for i in range(4) if r[3 + i].strip() == "Active"})
    return {"sm_mhz": statistics.median(sm) if sm else None,
            "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- GPU arm
class Timing:
    """CUDA-event timing on the current stream: eager steps, CUDA-graph replays of a step, and
    calls captured back to back in a graph (device time without host issue gaps)."""

    def __init__(self, world: int, device, hbm_gbs: float):
        self.world, self.device, self.hbm = world, device, hbm_gbs

    def barrier(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()

    def max_ranks(self, x: float) -> float:
        return max_over_ranks(x, self.world, self.device)

    def _events(self):
        import torch
        return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(self, step, arm, K, with_log=True, e2e=None):
        """K eager steps; (ms, per-step CallLogs, library launches)."""
        import torch

        from long_context_speculative_kv_b200 import api
        from long_context_speculative_kv_b200.step import CallLog
        logs = []
        self.barrier()
        torch.cuda.synchronize()
        e0, e1 = self._events()
        n0 = api.launch_count()
        e0.record()
        for _ in range(K):
            if e2e is not None:
                step.run_e2e(arm, *e2e)
            else:
                log = CallLog() if with_log else None
                step.run(arm, log)
                logs.append(log)
        e1.record()
        torch.cuda.synchronize()
        self.barrier()
        return e0.elapsed_time(e1), logs, api.launch_count() - n0

    def capture(self, step, arm):
        """One step of `arm` captured as a CUDA graph; (graph, library launches in it)."""
        import torch

        from long_context_speculative_kv_b200 import api
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            step.run(arm)
        torch.cuda.current_stream().wait_stream(side)
        g = torch.cuda.CUDAGraph()
        n0 = api.launch_count()
        with torch.cuda.graph(g):
            step.run(arm)
        torch.cuda.synchronize()
        return g, api.launch_count() - n0

    def capture_e2e(self, step, arm, h_in, h_out):
        """One end-to-end step captured as a CUDA graph: the H2D copies of the step's inputs from
        the pinned host buffers, the step's C-ABI calls and the D2H copies of the accepted tokens
        (memcpy nodes; each replay copies whatever the host buffers hold then)."""
        import torch
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            step.run_e2e(arm, h_in, h_out)
        torch.cuda.current_stream().wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step.run_e2e(arm, h_in, h_out)
        torch.cuda.synchronize()
        return g

    def timed_graph(self, step, g, K, e2e=None):
        import torch
        self.barrier()
        torch.cuda.synchronize()
        e0, e1 = self._events()
        e0.record()
        for _ in range(K):
            if e2e is not None:
                h_in_, h_out_ = e2e
                for n, t in h_in_.items():
                    getattr(step.b, n).copy_(t, non_blocking=True)
            g.replay()
            if e2e is not None:
                for n, t in h_out_.items():
                    t.copy_(step.b.out[n], non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        self.barrier()
        return e0.elapsed_time(e1)

    def graph_call_us(self, calls, replays):
        """Mean device time of one call: `calls` captured back to back in one graph, replayed."""
        import torch
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for c in calls:
                c()
        torch.cuda.current_stream().wait_stream(side)
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            for c in calls:
                c()
        gr.replay()
        torch.cuda.synchronize()
        e0, e1 = self._events()
        e0.record()
        for _ in range(replays):
            gr.replay()
        e1.record()
        torch.cuda.synchronize()
        del gr
        return e0.elapsed_time(e1) * 1e3 / (replays * len(calls))

    def kstat(self, label_times, nbytes):
        """Mean / median of per-call times (ms) as µs, with GB/s and the fraction of HBM peak."""
        if not label_times:
            return None
        us = statistics.mean(label_times) * 1e3
        gbs = nbytes / (us * 1e-6) / 1e9
        return {"us": round(us, 3), "us_median": round(statistics.median(label_times) * 1e3, 3),
                "bytes": nbytes, "GBps": round(gbs, 1), "frac_of_hbm_peak": round(gbs / self.hbm, 4)}


def per_label(logs):
    d = {}
    for lg in logs:
        for lab, ms in lg.durations_ms():
            d.setdefault(lab, []).append(ms)
    return d


def phases(logs, draft_labels):
    t_d, t_v, t_a = [], [], []
    for lg in logs:
        dur = lg.durations_ms()
        t_d.append(sum(ms for lab, ms in dur if lab in draft_labels))
        t_v.append(sum(ms for lab, ms in dur if lab == "verify"))
        t_a.append(sum(ms for lab, ms in dur if lab == "accept"))
    return statistics.mean(t_d) * 1e3, statistics.mean(t_v) * 1e3, statistics.mean(t_a) * 1e3


WINDOWED_LABELS = {"window_ctx", "window_fwd"}
NATIVE_LABELS = {"full_ctx", "full_fwd"}


def workload_step_bytes(w, lens, gamma, window, n_q_v):
    """Algorithmic KV bytes of the step's calls (SURVEY-style per-call formulas)."""
    from long_context_speculative_kv_b200 import accounting as acc
    row = acc.kv_row_bytes(w.Hkv, w.D)
    return {
        "verify": sum(L + n_q_v for L in lens) * row,
        "full_fwd": sum(L + gamma + 2 for L in lens) * row,      # the last forward's length
        "full_ctx": sum(L + gamma + 1 for L in lens) * row,
        "window": sum(acc.window_keys(L + gamma + 1, w.n_sink, window) for L in lens) * row,
        "append_1": acc.append_bytes(1, w.Hkv, w.D) * w.B,
    }


def run_gpu(args):
    import gc

    import torch
    import torch.distributed as dist

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)
    peaks = measured_peaks()
    T = Timing(world, device, peaks["hbm_gbs"])
    line = measure_headline(args, T, peaks, rank, world, local, device)
    if not args.no_others:
        gc.collect()
        torch.cuda.empty_cache()
        line["workloads"] = measure_other_workloads(args, T, device)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def measure_headline(args, T, peaks, rank, world, local, device):
    import torch

    from long_context_speculative_kv_b200 import accounting as acc
    from long_context_speculative_kv_b200 import api
    from long_context_speculative_kv_b200.loop import DecodeLoop, LoopState
    from long_context_speculative_kv_b200.step import CallLog, DecodeStep, StepBuffers
    from synthetic import configs, workload

    w = configs.BY_NAME[args.workload]
    if args.context:
        import dataclasses
        w = dataclasses.replace(w, L=args.context, ragged=(0, 0), name=f"{w.name}@L{args.context}")
    window = args.window or w.windows[0]
    gammas = sorted(set(w.gammas) | {args.gamma}) if not args.no_sweep else [args.gamma]
    if w.tree_nodes:
        gammas = [args.gamma]
    max_nq = max([w.tree_nodes or (g + 1) for g in gammas])
    do_loop = not args.no_loop and not w.tree_nodes
    loop_extra = 24                                   # untimed loop steps per arm (warm-up, breakdown)
    slack = (max(gammas) + 1) * (args.steps + args.warmup + loop_extra) if do_loop else 0
    shared = workload.shared_inputs(w, device, max_nq_verify=max_nq, max_gamma=max(gammas),
                                    window=window, n_layers=args.layers or None, slack=slack)
    lens = shared["lens"]

    def make_step(gamma):
        return DecodeStep(StepBuffers(**workload.step_inputs(w, shared, gamma, device)), gamma)

    step = make_step(args.gamma)
    n_q_v = step.n_q_verify
    n_layers = step.n_layers
    nb = workload_step_bytes(w, lens, args.gamma, window, n_q_v)
    kstat = T.kstat

    for _ in range(args.warmup):
        step.run("windowed")
        step.run("native")
    torch.cuda.synchronize()
    assert api.device_status() == 0

    props = torch.cuda.get_device_properties(device)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local)
    use_graph = not args.eager
    if use_graph:
        g_w, per_step_launches = T.capture(step, "windowed")
        g_n, per_step_launches_n = T.capture(step, "native")
        for _ in range(2):
            g_w.replay()
            g_n.replay()
    clocks = ClockSampler(gpu_id)
    time.sleep(0.3)
    if use_graph:
        ms_w = T.timed_graph(step, g_w, args.steps)
        ms_n = T.timed_graph(step, g_n, args.steps)
        launches = per_step_launches * args.steps
    else:
        ms_w, _, launches = T.timed(step, "windowed", args.steps, with_log=False)
        ms_n, _, _ = T.timed(step, "native", args.steps, with_log=False)
        per_step_launches_n = None
    clk = clocks.stop()
    # per-call breakdown from eager launches with CUDA events between calls
    ms_w_eager, logs_w, _ = T.timed(step, "windowed", args.steps)
    ms_n_eager, logs_n, _ = T.timed(step, "native", args.steps)
    assert api.device_status() == 0

    lw, ln = per_label(logs_w), per_label(logs_n)
    us_w_local = ms_w * 1e3 / args.steps
    us_n_local = ms_n * 1e3 / args.steps
    ms_w_max, ms_n_max = T.max_ranks(ms_w), T.max_ranks(ms_n)
    value = per_replica_us_per_step(ms_w_max, args.steps)
    tdw, tvw, taw = phases(logs_w, WINDOWED_LABELS)
    tdn, tvn, tan = phases(logs_n, NATIVE_LABELS)
    hbm = peaks["hbm_gbs"]

    kernels = {
        "verify_attn": kstat(lw.get("verify"), nb["verify"]),
        "draft_attn_full_fwd": kstat(ln.get("full_fwd"), nb["full_fwd"]),
        "draft_attn_full_ctx": kstat(ln.get("full_ctx"), nb["full_ctx"]),
        "draft_attn_window_append_fwd_inloop": kstat(lw.get("window_fwd"), nb["window"]),
        "draft_attn_window_append_ctx_inloop": kstat(lw.get("window_ctx"), nb["window"]),
        "accept_greedy": kstat(lw.get("accept"), w.B * n_q_v * w.vocab * 4),
    }

    # ---- stochastic acceptance on the step's verify nodes (softmax probabilities in) ----------
    if not w.tree_nodes:
        gs = torch.Generator(device=device)
        gs.manual_seed(w.seed + 5)
        p_ = torch.softmax(torch.randn((w.B, n_q_v, w.vocab), generator=gs, device=device), -1)
        q_ = torch.softmax(torch.randn((w.B, n_q_v - 1, w.vocab), generator=gs, device=device), -1)
        ua = torch.randint(0, 1 << 24, (w.B, n_q_v - 1), generator=gs, device=device, dtype=torch.int32)
        us = torch.randint(-(1 << 31), (1 << 31) - 1, (w.B,), generator=gs, device=device, dtype=torch.int32)
        acc_, nacc_ = api.accept_stochastic(p_, q_, step.b.tokens, ua, us)
        ev = []
        for _ in range(50):
            e0, e1 = T._events()
            e0.record()
            api.accept_stochastic(p_, q_, step.b.tokens, ua, us, accepted=acc_, n_accepted=nacc_)
            e1.record()
            ev.append((e0, e1))
        torch.cuda.synchronize()
        assert api.device_status() == 0
        kernels["accept_stochastic"] = kstat([a.elapsed_time(c) for a, c in ev[5:]], 2 * w.B * w.vocab * 4)

    # ---- device-side phase and small-call times: calls captured back to back in one CUDA graph
    #      and replayed (as the step runs), so the host's issue time between eager calls, which
    #      exceeds the device time of the small calls, is not counted ---------------------------
    phases_graph, kernels_graph = None, {}
    if use_graph:
        Kp = max(5, args.steps // 10)
        b_ = step.b
        phases_graph = {
            "windowed_t_draft_us": round(T.graph_call_us([step.draft_windowed], Kp), 2),
            "native_t_draft_us": round(T.graph_call_us([step.draft_native], Kp), 2),
            "t_verify_us": round(T.graph_call_us([step.verify], Kp), 2),
            "t_accept_us": round(T.graph_call_us([step.accept] * 10, Kp), 2),
        }
        # one draft forward (ring append fused into the windowed attention) and the plain
        # windowed call; 20 back to back, as the decode loop issues them
        fwd_us = T.graph_call_us([lambda: step._forward(b_.q_fwd[0], b_.k_fwd[0], b_.v_fwd[0], b_.out["fwd"],
                                                        b_.out["fwd_lse"])] * 20, Kp)
        win_us = T.graph_call_us([lambda: step._window(b_.q_fwd[0], b_.out["fwd"], b_.out["fwd_lse"])] * 20, Kp)
        app_us = T.graph_call_us([lambda: step._append(b_.k_fwd[0], b_.v_fwd[0])] * 20, Kp)
        ctx_us = T.graph_call_us([lambda: step._forward(b_.q_ctx, b_.k_ctx, b_.v_ctx, b_.out["ctx"],
                                                        b_.out["ctx_lse"])] * 10, Kp)
        full_us = T.graph_call_us([lambda: step._full(b_.q_fwd[0], b_.kv_len_fwd[0], b_.out["fwd"],
                                                      b_.out["fwd_lse"])] * 4, Kp)
        kernels_graph = {
            "draft_attn_window_append_fwd": kstat([fwd_us / 1e3], nb["window"]),
            "draft_attn_window_append_ctx": kstat([ctx_us / 1e3], nb["window"]),
            "draft_attn_window_call": kstat([win_us / 1e3], nb["window"]),
            "ring_kv_append_1": kstat([app_us / 1e3], nb["append_1"]),
            "draft_attn_full_fwd": kstat([full_us / 1e3], nb["full_fwd"]),
            "accept_greedy": kstat([phases_graph["t_accept_us"] / 1e3], w.B * n_q_v * w.vocab * 4),
        }
        # the step's ring has grown by the calls above; put its length back
        b_.ring_len.copy_(shared["ring_len0"])
        assert api.device_status() == 0

    # ---- windowed draft with a cold L2: rotate over ring copies larger than 2x L2 ----------
    cold = None
    if "ring_k" in shared:
        l2 = props.L2_cache_size if hasattr(props, "L2_cache_size") else 126 << 20
        ring_bytes = shared["ring_k"].numel() * 4
        R = max(4, int(2.5 * l2 // ring_bytes) + 1)
        rings = [(torch.empty_like(shared["ring_k"]).normal_(), torch.empty_like(shared["ring_v"]).normal_())
                 for _ in range(R)]
        rl = shared["ring_len0"] + args.gamma + 2
        b = step.b
        times = []
        for it in range(3 * R):
            rk, rv = rings[it % R]
            e0, e1 = T._events()
            e0.record()
            api.draft_attn_window(b.q_fwd[0], rk, rv, rl, w.n_sink, window, w.sm_scale, b.ws,
                                  out=b.out["fwd"], lse=b.out["fwd_lse"])
            e1.record()
            times.append((e0, e1))
        torch.cuda.synchronize()
        t = [a.elapsed_time(c) for a, c in times[R:]]
        cold = kstat(t, nb["window"])
        cold["rotating_copies"] = R
        if use_graph:
            def win_call(rk, rv):
                return lambda: api.draft_attn_window(b.q_fwd[0], rk, rv, rl, w.n_sink, window, w.sm_scale,
                                                     b.ws, out=b.out["fwd"], lse=b.out["fwd_lse"])
            cold_us = T.graph_call_us([win_call(rk, rv) for rk, rv in rings], 3)
            kernels_graph["draft_attn_window_call_cold"] = dict(kstat([cold_us / 1e3], nb["window"]),
                                                               rotating_copies=R)
        del rings
        torch.cuda.empty_cache()

    # ---- end to end through the public API with host buffers --------------------------------
    step.pack_io()          # one H2D and one D2H copy per step
    h_in, h_out = step.host_inputs(), step.host_outputs()
    for _ in range(2):
        step.run_e2e("windowed", h_in, h_out)
    ms_e2e_eager, _, _ = T.timed(step, "windowed", args.steps, e2e=(h_in, h_out))
    if use_graph:
        g_e2e = T.capture_e2e(step, "windowed", h_in, h_out)
        ms_e2e = T.timed_graph(step, g_e2e, args.steps)
        del g_e2e
    else:
        ms_e2e = ms_e2e_eager
    e2e_value = per_replica_us_per_step(T.max_ranks(ms_e2e), args.steps)
    e2e_eager_value = per_replica_us_per_step(T.max_ranks(ms_e2e_eager), args.steps)
    if use_graph:
        del g_w, g_n

    # ---- draft-depth sweep -------------------------------------------------------------
    sweep = {}
    if len(gammas) > 1:
        Ks = max(5, args.steps // 10)
        base_step = step
        for g in gammas:
            st = base_step if g == args.gamma else make_step(g)
            for _ in range(2):
                st.run("windowed")
                st.run("native")
            _, lgw, _ = T.timed(st, "windowed", Ks)
            _, lgn, _ = T.timed(st, "native", Ks)
            if use_graph:
                gw, _ = T.capture(st, "windowed")
                gn, _ = T.capture(st, "native")
                mw, mn = T.timed_graph(st, gw, Ks), T.timed_graph(st, gn, Ks)
                del gw, gn
            else:
                mw, _, _ = T.timed(st, "windowed", Ks, with_log=False)
                mn, _, _ = T.timed(st, "native", Ks, with_log=False)
            dw, vw, _ = phases(lgw, WINDOWED_LABELS)
            dn, vn, _ = phases(lgn, NATIVE_LABELS)
            sweep[str(g)] = {"windowed_us": round(T.max_ranks(mw) * 1e3 / Ks, 2),
                             "native_us": round(T.max_ranks(mn) * 1e3 / Ks, 2),
                             "t_draft_windowed_us": round(dw, 2), "t_draft_native_us": round(dn, 2),
                             "t_verify_us": round((vw + vn) / 2, 2)}
            sweep[str(g)]["step_cost_reduction_pct"] = round(
                100 * (sweep[str(g)]["native_us"] / sweep[str(g)]["windowed_us"] - 1), 2)
            if st is not base_step:
                del st

    # ---- context sweep and linear fit of the draft terms (the Table 6 analogue) ------------
    ctx_sweep = None
    if not args.no_sweep and w.B == 1 and not w.tree_nodes:
        Ls = [x for x in (1 << 16, 1 << 17, 1 << 18, 1 << 19, 1 << 20) if x <= lens[0]]
        if len(Ls) >= 3:
            Kc = max(5, args.steps // 10)
            pts = []
            for Lx in Ls:
                st = DecodeStep(StepBuffers(**workload.step_inputs(w, shared, args.gamma, device,
                                                                   lens=[Lx])), args.gamma)
                for _ in range(2):
                    st.run("windowed")
                    st.run("native")
                _, lgw, _ = T.timed(st, "windowed", Kc)
                _, lgn, _ = T.timed(st, "native", Kc)
                if use_graph:
                    gw, _ = T.capture(st, "windowed")
                    gn, _ = T.capture(st, "native")
                    mw, mn = T.timed_graph(st, gw, Kc), T.timed_graph(st, gn, Kc)
                    del gw, gn
                else:
                    mw, _, _ = T.timed(st, "windowed", Kc, with_log=False)
                    mn, _, _ = T.timed(st, "native", Kc, with_log=False)
                lw_, ln_ = per_label(lgw), per_label(lgn)
                pt = {"L": Lx,
                      "t_fwd_draft_windowed_us": round(statistics.mean(lw_["window_fwd"]) * 1e3, 3),
                      "t_fwd_draft_native_us": round(statistics.mean(ln_["full_fwd"]) * 1e3, 3),
                      "t_ctx_draft_windowed_us": round(statistics.mean(lw_["window_ctx"]) * 1e3, 3),
                      "t_ctx_draft_native_us": round(statistics.mean(ln_["full_ctx"]) * 1e3, 3),
                      "step_windowed_us": round(T.max_ranks(mw) * 1e3 / Kc, 2),
                      "step_native_us": round(T.max_ranks(mn) * 1e3 / Kc, 2)}
                if use_graph:
                    # the same draft terms on the device alone: each term's calls captured back
                    # to back in a CUDA graph and replayed
                    sb_ = st.b
                    pt["t_fwd_draft_windowed_graph_us"] = round(T.graph_call_us(
                        [lambda: st._forward(sb_.q_fwd[0], sb_.k_fwd[0], sb_.v_fwd[0], sb_.out["fwd"],
                                             sb_.out["fwd_lse"])] * 10, Kc), 3)
                    pt["t_ctx_draft_windowed_graph_us"] = round(T.graph_call_us(
                        [lambda: st._forward(sb_.q_ctx, sb_.k_ctx, sb_.v_ctx, sb_.out["ctx"],
                                             sb_.out["ctx_lse"])] * 10, Kc), 3)
                    pt["t_fwd_draft_native_graph_us"] = round(T.graph_call_us(
                        [lambda: st._full(sb_.q_fwd[0], sb_.kv_len_fwd[0], sb_.out["fwd"], sb_.out["fwd_lse"])] * 4,
                        Kc), 3)
                    pt["t_ctx_draft_native_graph_us"] = round(T.graph_call_us(
                        [lambda: st._full(sb_.q_ctx, sb_.kv_len_ctx, sb_.out["ctx"], sb_.out["ctx_lse"])] * 4,
                        Kc), 3)
                    assert api.device_status() == 0
                pts.append(pt)
                del st
            fits = {}
            xs = [p_["L"] for p_ in pts]
            keys = ["t_fwd_draft_windowed_us", "t_fwd_draft_native_us", "t_ctx_draft_windowed_us",
                    "t_ctx_draft_native_us", "step_windowed_us", "step_native_us"]
            if use_graph:
                keys += ["t_fwd_draft_windowed_graph_us", "t_fwd_draft_native_graph_us",
                         "t_ctx_draft_windowed_graph_us", "t_ctx_draft_native_graph_us"]
            for key in keys:
                m, c, r2 = acc.linear_fit(xs, [p_[key] for p_ in pts])
                fits[key[:-3]] = {"slope_us_per_1k_tokens": round(m * 1e3, 5),
                                  "intercept_us": round(c, 3), "r2": round(r2, 5)}
            sn, sw = fits["step_native"]["slope_us_per_1k_tokens"], fits["step_windowed"]["slope_us_per_1k_tokens"]
            ctx_sweep = {"points": pts, "fits": fits, "gamma": args.gamma,
                         "step_slope_reduction_pct": round(100 * (1 - sw / sn), 2) if sn > 0 else None,
                         "timing": "step: CUDA-graph replay; per-call terms: eager launches with events, "
                                   "and (*_graph) the same calls captured back to back in a CUDA graph"}

    # ---- decode loop: real acceptance from the synthetic heads, rollback, graph per step -------
    loop_res = None
    if do_loop:
        agree24 = int(round(args.agree * (1 << 24)))
        T0 = [L + 1 for L in lens]

        def make_loop(arm_seed):
            kw = workload.step_inputs(w, shared, args.gamma, device, seed=w.seed + 17 * arm_seed)
            gl = torch.Generator(device=device)
            gl.manual_seed(w.seed + 99)
            hist = torch.randint(0, w.vocab, (w.B, max(T0) + slack), generator=gl, device=device,
                                 dtype=torch.int32)
            state = LoopState.start(hist, T0, args.gamma)
            C = w.n_sink + window + args.gamma
            rk = torch.empty((w.B, w.Hkv, C, w.D), dtype=torch.bfloat16, device=device).normal_(generator=gl)
            rv = torch.empty_like(rk).normal_(generator=gl)
            kw.update(ring_k=rk, ring_v=rv, ring_len=torch.zeros(w.B, dtype=torch.int64, device=device),
                      kv_len_v=state.verify_len)
            return DecodeLoop(StepBuffers(**kw), args.gamma, state, w.vocab, w.seed + 1000, w.seed + 2000, agree24)

        loop_res = {"agree": args.agree, "gamma": args.gamma,
                    "step": "ring append at the committed position (rollback) + window ctx pass, gamma "
                            "fused forwards (append + windowed attention), synthetic draft proposals, "
                            "verify x layers, synthetic target logits, accept_greedy, spec_commit; one "
                            "CUDA graph per step"}
        for arm in ("windowed", "native"):
            lp = make_loop(0 if arm == "windowed" else 1)
            for _ in range(2):
                lp.step(arm)
            side = torch.cuda.Stream()
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                lp.step(arm)
            torch.cuda.current_stream().wait_stream(side)
            gl_ = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gl_):
                lp.step(arm)
            for _ in range(args.warmup):
                gl_.replay()
            torch.cuda.synchronize()
            t_before = lp.s.n_tokens.clone()
            ms = T.timed_graph(step, gl_, args.steps)
            committed = int((lp.s.n_tokens - t_before).sum().item())
            del gl_
            logs = []
            for _ in range(8):
                lg = CallLog()
                lp.step(arm, lg)
                logs.append(lg)
            torch.cuda.synchronize()
            assert api.device_status() == 0
            d = per_label(logs)
            draft_labels = ("append_ctx", "window_ctx", "window_fwd", "full_ctx", "full_fwd")
            ms_max = T.max_ranks(ms)
            loop_res[arm] = {
                "us_per_step": round(ms_max * 1e3 / args.steps, 2),
                "tokens_committed": committed,
                "mean_accepted_per_step": round(committed / (args.steps * w.B), 4),
                "us_per_token": round(ms_max * 1e3 / max(1, committed), 2),
                "t_draft_us": round(sum(statistics.mean(d[k]) * len(d[k]) / len(logs) for k in draft_labels if k in d) * 1e3, 2),
                "t_ctx_draft_us": round(sum(statistics.mean(d[k]) for k in ("append_ctx", "window_ctx", "full_ctx") if k in d) * 1e3, 2),
                "t_verify_us": round(statistics.mean(d["verify"]) * len(d["verify"]) / len(logs) * 1e3, 2),
                "t_heads_accept_commit_us": round(sum(statistics.mean(d[k]) for k in ("propose", "target_logits", "accept", "commit")) * 1e3, 2),
            }
            del lp
        loop_res["step_cost_reduction_pct"] = round(
            100 * (loop_res["native"]["us_per_step"] / loop_res["windowed"]["us_per_step"] - 1), 2)
        loop_res["per_token_speedup"] = round(loop_res["native"]["us_per_token"] / loop_res["windowed"]["us_per_token"], 4)

    # ---- fp8 (E4M3) KV: the same step with every K/V cache in fp8 ---------------------------
    fp8_res = None
    if not args.no_fp8:
        shared8 = workload.shared_inputs(w, device, max_nq_verify=n_q_v, max_gamma=args.gamma,
                                         window=window, n_layers=args.layers or None, kv8=True)
        st8 = DecodeStep(StepBuffers(**workload.step_inputs(w, shared8, args.gamma, device)), args.gamma)
        K8 = max(10, args.steps // 4)
        for _ in range(2):
            st8.run("windowed")
            st8.run("native")
        _, lg8w, _ = T.timed(st8, "windowed", K8)
        _, lg8n, _ = T.timed(st8, "native", K8)
        if use_graph:
            gw8, _ = T.capture(st8, "windowed")
            gn8, _ = T.capture(st8, "native")
            m8w, m8n = T.timed_graph(st8, gw8, K8), T.timed_graph(st8, gn8, K8)
            del gw8, gn8
            v8_us = T.graph_call_us([st8.verify], max(5, args.steps // 10)) / n_layers
        else:
            m8w, _, _ = T.timed(st8, "windowed", K8, with_log=False)
            m8n, _, _ = T.timed(st8, "native", K8, with_log=False)
            v8_us = None
        assert api.device_status() == 0
        l8w, l8n = per_label(lg8w), per_label(lg8n)
        row8 = w.Hkv * w.D * 2                                 # K + V bytes of one position
        fp8_res = {
            "k_scale": st8.b.k_scale, "v_scale": st8.b.v_scale,
            "windowed_us": round(T.max_ranks(m8w) * 1e3 / K8, 2),
            "native_us": round(T.max_ranks(m8n) * 1e3 / K8, 2),
            "kernels": {
                "verify_attn_fp8": kstat(l8w.get("verify"), sum(L + n_q_v for L in lens) * row8),
                "draft_attn_full_fp8_fwd": kstat(l8n.get("full_fwd"), sum(L + args.gamma + 2 for L in lens) * row8),
                "draft_attn_window_append_fp8_fwd_inloop": kstat(
                    l8w.get("window_fwd"),
                    sum(acc.window_keys(L + args.gamma + 1, w.n_sink, window) for L in lens) * row8),
            },
        }
        if v8_us is not None:
            fp8_res["kernels_graph"] = {"verify_attn_fp8": kstat([v8_us / 1e3], sum(L + n_q_v for L in lens) * row8)}
        fp8_res["step_cost_reduction_pct"] = round(100 * (fp8_res["native_us"] / fp8_res["windowed_us"] - 1), 2)
        fp8_res["windowed_speedup_over_bf16"] = round(us_w_local / fp8_res["windowed_us"], 4)
        del st8, shared8
        torch.cuda.empty_cache()

    # ---- KV accounting -------------------------------------------------------------------
    Lm = int(statistics.mean(lens))
    sb_w = acc.step_bytes(Lm, args.gamma, n_q_v, w.Hkv, w.D, n_layers, w.n_sink, window, windowed=True)
    sb_n = acc.step_bytes(Lm, args.gamma, n_q_v, w.Hkv, w.D, n_layers, w.n_sink, window, windowed=False)
    accounting = {
        "draft_kv_bytes_per_step_windowed": sb_w.draft * w.B,
        "draft_kv_bytes_per_step_native": sb_n.draft * w.B,
        "draft_kv_entries_dropped": round(acc.dropped_fraction(Lm, w.n_sink + window), 6),
        "kv_reclaimed_share_of_total": round(acc.reclaimed_share_of_total(Lm, w.n_sink + window, n_layers), 6),
        "pages_quote": "+28% to +44% per-decode-step cost reduction at 1M, ~99% draft KV dropped, "
                       "7.7-11% of total KV reclaimed (one GPU in SGLang, hardware unstated)",
    }

    # ---- CPU baseline: the oracle on the host cores (rank 0, one GPU only) ------------------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_step_estimate(w, args.gamma, window, lens, n_q_v, n_layers)

    traffic = committed_traffic("verify_attn", w.name)
    v = kernels["verify_attn"]
    v_src = "eager verify calls with CUDA events between calls"
    if phases_graph:
        # the step's verify layers as they run in the step's graph: back to back, each the
        # attention kernel plus its LSE merge; per-layer mean of the replayed graph
        v = kstat([phases_graph["t_verify_us"] / n_layers / 1e3], nb["verify"])
        kernels_graph["verify_attn"] = v
        v_src = "CUDA events around a graph of the step's verify layers, replayed; mean per layer"
    roofline = {"kernel": "verify_attn (split attention + LSE merge, one target layer)",
                "bound": "hbm", "achieved": v["GBps"], "peak": hbm, "unit": "GB/s",
                "frac": v["frac_of_hbm_peak"], "us_per_launch": v["us"], "duration_source": v_src,
                "traffic": traffic, "peak_source": peaks["source"] + " (MEASURED_PEAKS.json hbm_gbs)"
                if peaks["source"] == "measured" else "fallback 6.65 TB/s"}

    cfg = {"workload": f"{w.name}: B={w.B} L={'ragged ' + str(w.ragged) if w.ragged[1] else w.L} "
                       f"Hq={w.Hq} Hkv={w.Hkv} D={w.D} page={w.page_size} window={w.n_sink}+{window} "
                       f"gamma={args.gamma} verify_layers={n_layers}"
                       + (f" tree={w.tree_nodes}" if w.tree_nodes else " chain"),
           "gamma": args.gamma, "window": window, "n_sink": w.n_sink, "verify_layers": n_layers,
           "batch": w.B, "context": lens if w.B <= 8 else Lm,
           "l2": "inputs larger than L2 (each step streams %.1f GiB of KV)" % (sb_w.total * w.B / 2 ** 30),
           "value_is": "windowed-arm us per decode step of one replica = max-over-ranks time / steps",
           "parallelism": f"replicas x{world}",
           "launch_mode": "CUDA graph of one decode step, replayed" if use_graph else "eager launches"}
    return {
        "metric": METRIC, "value": round(value, 3), "unit": "us/step", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(value / 1e3, 6),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 Q/K/V, random page tables)", "config": cfg,
        "aggregate_steps_per_s": round(aggregate_steps_per_s(ms_w_max, args.steps, world), 2),
        "windowed": {"us_per_step": round(us_w_local, 2), "us_per_step_eager": round(ms_w_eager * 1e3 / args.steps, 2),
                     "t_draft_us": round(tdw, 2), "t_verify_us": round(tvw, 2), "t_accept_us": round(taw, 2)},
        "native": {"us_per_step": round(us_n_local, 2), "us_per_step_eager": round(ms_n_eager * 1e3 / args.steps, 2),
                   "t_draft_us": round(tdn, 2), "t_verify_us": round(tvn, 2), "t_accept_us": round(tan, 2)},
        "phase_times_from": "eager launches with CUDA events between calls",
        "phases_graph": phases_graph,
        "kernels_graph": kernels_graph or None,
        "kernels_graph_note": "each phase or call captured back to back in a CUDA graph and replayed; "
                              "device time without the host issue gaps of eager calls",
        "step_cost_ratio_native_over_windowed": round(ms_n_max / ms_w_max, 4),
        "step_cost_reduction_pct": round(100 * (ms_n_max / ms_w_max - 1), 2),
        "kernels": dict(kernels, draft_attn_window_call_cold=cold),
        "gamma_sweep": sweep, "context_sweep": ctx_sweep, "decode_loop": loop_res, "fp8_kv": fp8_res,
        "kv_accounting": accounting,
        "roofline": roofline, "cpu_baseline": cpu,
        "e2e": {"value": round(e2e_eager_value, 3), "unit": "us/step",
                "h2d_bytes_per_step": DecodeStep.bytes_of(h_in), "d2h_bytes_per_step": DecodeStep.bytes_of(h_out),
                "mode": "every C-ABI call of the step issued from the host each step, with one copy of the "
                        "step's inputs from pinned host memory before them and one copy of the accepted "
                        "tokens to pinned host memory after them, all inside the timed region",
                "graph_value": round(e2e_value, 3),
                "graph_mode": "the same step (copies included) captured once as a CUDA graph and replayed"},
        "gpu_launches": launches, "gpu_launches_per_step": launches / args.steps,
        "gpu_launches_per_step_native": per_step_launches_n,
        "clocks": clk, "kernel_source": kernel_source_hash(),
    }


def measure_other_workloads(args, T, device):
    """Compact records of the other workloads, each built after the previous one is freed: the
    step per arm (CUDA-graph replays), the device-side phase split, verify per layer against the
    HBM peak, one draft forward (ring append + windowed attention in one call) and the plain
    windowed call, and the KV accounting.  The NoPE workload adds its window sweep."""
    import gc

    import torch

    from long_context_speculative_kv_b200 import accounting as acc
    from long_context_speculative_kv_b200 import api
    from long_context_speculative_kv_b200.step import DecodeStep, StepBuffers
    from synthetic import configs, workload
    from synthetic import torch_gen as tg

    K = args.sub_steps
    out = {}
    for name, gamma in (("ctx128k", 3), ("batch8-tree", 7), ("nope1m-outlier", 5)):
        if name == args.workload:
            continue
        w = configs.BY_NAME[name]
        t0 = time.perf_counter()
        shared = workload.shared_inputs(w, device, max_nq_verify=w.tree_nodes or gamma + 1,
                                        max_gamma=gamma, window=w.windows[0] if name != "nope1m-outlier" else 4092)
        window = shared["window"]
        lens = shared["lens"]
        step = DecodeStep(StepBuffers(**workload.step_inputs(w, shared, gamma, device)), gamma)
        n_q_v, n_layers = step.n_q_verify, step.n_layers
        nb = workload_step_bytes(w, lens, gamma, window, n_q_v)
        for _ in range(3):
            step.run("windowed")
            step.run("native")
        g_w, _ = T.capture(step, "windowed")
        g_n, _ = T.capture(step, "native")
        g_w.replay()
        g_n.replay()
        mw, mn = T.timed_graph(step, g_w, K), T.timed_graph(step, g_n, K)
        del g_w, g_n
        b_ = step.b
        Kp = max(3, K // 2)
        ph = {"windowed_t_draft_us": round(T.graph_call_us([step.draft_windowed], Kp), 2),
              "native_t_draft_us": round(T.graph_call_us([step.draft_native], Kp), 2),
              "t_verify_us": round(T.graph_call_us([step.verify], Kp), 2)}
        fwd = T.graph_call_us([lambda: step._forward(b_.q_fwd[0], b_.k_fwd[0], b_.v_fwd[0], b_.out["fwd"],
                                                     b_.out["fwd_lse"])] * 20, Kp)
        win = T.graph_call_us([lambda: step._window(b_.q_fwd[0], b_.out["fwd"], b_.out["fwd_lse"])] * 20, Kp)
        assert api.device_status() == 0
        Lm = int(statistics.mean(lens))
        sb_w = acc.step_bytes(Lm, gamma, n_q_v, w.Hkv, w.D, n_layers, w.n_sink, window, windowed=True)
        sb_n = acc.step_bytes(Lm, gamma, n_q_v, w.Hkv, w.D, n_layers, w.n_sink, window, windowed=False)
        us_w, us_n = T.max_ranks(mw) * 1e3 / K, T.max_ranks(mn) * 1e3 / K
        rec = {
            "config": f"B={w.B} L={'U' + str(list(w.ragged)) if w.ragged[1] else w.L} Hq={w.Hq} Hkv={w.Hkv} "
                      f"window={w.n_sink}+{window} gamma={gamma} verify_layers={n_layers}"
                      + (f" tree={w.tree_nodes}" if w.tree_nodes else " chain")
                      + (f" outliers={w.outlier_p}x{w.outlier_factor}" if w.outlier_p else ""),
            "windowed_us_per_step": round(us_w, 2), "native_us_per_step": round(us_n, 2),
            "step_cost_reduction_pct": round(100 * (us_n / us_w - 1), 2),
            "phases_graph": ph,
            "verify_attn_per_layer": T.kstat([ph["t_verify_us"] / n_layers / 1e3], nb["verify"]),
            "draft_attn_window_append_fwd": T.kstat([fwd / 1e3], nb["window"]),
            "draft_attn_window_call": T.kstat([win / 1e3], nb["window"]),
            "draft_kv_bytes_per_step_windowed": sb_w.draft * w.B,
            "draft_kv_bytes_per_step_native": sb_n.draft * w.B,
            "draft_kv_entries_dropped": round(acc.dropped_fraction(Lm, w.n_sink + window), 6),
            "kv_reclaimed_share_of_total": round(acc.reclaimed_share_of_total(Lm, w.n_sink + window, n_layers), 6),
            "steps": K,
        }
        if name == "nope1m-outlier":
            # the window sweep: rings of n_sink + W slots, the same queries and new rows
            sweep = {}
            g = tg.generator(w.seed + 31, device)
            for W in w.windows:
                C = w.n_sink + W
                rk, rv = tg.kv_rows_bf16((w.B, w.Hkv, C, w.D), g, device, w.k_scale, w.outlier_p)
                rl = torch.tensor(lens, dtype=torch.int64, device=device)
                byt = sum(acc.window_keys(L + 1, w.n_sink, W) for L in lens) * acc.kv_row_bytes(w.Hkv, w.D)

                def fwd_w():
                    api.draft_attn_window_append(b_.q_fwd[0], rk, rv, rl, b_.k_fwd[0], b_.v_fwd[0], w.n_sink, W,
                                                 w.sm_scale, b_.ws, out=b_.out["fwd"], lse=b_.out["fwd_lse"])

                def win_w():
                    api.draft_attn_window(b_.q_fwd[0], rk, rv, rl, w.n_sink, W, w.sm_scale, b_.ws,
                                          out=b_.out["fwd"], lse=b_.out["fwd_lse"])
                f_us = T.graph_call_us([fwd_w] * 20, Kp)
                c_us = T.graph_call_us([win_w] * 20, Kp)
                sb = acc.step_bytes(Lm, gamma, n_q_v, w.Hkv, w.D, n_layers, w.n_sink, W, windowed=True)
                sweep[str(W)] = {
                    "draft_attn_window_append_fwd": T.kstat([f_us / 1e3], byt),
                    "draft_attn_window_call": T.kstat([c_us / 1e3], byt),
                    "draft_kv_bytes_per_step": sb.draft * w.B,
                    "kv_reclaimed_vs_full_draft_cache": round(acc.dropped_fraction(Lm, C), 6),
                    "kv_reclaimed_share_of_total": round(acc.reclaimed_share_of_total(Lm, C, n_layers), 6),
                }
                del rk, rv
            assert api.device_status() == 0
            rec["window_sweep"] = sweep
        rec["wall_s"] = round(time.perf_counter() - t0, 1)
        out[name] = rec
        del step, shared, b_
        gc.collect()
        torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------------------- CPU oracle
class OracleSample:
    """A bounded sample of one windowed-arm decode step for the fp64 oracle: a few query rows of
    one verify layer at the workload's context, every windowed-draft row of one kv head, and one
    acceptance.  Inputs are drawn once; ``estimate()`` times the oracle on them and scales each
    part by the rows the full step has (at a fixed key count the cost per row does not depend on
    the row)."""

    def __init__(self, w, gamma, window, L, n_q_v, n_layers, rows=None):
        import numpy as np

        import oracle
        from synthetic import gen

        self.oracle = oracle
        self.w, self.gamma, self.window, self.n_q_v, self.n_layers = w, gamma, window, n_q_v, n_layers
        self.cores = oracle.max_threads()
        self.rows_n = rows or max(2, self.cores)
        rng = np.random.default_rng(w.seed)
        self.Lv = L + n_q_v
        G, D = w.G, w.D
        self.kv, self.vv = gen.kv_pair_bf16(rng, (1, 1, self.Lv, D), k_scale=w.k_scale, outlier_p=w.outlier_p)
        self.qv = gen.normal_bf16(rng, (1, n_q_v, G, D))
        self.Ld = L + gamma + 1
        self.kd, self.vd = gen.kv_pair_bf16(rng, (1, 1, self.Ld + gamma, D), k_scale=w.k_scale,
                                            outlier_p=w.outlier_p)
        self.qc = gen.normal_bf16(rng, (1, gamma + 1, G, D))
        self.qf = gen.normal_bf16(rng, (1, 1, G, D))
        self.logits = gen.uniform_logits(rng, (w.B, n_q_v, w.vocab))
        self.toks = rng.integers(0, w.vocab, size=(w.B, n_q_v)).astype(np.int32)

    def _time(self, fn):
        t0 = time.perf_counter()
        fn()
        return time.perf_counter() - t0

    def estimate(self):
        o, w, g = self.oracle, self.w, self.gamma
        G = w.G
        rows = [(0, i % self.n_q_v, (i // self.n_q_v) % G) for i in range(self.rows_n)]
        t_rows = self._time(lambda: o.attention(self.qv, self.kv, self.vv, [self.Lv], o.MODE_CAUSAL,
                                                w.sm_scale, rows=rows))
        scale_v = self.n_q_v * w.Hq * self.n_layers * w.B / self.rows_n
        t_verify = t_rows * scale_v
        t_ctx = self._time(lambda: o.attention(self.qc, self.kd, self.vd, [self.Ld], o.MODE_WINDOW,
                                               w.sm_scale, n_sink=w.n_sink, window=self.window))
        t_fwd = self._time(lambda: o.attention(self.qf, self.kd, self.vd, [self.Ld + 1], o.MODE_WINDOW,
                                               w.sm_scale, n_sink=w.n_sink, window=self.window))
        t_draft = (t_ctx + g * t_fwd) * w.Hkv * w.B
        t_acc = self._time(lambda: o.accept_greedy(self.logits, self.toks))
        total = t_verify + t_draft + t_acc
        return {"value": round(total * 1e6, 1), "unit": "us/step", "cores": self.cores, "kind": "oracle",
                "sample": f"{self.rows_n} verify query rows at {self.Lv} keys (x{scale_v:.0f}), every "
                          f"windowed-draft row of one kv head (x{w.Hkv * w.B}), one acceptance",
                "t_verify_us": round(t_verify * 1e6, 1), "t_draft_windowed_us": round(t_draft * 1e6, 1),
                "t_accept_us": round(t_acc * 1e6, 1)}


def oracle_step_estimate(w, gamma, window, lens, n_q_v, n_layers):
    """The all-core estimate, plus the same verify sample on one core (the oracle's per-row
    loop parallelises over rows, so the one-core figure scales the verify part)."""
    smp = OracleSample(w, gamma, window, int(lens[0]), n_q_v, n_layers)
    res = smp.estimate()
    o = smp.oracle
    rows = [(0, i % smp.n_q_v, (i // smp.n_q_v) % w.G) for i in range(4)]
    t1 = smp._time(lambda: o.attention(smp.qv, smp.kv, smp.vv, [smp.Lv], o.MODE_CAUSAL, w.sm_scale,
                                       rows=rows, n_threads=1))
    t_verify_1 = t1 * smp.n_q_v * w.Hq * smp.n_layers * w.B / len(rows)
    res["value_1_core"] = round((t_verify_1 + res["t_draft_windowed_us"] * 1e-6 * smp.cores
                                 + res["t_accept_us"] * 1e-6) * 1e6, 1)
    res["value_1_core_is"] = ("verify from 4 rows on one core; windowed draft scaled from the all-core "
                              "time by the core count")
    return res


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from synthetic import configs

    w = configs.BY_NAME[args.workload]
    window = args.window or w.windows[0]
    n_q_v = w.tree_nodes or args.gamma + 1
    lens = [w.L] * w.B if not w.ragged[1] else [(w.ragged[0] + w.ragged[1]) // 2] * w.B
    sample = OracleSample(w, args.gamma, window, lens[0], n_q_v, w.verify_layers)
    for _ in range(args.warmup):
        sample.estimate()
    vals = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        r = sample.estimate()
        vals.append(r["value"])
    wall = time.perf_counter() - t0
    value = statistics.mean(vals)
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": "us/step",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(value / 1e3, 3), "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{w.name} (oracle sample per step, scaled)", "gamma": args.gamma,
                       "window": window},
            # the value is an estimate: each timed step runs a bounded sample of the decode step
            # on the oracle and scales it to the whole step, so value x steps exceeds the run time
            "estimate": True,
            "estimate_from": {"sample": r["sample"], "sample_wall_s_per_step": round(wall / max(1, args.steps), 3),
                              "scale": "verify rows x (query rows x layers / sampled rows); windowed draft "
                                       "of one kv head x kv heads"},
            "cpu_baseline": {"value": round(value, 1), "unit": "us/step", "cores": sample.cores,
                             "kind": "oracle", "sample": r["sample"], "estimate": True},
            "e2e": {"value": round(value, 1), "unit": "us/step", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "wall_s": round(wall, 2)}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
