"""Benchmark of the packed joint text+image attention forward on B200.

One step = one pass of the whole hot path over one synthetic pack: the
QK-RMSNorm + 2D-RoPE prologue and the block-diagonal attention, launched
through the C ABI on the current stream. Default workload: the
high-resolution pack (a 2048^2 sample of 16,896 tokens and a 4:1 sample of
4,352 tokens, 24 heads, head_dim 128, 1% of key rows x8).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl native|reference]

Under torchrun every rank runs its own replica of the workload (the pack's
(sample, head) units are independent; there is no collective on the data
path) and rank 0 prints one JSON line with the whole-job throughput.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "packed joint-attention TFLOP/s and tokens/s on 1 B200; % of dense-BF16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCE = os.path.join(ROOT, "packed_attention_b200", "csrc", "packed_attention.cuh")
# DRAM bytes (read + write) of one attention launch, from one ncu capture of
# the full workload (profiles/traffic_packed_attention_kernel_*.md), keyed by
# the kernel code it was taken on (the sha256 of the source with comments and
# blank lines removed, so that a comment edit keeps the figure): any other
# code reports null.
MEASURED_TRAFFIC = {
    ("7957cc8480356449", "hires_2048sq_4to1"): 395_591_936 + 110_353_664,
}


def kernel_code_sha(path=KERNEL_SOURCE):
    import hashlib
    import re
    with open(path) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    lines = [re.sub(r"//.*$", "", ln).rstrip() for ln in src.splitlines()]
    code = "\n".join(ln for ln in lines if ln.strip())
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def kernel_traffic(workload_name):
    return MEASURED_TRAFFIC.get((kernel_code_sha(), workload_name))


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="4",
                    help="workload index 0-4 (default 4), or 'all' for one report line per "
                         "workload (timing only, no e2e / CPU baseline)")
    ap.add_argument("--impl", choices=("native", "reference"), default="native")
    ap.add_argument("--block", action="store_true",
                    help="time the joint-attention sub-layer around the path (adaLN, "
                         "projections, attention, gate) of the chosen workload on one GPU")
    ap.add_argument("--train", action="store_true",
                    help="time the training pass (forward with log-normaliser + backward) of "
                         "the chosen workload on one GPU and print one JSON line")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-seconds", type=float, default=120.0,
                    help="CPU time the reference arm spends over all its steps")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def wait_first_row(self, limit_s: float = 5.0):
        """Block until nvidia-smi has written its first row (its start-up,
        which can take a second, is then over before any timed work)."""
        t0 = time.time()
        while self.proc is not None and time.time() - t0 < limit_s:
            if os.path.getsize(self.path) > 0 or self.proc.poll() is not None:
                return
            time.sleep(0.02)

    def stop(self):
        if self.proc is None:
            if self.path and os.path.exists(self.path):
                os.unlink(self.path)
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows
                                   if r[3].replace(".", "").isdigit()) if rows else None}


def oracle_sample_rows(w, rng, n_blocks, block=64):
    """Rows for a bounded oracle sample: blocks of `block` consecutive tokens of
    one head, drawn in proportion to the tokens of each sample. Returns the
    distinct flat rows (token * H + head) and their algorithmic FLOPs
    (4 * d * L of the row's sample each)."""
    lens = np.array(w.seg_lens)
    starts = np.concatenate([[0], np.cumsum(lens)])
    seg_of_token = np.repeat(np.arange(len(lens)), lens)
    rows = []
    for _ in range(n_blocks):
        s = int(rng.choice(len(lens), p=lens / lens.sum()))
        h = int(rng.integers(0, w.heads))
        b = int(rng.integers(0, max(1, lens[s] - block + 1)))
        toks = np.arange(starts[s] + b, starts[s] + min(b + block, lens[s]))
        rows.append(toks * w.heads + h)
    rows = np.unique(np.concatenate(rows))
    flops = int(4 * w.head_dim * lens[seg_of_token[rows // w.heads]].sum())
    return rows, flops


def cpu_model():
    """The host CPU's model name (first ``model name`` line of /proc/cpuinfo)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or None


def oracle_one_thread(seconds=4.0, seed=0):
    """The fp64 oracle on ONE host thread, on sampled query rows of the
    uniform 512^2 pack (4 x (128 text + 32x32), 24 heads, d = 128): per-core
    context for the all-core figure."""
    import oracle
    from packed_attention_b200.workloads import WORKLOADS, make_inputs
    w = WORKLOADS[1]
    inp = make_inputs(w)
    rng = np.random.default_rng(seed)
    rows, flops = oracle_sample_rows(w, rng, 1)
    t0 = time.perf_counter()
    oracle.joint_attn(inp["q"], inp["k"], inp["v"], inp, w.samples, eps=w.eps, rows=rows,
                      n_threads=1)
    dt = time.perf_counter() - t0
    n_blocks = max(1, int(seconds / max(dt, 1e-3)))
    rows, flops = oracle_sample_rows(w, rng, n_blocks)
    t0 = time.perf_counter()
    oracle.joint_attn(inp["q"], inp["k"], inp["v"], inp, w.samples, eps=w.eps, rows=rows,
                      n_threads=1)
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": 1, "workload": w.name,
            "sample": f"{len(rows)} (token, head) query rows in 64-token blocks, "
                      f"{flops / 1e9:.2f} GFLOP, {dt:.1f} s"}


def oracle_throughput(w, inp, seconds, seed=0):
    """The fp64 oracle, as it stands, on all host cores: TFLOP/s on sampled rows."""
    import oracle
    rng = np.random.default_rng(seed)
    cores = os.cpu_count() or 1
    rows, flops = oracle_sample_rows(w, rng, max(1, cores))
    t0 = time.perf_counter()
    oracle.joint_attn(inp["q"], inp["k"], inp["v"], inp, w.samples, eps=w.eps, rows=rows)
    dt = time.perf_counter() - t0
    n_blocks = max(cores, int(cores * seconds / max(dt, 1e-3)))
    rows, flops = oracle_sample_rows(w, rng, n_blocks)
    t0 = time.perf_counter()
    oracle.joint_attn(inp["q"], inp["k"], inp["v"], inp, w.samples, eps=w.eps, rows=rows)
    dt = time.perf_counter() - t0
    return flops / dt / 1e12, cores, f"{len(rows)} of {w.total_tokens * w.heads} (token, head) " \
        f"query rows in 64-token blocks, {flops / 1e9:.1f} GFLOP, {dt:.1f} s"


def max_over_ranks(values, world, device=None):
    """Element-wise max of per-rank timings (a list of floats) over all ranks."""
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_throughput(flops_per_replica, tokens_per_replica, world, steps, max_total_ms):
    """Replicas: every rank runs the whole workload; the job's throughput is all
    ranks' work divided by the slowest rank's time."""
    step_s = max_total_ms / steps / 1e3
    return flops_per_replica * world / step_s / 1e12, tokens_per_replica * world / step_s


def run_reference(args, w):
    """Reference arm: the fp64 oracle on host cores, one bounded sample per step."""
    from packed_attention_b200.workloads import make_inputs
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    inp = make_inputs(w)
    cores = os.cpu_count() or 1
    import oracle
    rng = np.random.default_rng(1234)
    budget = args.ref_seconds / max(1, args.steps + args.warmup)  # CPU seconds per step
    # calibrate block count per step
    rows, _ = oracle_sample_rows(w, rng, cores)
    t0 = time.perf_counter()
    oracle.joint_attn(inp["q"], inp["k"], inp["v"], inp, w.samples, eps=w.eps, rows=rows)
    per_block = (time.perf_counter() - t0) / cores
    n_blocks = max(1, int(budget / max(per_block, 1e-4)))
    n_blocks = min(n_blocks, 4 * (w.total_tokens * w.heads) // 64 + 1)  # enough to cover every row
    for _ in range(args.warmup):
        rows, _ = oracle_sample_rows(w, rng, n_blocks)
        oracle.joint_attn(inp["q"], inp["k"], inp["v"], inp, w.samples, eps=w.eps, rows=rows)
    total_flops, total_t = 0, 0.0
    for _ in range(args.steps):
        rows, fl = oracle_sample_rows(w, rng, n_blocks)
        t0 = time.perf_counter()
        oracle.joint_attn(inp["q"], inp["k"], inp["v"], inp, w.samples, eps=w.eps, rows=rows)
        total_t += time.perf_counter() - t0
        total_flops += fl
    value = total_flops / total_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_t / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "total_tokens": w.total_tokens, "heads": w.heads,
                   "head_dim": w.head_dim, "samples": [list(s) for s in w.samples]},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: {n_blocks} blocks of 64 query rows of one head, "
                                   f"fp64 oracle on {cores} threads"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _device_inputs(inp, dev, pa, torch):
    t = {n: torch.from_numpy(inp[n].view(np.int16)).view(torch.bfloat16).to(dev)
         for n in ("q", "k", "v")}
    t.update({n: torch.from_numpy(inp[n]).to(dev) for n in pa.GAMMA_NAMES})
    return t


def _median_step_ms(runs, steps, warmup):
    """Median device time (ms) per step of each stage. ``runs`` is a list of
    (tensors, plan, workspace, out, eps, frame_dims); one step launches every
    run's prologue and attention in order, with an event between stages."""
    import torch
    import packed_attention_b200 as pa
    stream = torch.cuda.current_stream()

    def launch(evs=None):
        for i, (t, plan, ws, out, eps, frame_dims) in enumerate(runs):
            pa.qk_prologue(t["q"], t["k"], t, plan, ws, eps=eps, frame_dims=frame_dims)
            if evs:
                evs[2 * i + 1].record(stream)
            pa.packed_attention(t["v"], plan, ws, out)
            if evs:
                evs[2 * i + 2].record(stream)

    for _ in range(max(3, warmup)):
        launch()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * len(runs) + 1)]
           for _ in range(steps)]
    for e in evs:
        e[0].record(stream)
        launch(e)
    torch.cuda.synchronize()
    if pa.device_error() != 0:
        raise RuntimeError("kernel reported a device-side error")
    med = lambda xs: sorted(xs)[len(xs) // 2]
    total = med([e[0].elapsed_time(e[-1]) for e in evs])
    pro = med([sum(e[2 * i].elapsed_time(e[2 * i + 1]) for i in range(len(runs))) for e in evs])
    att = med([sum(e[2 * i + 1].elapsed_time(e[2 * i + 2]) for i in range(len(runs))) for e in evs])
    return total, pro, att


def _prologue_ms_flushed(run, steps):
    """Median prologue time (ms) with L2 flushed before each launch: a
    256 MB buffer (twice the 126 MB L2) is written between launches, outside
    the timed interval."""
    import torch
    import packed_attention_b200 as pa
    t, plan, ws, out, eps, frame_dims = run
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=t["q"].device)
    stream = torch.cuda.current_stream()
    times = []
    for _ in range(steps):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        pa.qk_prologue(t["q"], t["k"], t, plan, ws, eps=eps, frame_dims=frame_dims)
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    return sorted(times)[len(times) // 2]


def _oracle_backward_rate(w, inp):
    """The fp64 oracle's forward + backward (oracle.attn_grad) timed on the
    host cores on one head of the pack's longest sample: its rate in the
    backward's FLOP convention (2.5x the forward's 4 * d * L^2)."""
    import oracle
    from packed_attention_b200 import synth
    L = max(w.seg_lens)
    i = w.seg_lens.index(L)
    start = sum(w.seg_lens[:i])
    sl = slice(start, start + L)
    q, k, v = (synth.bf16_bits_to_f64(inp[n][sl, :1]) for n in ("q", "k", "v"))
    dout = np.random.default_rng(0).standard_normal(q.shape)
    gam = {n: inp[n].astype(np.float64) for n in ("g_q_text", "g_q_img", "g_k_text", "g_k_img")}
    t0 = time.perf_counter()
    oracle.attn_grad(q, k, v, gam, [w.samples[i]], dout=dout, eps=w.eps,
                     frame_dims=w.rope_frame_dims)
    sec = time.perf_counter() - t0
    flops = 2.5 * 4.0 * w.head_dim * L * L
    return {"value": flops / sec / 1e12, "unit": "TFLOP/s", "cores": os.cpu_count(),
            "kind": "oracle", "sample": f"one head of the {L}-token sample, {sec:.1f} s"}


def training_line(w, key, steps, warmup, peaks, peak_src, with_oracle=False):
    """Device time of one training pass over the pack: the forward with its
    log-normaliser (``mf_joint_attn_fwd_lse``) and the backward
    (``mf_joint_attn_bwd``), medians over ``steps``. Backward FLOPs are counted
    as 2.5x the forward's: five products of the forward's size (S again, dP,
    dV, dK, dQ), the convention of FlashAttention's papers."""
    import torch
    import packed_attention_b200 as pa
    from packed_attention_b200.workloads import make_inputs
    dev = torch.device("cuda", torch.cuda.current_device())
    sustained = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    burst = float(peaks["bf16_tflops"])
    inp = make_inputs(w)
    t = _device_inputs(inp, dev, pa, torch)
    plan = pa.PackedPlan(w.samples, w.heads, w.head_dim, w.token_budget, device=dev)
    ws = plan.new_workspace()
    out = torch.empty_like(t["q"])
    lse = torch.empty(w.heads, w.total_tokens, dtype=torch.float32, device=dev)
    gen = torch.Generator(device=dev).manual_seed(w.seed)
    dout = torch.randn(out.shape, generator=gen, device=dev).to(torch.bfloat16)
    bws = torch.empty(pa.bwd_workspace_bytes(plan), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    fd = w.rope_frame_dims

    def fwd():
        pa.joint_attention_fwd_lse(t["q"], t["k"], t["v"], t, plan, eps=w.eps, frame_dims=fd,
                                   out=out, lse=lse, workspace=ws)

    def bwd():
        pa.joint_attention_bwd(t["q"], t["k"], t["v"], t, plan, out, lse, dout, eps=w.eps,
                               frame_dims=fd, workspace=bws)

    for _ in range(max(3, warmup)):
        fwd()
        bwd()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for e in evs:
        e[0].record(stream)
        fwd()
        e[1].record(stream)
        bwd()
        e[2].record(stream)
    torch.cuda.synchronize()
    if pa.device_error() != 0:
        raise RuntimeError("kernel reported a device-side error")
    f_ms = sorted(e[0].elapsed_time(e[1]) for e in evs)[steps // 2]
    b_ms = sorted(e[1].elapsed_time(e[2]) for e in evs)[steps // 2]
    oracle_line = _oracle_backward_rate(w, inp) if with_oracle else None
    return {"workload": w.name, "config": key, "phase": "training",
            "cpu_oracle_backward": oracle_line,
            "gflop_forward": w.flops / 1e9, "median_ms_forward_lse": f_ms,
            "median_ms_backward": b_ms, "tflops_forward": w.flops / (f_ms / 1e3) / 1e12,
            "tflops_backward": 2.5 * w.flops / (b_ms / 1e3) / 1e12,
            "frac_sustained_peak_backward": 2.5 * w.flops / (b_ms / 1e3) / 1e12 / sustained,
            "frac_burst_peak_backward": 2.5 * w.flops / (b_ms / 1e3) / 1e12 / burst,
            "tokens_per_s_training": w.total_tokens / ((f_ms + b_ms) / 1e3), "peaks": peak_src}


def block_line(w, key, steps, warmup, peaks, peak_src):
    """Device time of ``mf_attn_block_fwd`` on the pack with hidden size
    C = heads * head_dim and random weights. FLOPs: the two projections,
    2*T*C*3C + 2*T*C*C (each row computed once; a 128-row tile holding both
    modalities is computed twice and that repeat is not credited), plus the
    attention's 4*H*d*sum L^2."""
    import torch
    import packed_attention_b200 as pa
    from packed_attention_b200.workloads import make_block_inputs
    dev = torch.device("cuda", torch.cuda.current_device())
    inp = make_block_inputs(w)
    t = {}
    for k, v in inp.items():
        t[k] = (torch.from_numpy(v.view(np.int16)).view(torch.bfloat16) if v.dtype == np.uint16
                else torch.from_numpy(np.ascontiguousarray(v))).to(dev)
    plan = pa.PackedPlan(w.samples, w.heads, w.head_dim, w.token_budget, device=dev)
    ws = torch.empty(pa.block_workspace_bytes(plan), dtype=torch.uint8, device=dev)
    out = torch.empty_like(t["h"])
    stream = torch.cuda.current_stream()
    for _ in range(max(3, warmup)):
        pa.attn_block_fwd(t["h"], t, t, plan, out=out, workspace=ws)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for e0, e1 in evs:
        e0.record(stream)
        pa.attn_block_fwd(t["h"], t, t, plan, out=out, workspace=ws)
        e1.record(stream)
    torch.cuda.synchronize()
    if pa.device_error() != 0:
        raise RuntimeError("kernel reported a device-side error")
    ms = sorted(e0.elapsed_time(e1) for e0, e1 in evs)[steps // 2]
    T, C = w.total_tokens, w.heads * w.head_dim
    gemm = 8.0 * T * C * C
    return {"workload": w.name, "config": key, "phase": "attention sub-layer", "hidden": C,
            "median_ms": ms, "gflop_projections": gemm / 1e9, "gflop_attention": w.flops / 1e9,
            "tflops": (gemm + w.flops) / (ms / 1e3) / 1e12,
            "tokens_per_s": T / (ms / 1e3), "peaks": peak_src}


def report_all(args):
    """One JSON line per workload: device time of both stages, TFLOP/s, tokens/s,
    fraction of the measured peaks (single GPU). Then one line per packed-CFG
    pack: the pack in one forward against its two branches in two forwards."""
    import torch
    import packed_attention_b200 as pa
    from packed_attention_b200.workloads import CFG_PACKS, EXTRA_WORKLOADS, WORKLOADS, make_inputs
    peaks, peak_src = load_peaks()
    sustained = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    burst = float(peaks["bf16_tflops"])
    dev = torch.device("cuda", 0)

    def prepare(w, inp):
        t = _device_inputs(inp, dev, pa, torch)
        plan = pa.PackedPlan(w.samples, w.heads, w.head_dim, w.token_budget, device=dev)
        return (t, plan, plan.new_workspace(), torch.empty_like(t["q"]), w.eps, w.rope_frame_dims)

    for cfg, w in list(WORKLOADS.items()) + list(EXTRA_WORKLOADS.items()):
        run = prepare(w, make_inputs(w))
        _, pro, att = _median_step_ms([run], args.steps, args.warmup)
        pro_flushed = _prologue_ms_flushed(run, 20)
        T, H, d = w.total_tokens, w.heads, w.head_dim
        print(json.dumps({
            "workload": w.name, "config": cfg, "total_tokens": T, "heads": H, "head_dim": d,
            "gflop": w.flops / 1e9, "median_ms_prologue": pro, "median_ms_attention": att,
            "tflops_step": w.flops / ((pro + att) / 1e3) / 1e12,
            "tflops_attention": w.flops / (att / 1e3) / 1e12,
            "frac_sustained_peak_attention": w.flops / (att / 1e3) / 1e12 / sustained,
            "frac_burst_peak_attention": w.flops / (att / 1e3) / 1e12 / burst,
            "tokens_per_s": T / ((pro + att) / 1e3),
            "prologue_gbs": 8 * T * H * d / (pro / 1e3) / 1e9,
            "prologue_gbs_l2_flushed": 8 * T * H * d / (pro_flushed / 1e3) / 1e9,
            "rope_frame_dims": w.rope_frame_dims, "peaks": peak_src,
            "gpu": torch.cuda.get_device_name(dev)}), flush=True)

    # Training: forward with the log-normaliser, then the backward.
    for key, w in [(1, WORKLOADS[1]), (2, WORKLOADS[2]), (3, WORKLOADS[3]), (4, WORKLOADS[4]),
                   ("edit_1024sq_rope3d", EXTRA_WORKLOADS["edit_1024sq_rope3d"])]:
        print(json.dumps(training_line(w, key, max(5, args.steps // 5), args.warmup, peaks,
                                       peak_src, with_oracle=key in (1, 3))), flush=True)

    # The joint-attention sub-layer around the path (adaLN, per-modality QKV
    # projection with the QK-norm and rotation in its epilogue, attention,
    # per-modality output projection with gate and residual in its epilogue).
    from packed_attention_b200.workloads import make_block_inputs
    for key in (3, 4):
        w = WORKLOADS[key]
        print(json.dumps(block_line(w, key, max(5, args.steps // 5), args.warmup, peaks, peak_src)),
              flush=True)

    for name, cp in CFG_PACKS.items():
        w = cp.packed()
        inp = make_inputs(w)
        packed = _median_step_ms([prepare(w, inp)], args.steps, args.warmup)
        branches = []
        for b in ("cond", "uncond"):
            tok = cp.branch_tokens(b)
            sub = {n: np.ascontiguousarray(inp[n][tok]) for n in ("q", "k", "v")}
            sub.update({n: inp[n] for n in pa.GAMMA_NAMES})
            branches.append(prepare(cp.branch(b), sub))
        separate = _median_step_ms(branches, args.steps, args.warmup)
        print(json.dumps({
            "workload": name, "total_tokens": w.total_tokens, "heads": w.heads,
            "head_dim": w.head_dim, "gflop": w.flops / 1e9,
            "packed_ms": {"step": packed[0], "prologue": packed[1], "attention": packed[2]},
            "two_calls_ms": {"step": separate[0], "prologue": separate[1],
                             "attention": separate[2]},
            "speedup_step": separate[0] / packed[0],
            "speedup_attention": separate[2] / packed[2],
            "tflops_attention_packed": w.flops / (packed[2] / 1e3) / 1e12,
            "peaks": peak_src}), flush=True)


def main():
    args = parse_args()
    from packed_attention_b200.workloads import WORKLOADS, make_inputs
    if args.config == "all":
        report_all(args)
        return
    w = WORKLOADS[int(args.config)]
    if args.block:
        import torch
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        peaks, peak_src = load_peaks()
        print(json.dumps(block_line(w, int(args.config), args.steps, args.warmup, peaks, peak_src)),
              flush=True)
        return
    if args.train:
        import torch
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        peaks, peak_src = load_peaks()
        print(json.dumps(training_line(w, int(args.config), args.steps, args.warmup, peaks,
                                       peak_src)), flush=True)
        return
    if args.impl == "reference":
        run_reference(args, w)
        return

    import torch
    import torch.distributed as dist

    import packed_attention_b200 as pa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    inp = make_inputs(w)
    T, H, d = w.total_tokens, w.heads, w.head_dim
    t = {n: torch.from_numpy(inp[n].view(np.int16)).view(torch.bfloat16).to(dev)
         for n in ("q", "k", "v")}
    t.update({n: torch.from_numpy(inp[n]).to(dev) for n in pa.GAMMA_NAMES})
    plan = pa.PackedPlan(w.samples, H, d, w.token_budget, device=dev)
    ws = plan.new_workspace()
    out = torch.empty_like(t["q"])
    stream = torch.cuda.current_stream()

    def step(e0=None, e1=None, e2=None):
        if e0 is not None:
            e0.record(stream)
        pa.qk_prologue(t["q"], t["k"], t, plan, ws, eps=w.eps)
        if e1 is not None:
            e1.record(stream)
        pa.packed_attention(t["v"], plan, ws, out)
        if e2 is not None:
            e2.record(stream)

    # The clock sampler is up (its first row written) before the warm-up, so
    # that its start-up does not overlap the timed region and the timed
    # region follows the warm-up with no idle gap in which the clocks could
    # drop.
    sampler = ClockSampler(local_rank) if rank == 0 else None
    if sampler:
        sampler.start()
        sampler.wait_first_row()
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if pa.device_error() != 0:
        raise RuntimeError("kernel reported a device-side error during warm-up")

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(K):
        step(*evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop() if sampler else None
    if pa.device_error() != 0:
        raise RuntimeError("kernel reported a device-side error in the timed region")

    total_ms = start.elapsed_time(end)
    pro_steps = [e[0].elapsed_time(e[1]) for e in evs]
    att_steps = [e[1].elapsed_time(e[2]) for e in evs]
    step_steps = [e[0].elapsed_time(e[2]) for e in evs]
    pro_ms = sum(pro_steps) / K
    att_ms = sum(att_steps) / K
    per_step = [statistics.median(step_steps), min(step_steps), max(step_steps),
                statistics.median(pro_steps), min(pro_steps), statistics.median(att_steps),
                min(att_steps), max(att_steps)]
    total_ms, pro_ms, att_ms, *per_step = max_over_ranks(
        [total_ms, pro_ms, att_ms, *per_step], world, dev)

    # ---- end to end through the public API on host buffers (copies timed) ----
    # Every step copies its inputs from pinned host memory and reads its
    # result back; HostPipeline overlaps step n's upload with step n-1's
    # compute and step n-2's read-back (three streams, two buffer sets).
    host = {n: t[n].cpu().pin_memory() for n in ("q", "k", "v", *pa.GAMMA_NAMES)}
    out_host = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    pipe = pa.HostPipeline(plan, eps=w.eps)
    for _ in range(3):
        pipe.submit(host["q"], host["k"], host["v"], host, out_host)
    pipe.synchronize()
    torch.cuda.synchronize()
    e_s, e_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e_s.record(pipe.s_in)
    for _ in range(args.e2e_steps):
        pipe.submit(host["q"], host["k"], host["v"], host, out_host)
    e_e.record(pipe.s_out)
    pipe.synchronize()
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks([e_s.elapsed_time(e_e) / args.e2e_steps], world, dev)[0]

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks, peak_src = load_peaks()
    flops = w.flops
    value, tokens_per_s = whole_job_throughput(flops, T, world, K, total_ms)
    att_tflops = flops / (att_ms / 1e3) / 1e12
    peak_sus = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    peak_burst = float(peaks["bf16_tflops"])
    # The burst peak (a GEMM timed alone) applies to a timed region that is
    # over before the 1 kW power cap pulls the clock down; the sustained one
    # (a seconds-long GEMM loop) to a region of a second or more.
    timed_s = total_ms / 1e3
    long_region = timed_s >= 1.0
    peak = peak_sus if long_region else peak_burst
    peak_kind = (f"{peak_src} bf16 dense, " + ("sustained (timed region >= 1 s)" if long_region
                                                else "burst (timed region < 1 s)"))
    sm_mhz = clocks.get("sm_mhz") if clocks else None
    pro_bytes = 8 * T * H * d
    pro_gbs = pro_bytes / (pro_ms / 1e3) / 1e9
    hbm = float(peaks["hbm_gbs"])

    cpu = None
    if not args.no_cpu_baseline and world == 1:
        v_cpu, cores, sample = oracle_throughput(w, inp, args.cpu_seconds)
        cpu = {"value": v_cpu, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
               "sample": sample, "cpu_model": cpu_model(),
               "one_thread": oracle_one_thread()}

    h2d = sum(host[n].numel() * host[n].element_size() for n in host)
    d2h = out_host.numel() * out_host.element_size()
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": w.name, "samples": [list(s) for s in w.samples], "total_tokens": T,
            "heads": H, "head_dim": d, "sum_L2": w.sum_L2, "gflop_per_step": flops / 1e9,
            "parallelism": "independent replicas" if world > 1 else "single gpu",
            "l2": f"inputs q,k,v = {3 * T * H * d * 2 / 1e6:.0f} MB > 126 MB L2 (not flushed)",
        },
        "tokens_per_s": tokens_per_s,
        "pct_of_peak": 100.0 * value / world / peak,
        "per_step_ms": {"step_median": per_step[0], "step_min": per_step[1],
                        "step_max": per_step[2], "prologue_median": per_step[3],
                        "prologue_min": per_step[4], "attention_median": per_step[5],
                        "attention_min": per_step[6], "attention_max": per_step[7]},
        "roofline": {
            "kernel": "packed_attention_kernel", "bound": "tensor", "achieved": att_tflops,
            "peak": peak, "unit": "TFLOP/s", "frac": att_tflops / peak, "peak_kind": peak_kind,
            "frac_of_burst_peak": att_tflops / peak_burst,
            "frac_of_sustained_peak": att_tflops / peak_sus, "traffic": kernel_traffic(w.name),
            "algorithmic_flops_per_launch": flops, "avg_launch_ms": att_ms,
            "timed_region_s": timed_s, "sm_mhz_median": sm_mhz,
            # launch time x sampled SM clock: kilocycles per launch, comparable across clocks
            "avg_launch_kcycles": att_ms * sm_mhz if sm_mhz else None,
        },
        "prologue": {
            "kernel": "qk_prologue_kernel", "bound": "hbm", "achieved": pro_gbs, "peak": hbm,
            "unit": "GB/s", "frac": pro_gbs / hbm, "algorithmic_bytes_per_launch": pro_bytes,
            "avg_launch_ms": pro_ms,
        },
        "cpu_baseline": cpu,
        "e2e": {"value": flops * world / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "api": "HostPipeline: per-step upload, forward and read-back overlapped "
                       "across steps on three streams"},
        "gpu_launches": 2 * K,
        "clocks": clocks,
        "gpu": torch.cuda.get_device_name(dev),
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
