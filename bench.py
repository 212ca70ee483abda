"""Benchmark of the fine-grained FP8 linear hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload llama3_prefill|deepseek_mlp|llama3_decode|sweep|deepseek_moe]

One step (default workload, Llama-3-8B MLP prefill, M = 4096 tokens):
    quant_act(X1 [4096, 4096])   -> block_linear vs W_gate_up [28672, 4096]
    quant_act(X2 [4096, 14336])  -> block_linear vs W_down    [4096, 14336]
X ~ Student-t(df=4) with 0.5% of channels x50, W ~ N(0, 0.02), weights
quantized once before timing (load time).  Inputs of a step (~330 MB) are
larger than the 126 MB L2, so no flush is needed between steps.

Prints ONE JSON line (rank 0).  `value` is whole-job TFLOP/s (2 M N K per
linear, all ranks) over the device-timed K steps (CUDA events, max over
ranks).  `e2e` repeats the measurement through the public API with the
inputs copied from pinned host memory and the outputs copied back inside
every step, double-buffered (step k + 1's copy in and step k - 1's copy out
overlap step k's kernels).  `roofline` covers the dominant kernel (the block-scaled GEMM;
for the decode workload the weight-streaming decode kernel, against HBM)
against the measured peaks in MEASURED_PEAKS.json, from a second pass with
events around every kernel.  `fused` times fp8_block_linear_fused on the
same inputs with its workspace (codes staged in it) and, as `in_kernel`,
without one (the quantization inside the GEMM's tiles), and checks each
output equals the two-call path bit for bit.  `ue8m0` and `fp8r` time the
two other scale formats on the same inputs (power-of-two scales on the
tensor core's block-scaled MMA; one fp32 scale per activation row and weight
row), each with its GEMM's roofline and an oracle check of sampled rows.
`cpu_baseline` and
`--impl reference` time the plain CPU oracle on a bounded row sample.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "block-scaled FP8 linear TFLOP/s (% FP8 peak); act-quant GB/s (% HBM peak)"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FP8_OVER_BF16 = 2.0          # nominal dense ratio, 4.5 / 2.25 PFLOP/s


# ----------------------------------------------------------------- workloads

def workload_linears(name: str):
    """[(label, x_bits [M,K], w_bits [N,K])] for one step of the workload."""
    if name == "llama3_prefill":
        return [(f"{n}", *wl.llama3_prefill(n)) for n in ("gate_up", "down")]
    if name == "deepseek_mlp":
        return [(f"{n}", *wl.deepseek_mlp(n)) for n in ("up", "down")]
    if name == "llama3_decode":
        out = []
        for M in wl.DECODE_M:
            for n in ("qo", "kv", "gate_up", "down"):
                out.append((f"{n}_M{M}", *wl.llama3_decode(M, n)))
        return out
    if name == "sweep":
        w = wl.sweep_w()
        return [(f"M{M}", wl.sweep_x(M), w) for M in wl.SWEEP_M]
    raise ValueError(name)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


KERNEL_SOURCES = {
    "gemm_prefill_kernel": ("gemm.cu", "ptx_sm100.cuh", "quant_math.cuh"),
    "gemm_ue8m0_kernel": ("gemm_ue8m0.cu", "ptx_sm100.cuh"),
    "gemm_ue8m0_pair_kernel": ("gemm_ue8m0_pair.cu", "ptx_sm100.cuh"),
    "gemm_rowwise_kernel": ("gemm_rowwise.cu", "ptx_sm100.cuh"),
    "gemm_rowwise_pair_kernel": ("gemm_rowwise.cu", "ptx_sm100.cuh"),
}


def gemm_source_sha(kernel: str = "gemm_prefill_kernel") -> str:
    """Hash of the sources a kernel is compiled from (its traffic entry in
    profiles/traffic.txt is valid only while this matches)."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(ROOT, "fine_grained_block_token_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """dram bytes per launch from profiles/traffic.txt if the entry was taken
    on the current kernel source, else None."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    sha = gemm_source_sha(kernel)
    for line in open(p):
        if line.startswith("#") or not line.strip():
            continue
        kv = dict(tok.split("=", 1) for tok in line.split() if "=" in tok)
        if kv.get("kernel") == kernel and kv.get("workload") == workload and kv.get("source_sha") == sha:
            return float(kv["dram_bytes_per_launch"])
    return None


# ------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.lines = []

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- CPU side

def cpu_prepare(lins, rows_per_linear: int, seed: int = 0):
    """Load-time work of the CPU oracle: quantize the weights (not timed) and
    pick the row sample of every linear."""
    import oracle
    prepared = []
    for i, (label, xb, wb) in enumerate(lins):
        qw, sw = oracle.quant_weight(wb)
        g = np.random.default_rng([seed, i])
        M = xb.shape[0]
        rows = np.sort(g.choice(M, min(rows_per_linear, M), replace=False))
        prepared.append((label, rows, np.ascontiguousarray(xb[rows]), qw, sw))
    return prepared


def cpu_step(prepared):
    """One timed CPU step: the oracle's activation quantization of the sampled
    rows and its fp64 block-scaled GEMM for them (all N columns).
    Returns (seconds, flops, threads, {label: (rows, R)})."""
    import oracle
    threads = os.cpu_count() or 1
    out = {}
    t0 = time.perf_counter()
    flops = 0
    for label, rows, xs, qw, sw in prepared:
        qa, sa = oracle.quant_act(xs, nthreads=threads)
        out[label] = (rows, oracle.block_linear(qa, sa, qw, sw, nthreads=threads))
        flops += 2 * xs.shape[0] * qw.shape[0] * qw.shape[1]
    return time.perf_counter() - t0, flops, threads, out


def sample_desc(prepared):
    n = len(prepared[0][1]) if prepared else 0
    return (f"{n} random rows per linear ({', '.join(p[0] for p in prepared)}), all N columns; "
            "activation quant + fp64 GEMM of those rows; weights quantized before timing")


def pipelined_e2e(items, host_x, host_y, compute, steps, warmup, barrier, dev):
    """End to end through the public API with every step's input copied in
    from pinned host memory and its output copied back, double-buffered the
    way a serving loop overlaps them: step k's host-to-device copy runs on
    one stream, its kernels on the launching stream and its device-to-host
    copy on a third, with two device buffers per input and output so that
    step k + 1's input copy and step k - 1's output copy overlap step k's
    kernels (PCIe copies in both directions at once).  compute(xs, ys)
    launches one step's kernels reading xs and writing ys.  Returns the ms
    from the first copy in to the last copy out."""
    import torch
    cur = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    xs = [[it["x"], torch.empty_like(it["x"])] for it in items]
    ys = [[it["y"], torch.empty_like(it["y"])] for it in items]
    ev = lambda: torch.cuda.Event()
    copied, computed, drained = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    for e in computed + drained:
        e.record(cur)

    def step(k):
        b = k & 1
        s_in.wait_event(computed[b])           # the kernels that read this buffer are done
        with torch.cuda.stream(s_in):
            for x2, hx in zip(xs, host_x):
                x2[b].copy_(hx, non_blocking=True)
        copied[b].record(s_in)
        cur.wait_event(copied[b])
        cur.wait_event(drained[b])             # the copy out of this output buffer is done
        compute([x2[b] for x2 in xs], [y2[b] for y2 in ys])
        computed[b].record(cur)
        s_out.wait_event(computed[b])
        with torch.cuda.stream(s_out):
            for y2, hy in zip(ys, host_y):
                hy.copy_(y2[b], non_blocking=True)
        drained[b].record(s_out)

    for k in range(warmup):
        step(k)
    torch.cuda.synchronize(dev)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    barrier()
    a.record(cur)
    s_in.wait_stream(cur)
    s_out.wait_stream(cur)
    for k in range(steps):
        step(k)
    cur.wait_stream(s_in)
    cur.wait_stream(s_out)
    b.record(cur)
    barrier()
    return a.elapsed_time(b)


def decode_workload(name: str) -> bool:
    return name == "llama3_decode"


def variant_parity(name: str, v_items, lins, rows_per_linear: int, dev):
    """A variant leg's output on a few sampled rows against the oracle, which
    quantizes those rows of the same input bits itself (weights: the GPU's
    codes and scales, held bit-exact to the oracle by the test suite)."""
    import torch
    import oracle
    worst = 0.0
    for u, (label, xb, _) in zip(v_items, lins):
        M = xb.shape[0]
        rows = np.unique(np.linspace(0, M - 1, rows_per_linear).astype(np.int64))
        if name == "ue8m0":
            per_row = [oracle.quant_act_ue8m0_rows(xb, int(r), int(r) + 1) for r in rows]
        else:
            per_row = [oracle.quant_rowwise(xb, int(r), int(r) + 1) for r in rows]
        qa = np.concatenate([q for q, _ in per_row])
        sa = np.concatenate([c for _, c in per_row])
        qw = u["q_w"].view(torch.uint8).cpu().numpy()
        if name == "ue8m0":
            sw = u["s_w"].view(torch.uint8).cpu().numpy()
            R = oracle.block_linear_ue8m0(qa, sa, qw, sw, nthreads=os.cpu_count() or 1)
        else:
            sw = u["s_w"].cpu().numpy()
            R = oracle.linear_rowwise(qa, sa, qw, sw)
        Y = u["y"][torch.as_tensor(rows, device=dev)].float().cpu().numpy()
        worst = max(worst, within_tolerance(Y, R))
    return {"rows_per_linear": rows_per_linear, "within_tolerance": worst <= 1.0,
            "worst_bound_ratio": worst}


def within_tolerance(y, R):
    """GEMM tolerance: |y-R| <= 4e-3|R| + 1e-2 rms(R) pointwise.
    Returns the worst ratio of |y-R| to its bound (<= 1 passes)."""
    y = np.asarray(y, np.float64)
    R = np.asarray(R, np.float64)
    rms = float(np.sqrt(np.mean(R * R)))
    lim = 4e-3 * np.abs(R) + 1e-2 * rms
    return float(np.max(np.abs(y - R) / np.maximum(lim, 1e-300)))


# ------------------------------------------------------ multi-process host

def rank_info():
    """(world, rank, local_rank) from the torchrun environment (1, 0, 0 alone)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(values, device, world: int):
    """Element-wise maximum of `values` over all ranks (device-timed numbers
    are reported as the slowest rank's).  `device` is where the collective
    runs: the GPU under NCCL, the CPU under gloo."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_rate(world: int, work_per_step: float, steps: int, elapsed_ms: float) -> float:
    """Replicas: every rank runs the same steps, so the job does world x the
    work of one rank in the slowest rank's time (weak scaling)."""
    return world * work_per_step * steps / (elapsed_ms * 1e-3)


def run_reference(args):
    """The oracle, as it stands, on the host cores: one bounded row sample of
    the workload per step.  Under torchrun only rank 0 works."""
    _, rank, _ = rank_info()
    if rank != 0:
        return 0
    if args.workload == "deepseek_moe":
        return run_reference_moe(args)
    lins = workload_linears(args.workload)
    prepared = cpu_prepare(lins, args.ref_rows)
    for _ in range(args.warmup):
        cpu_step(prepared)
    tot_t, tot_f, thr = 0.0, 0, 1
    for _ in range(args.steps):
        t, f, thr, _ = cpu_step(prepared)
        tot_t += t
        tot_f += f
    desc = sample_desc(prepared)
    value = tot_f / tot_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot_t / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "sample": desc},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": thr, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ------------------------------------------------------------ MoE experts

def run_reference_moe(args):
    """Reference arm on the MoE workload: the oracle on `ref_rows` routed rows
    per expert linear, taken from the two largest experts (whose weights the
    oracle quantizes before timing).  The weights are drawn by torch's CPU
    generator (same distribution and seed as the GPU arm's, another stream)."""
    import torch
    import oracle
    g = np.random.default_rng(0)
    prepared = []
    for name in ("up", "down"):
        xb, off = wl.deepseek_moe(name)
        N, K = wl.MOE_LINEARS[name]
        E = wl.MOE_EXPERTS
        big = np.argsort(np.diff(off))[-2:]
        w = wl.deepseek_moe_weights(name, "cpu").view(torch.int16).numpy().view(np.uint16)
        q_w = np.zeros((E, N, K), np.uint8)
        s_w = np.full((E, N // 128, K // 128), 127, np.uint8)
        for e in big:
            q_w[e], s_w[e] = oracle.quant_weight_ue8m0(np.ascontiguousarray(w[e * N:(e + 1) * N]))
        cand = np.concatenate([np.arange(off[e], off[e + 1]) for e in big])
        rows = np.sort(g.choice(cand, min(args.ref_rows, len(cand)), replace=False))
        prepared.append((name, xb, q_w, s_w, off, rows))
    for _ in range(args.warmup):
        for name, xb, q_w, s_w, off, rows in prepared:
            moe_oracle_rows(xb, q_w, s_w, off, rows)
    tot_t, tot_f = 0.0, 0.0
    for _ in range(args.steps):
        for name, xb, q_w, s_w, off, rows in prepared:
            t, f, _ = moe_oracle_rows(xb, q_w, s_w, off, rows)
            tot_t += t
            tot_f += f
    value = tot_f / tot_t / 1e12
    desc = (f"{args.ref_rows} routed rows of the two largest experts per expert linear (up, down): "
            "ue8m0 activation quant + fp64 grouped GEMM of those rows; weights quantized before timing")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot_t / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "sample": desc},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": os.cpu_count() or 1,
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def moe_oracle_rows(xb, q_w, s_w, off, rows):
    """Oracle result of the sampled rows of one grouped linear: the oracle
    quantizes those rows of X itself; the weights are the GPU's codes (held
    bit-exact to the oracle by the tests).  Returns (seconds, flops, R)."""
    import oracle
    t0 = time.perf_counter()
    per_row = [oracle.quant_act_ue8m0_rows(xb, int(r), int(r) + 1) for r in rows]
    M = xb.shape[0]
    qa = np.zeros((M, xb.shape[1]), np.uint8)
    ca = np.full((M, xb.shape[1] // 128), 127, np.uint8)
    for r, (q, c) in zip(rows, per_row):
        qa[r], ca[r] = q[0], c[0]
    R = oracle.grouped_linear_ue8m0(qa, ca, q_w, s_w, off, rows=rows, nthreads=os.cpu_count() or 1)
    t = time.perf_counter() - t0
    return t, 2.0 * len(rows) * q_w.shape[1] * q_w.shape[2], R[rows]


def moe_items(fp8, dev):
    """The DeepSeek-V3 expert linears (up, down): routed activations, the
    experts' UE8M0-quantized weights, outputs and the CTA-pair workspace."""
    import torch
    items = []
    for name in ("up", "down"):
        xb, off = wl.deepseek_moe(name)
        N, K = wl.MOE_LINEARS[name]
        E = wl.MOE_EXPERTS
        w = wl.deepseek_moe_weights(name, dev)
        q_w, s_w = fp8.quant_weight_ue8m0(w)
        del w
        M = xb.shape[0]
        items.append(dict(label=name, xb=xb, x=wl.to_torch_bf16(xb).to(dev), off_np=off,
                          off=torch.from_numpy(off).to(dev), q_w=q_w.view(E, N, K),
                          s_w=s_w.view(E, N // 128, K // 128),
                          q_a=torch.empty((M, K), dtype=torch.float8_e4m3fn, device=dev),
                          s_a=torch.empty((M, K // 128), dtype=torch.float8_e8m0fnu, device=dev),
                          y=torch.empty((M, N), dtype=torch.bfloat16, device=dev), M=M, N=N, K=K))
        # the CTA-pair schedule's packed scale factors (allocated once, reused)
        items[-1]["ws"] = torch.empty(max(fp8.grouped_ue8m0_workspace_bytes(M, N, K, E), 16),
                                      dtype=torch.uint8, device=dev)
    torch.cuda.synchronize(dev)
    return items


def moe_step_fn(fp8, items):
    """One MoE step: per expert linear, the ue8m0 activation quantization of
    the routed rows and the grouped GEMM (events around each GEMM if given)."""
    def step(ev=None):
        for i, it in enumerate(items):
            fp8.quant_act_ue8m0(it["x"], it["q_a"], it["s_a"])
            if ev is not None:
                ev[2 * i].record()
            fp8.grouped_linear_ue8m0(it["q_a"], it["s_a"], it["q_w"], it["s_w"], it["off"], it["y"],
                                     workspace=it["ws"])
            if ev is not None:
                ev[2 * i + 1].record()
    return step


def moe_oracle_check(items, rows_per_linear, seed=0):
    """The oracle on sampled routed rows of each expert linear (CPU baseline
    and parity check)."""
    import torch
    t_tot, f_tot, worst = 0.0, 0.0, 0.0
    g = np.random.default_rng(seed)
    for it in items:
        rows = np.sort(g.choice(it["M"], rows_per_linear, replace=False))
        qw = it["q_w"].view(torch.uint8).cpu().numpy()
        sw = it["s_w"].view(torch.uint8).cpu().numpy()
        t, f, R = moe_oracle_rows(it["xb"], qw, sw, it["off_np"], rows)
        t_tot += t
        f_tot += f
        Y = it["y"][torch.as_tensor(rows, device=it["y"].device)].float().cpu().numpy()
        worst = max(worst, within_tolerance(Y, R))
    cpu = {"value": f_tot / t_tot / 1e12, "unit": "TFLOP/s", "cores": os.cpu_count() or 1,
           "kind": "oracle", "seconds": t_tot,
           "sample": f"{rows_per_linear} random routed rows per expert linear (up, down): "
                     "ue8m0 activation quant + fp64 grouped GEMM of those rows, all N columns"}
    parity = {"rows_per_linear": rows_per_linear, "within_tolerance": worst <= 1.0,
              "worst_bound_ratio": worst}
    return cpu, parity


def leg_moe(fp8, dev, barrier, args):
    """The grouped MoE step as a leg of the default run: graph-replayed
    steps, then a pass with events around the grouped GEMMs."""
    import torch
    items = moe_items(fp8, dev)
    step = moe_step_fn(fp8, items)
    for _ in range(min(args.warmup, 3)):
        step()
    g = capture_graph(step, dev)
    ms = timed_replays(g.replay, args.steps, barrier)
    del g
    n = len(items)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * n)] for _ in range(args.steps)]
    barrier()
    for k in range(args.steps):
        step(evs[k])
    barrier()
    gemm_ms = sum(e[2 * i].elapsed_time(e[2 * i + 1]) for e in evs for i in range(n))
    fp8.check()
    flops = sum(2 * it["M"] * it["N"] * it["K"] for it in items)
    return items, dict(ms=ms, gemm_ms=gemm_ms, flops=flops)


def moe_json(leg, world, args, cpu_ok, fp8_peak, peak_src):
    items, d = leg
    n = len(items)
    gemm_tf = d["flops"] * args.steps / (d["gemm_ms"] * 1e-3) / 1e12
    cpu, parity = moe_oracle_check(items, 4) if cpu_ok else (None, None)
    return {"deepseek_moe": {
        "value": whole_job_rate(world, d["flops"], args.steps, d["ms"]) / 1e12, "unit": "TFLOP/s",
        "ms_per_step": d["ms"] / args.steps,
        "config": {"workload": "deepseek_moe", "experts": wl.MOE_EXPERTS, "routed_rows": wl.MOE_ROWS,
                   "linears": {it["label"]: [it["M"], it["N"], it["K"]] for it in items},
                   "l2": "no flush: the step's expert weights (470 + 235 MB) exceed the 126 MB L2"},
        "gemm": {"kernel": "gemm_ue8m0_pair_kernel (grouped; timed with its two scale-pack kernels)",
                 "achieved": gemm_tf, "peak": fp8_peak, "unit": "TFLOP/s", "frac": gemm_tf / fp8_peak,
                 "ms_per_launch": d["gemm_ms"] / (args.steps * n),
                 "traffic": recorded_traffic("gemm_ue8m0_pair_kernel", "deepseek_moe")},
        "cpu_baseline": cpu, "parity": parity}}


def run_moe(args):
    """Grouped (MoE expert) UE8M0 linears: one step = per expert linear (up,
    down), ue8m0 activation quantization of the routed rows + the grouped
    GEMM over the experts' segments."""
    import torch
    import torch.distributed as dist

    import fine_grained_block_token_b200 as fp8

    world, rank, local = rank_info()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    hbm_peak, bf16_peak, peak_src = peaks()
    fp8_peak = bf16_peak * FP8_OVER_BF16
    items = moe_items(fp8, dev)
    flops_step = sum(2 * it["M"] * it["N"] * it["K"] for it in items)
    n = len(items)
    step = moe_step_fn(fp8, items)

    for _ in range(args.warmup):
        step()
    fp8.check()
    graph = None
    if not args.eager:
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            step()
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        torch.cuda.synchronize(dev)
    run_step = (lambda: graph.replay()) if graph is not None else step
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.3)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    a.record()
    for _ in range(args.steps):
        run_step()
    b.record()
    barrier()
    elapsed_ms = a.elapsed_time(b)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * n)] for _ in range(args.steps)]
    barrier()
    for k in range(args.steps):
        step(evs[k])
    barrier()
    gemm_ms = sum(e[2 * i].elapsed_time(e[2 * i + 1]) for e in evs for i in range(n))
    fp8.check()
    # end to end: X in from pinned host memory, Y back, every step
    host_x = [wl.to_torch_bf16(it["xb"]).pin_memory() for it in items]
    host_y = [torch.empty((it["M"], it["N"]), dtype=torch.bfloat16).pin_memory() for it in items]

    def e2e_compute(xs, ys):
        for it, x, y in zip(items, xs, ys):
            fp8.quant_act_ue8m0(x, it["q_a"], it["s_a"])
            fp8.grouped_linear_ue8m0(it["q_a"], it["s_a"], it["q_w"], it["s_w"], it["off"], y,
                                     workspace=it["ws"])

    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    e2e_ms = pipelined_e2e(items, host_x, host_y, e2e_compute, e2e_steps, min(args.warmup, 3),
                           barrier, dev)
    sampler.stop()
    fp8.check()
    elapsed_ms, gemm_ms, e2e_ms = max_over_ranks([elapsed_ms, gemm_ms, e2e_ms], dev, world)
    gemm_tf = flops_step * args.steps / (gemm_ms * 1e-3) / 1e12
    if rank == 0:
        cpu = parity = None
        if world == 1 and not args.no_cpu:
            cpu, parity = moe_oracle_check(items, args.cpu_rows)
        line = {
            "metric": METRIC, "value": whole_job_rate(world, flops_step, args.steps, elapsed_ms) / 1e12,
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3 (ue8m0 scales)", "data": "synthetic",
            "config": {"workload": "deepseek_moe", "experts": wl.MOE_EXPERTS, "routed_rows": wl.MOE_ROWS,
                       "linears": {it["label"]: [it["M"], it["N"], it["K"]] for it in items},
                       "segment_rows": {it["label"]: np.diff(it["off_np"]).tolist() for it in items},
                       "l2": "no flush: the step's expert weights (470 + 235 MB) exceed the 126 MB L2",
                       "parallelism": f"replicas x{world} (no data-path collective)",
                       "launch": "eager" if args.eager else "cuda_graph (one step captured, replayed)"},
            "roofline": {"bound": "tensor", "achieved": gemm_tf, "peak": fp8_peak, "unit": "TFLOP/s",
                         "frac": gemm_tf / fp8_peak,
                         "traffic": recorded_traffic("gemm_ue8m0_pair_kernel", "deepseek_moe"),
                         "kernel": "gemm_ue8m0_pair_kernel (grouped; timed with its two scale-pack kernels)",
                         "peak_source": f"{peak_src} bf16 burst x {FP8_OVER_BF16} (nominal fp8/bf16)",
                         "ms_per_launch": gemm_ms / (args.steps * n)},
            "e2e": {"value": whole_job_rate(world, flops_step, e2e_steps, e2e_ms) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": sum(t.numel() * 2 for t in host_x),
                    "d2h_bytes_per_step": sum(t.numel() * 2 for t in host_y), "steps": e2e_steps,
                    "schedule": "double-buffered: copy in, kernels, copy out on three streams"},
            # per linear: the quantizer, two scale-pack kernels and the GEMM
            "gpu_launches": 4 * n * args.steps,
            "clocks": sampler.summary(),
            "cpu_baseline": cpu,
            "parity": parity,
        }
        print(json.dumps(line))
    del graph
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ----------------------------------------------------- per-config legs
#
# The default run reports every workload of the build on the same JSON line:
# besides the headline prefill step, `decode` (the 16 Llama-3-8B decode
# linears and a whole layer per token count), `deepseek_mlp`, `sweep`,
# `tiny` and `deepseek_moe` (the grouped expert linears).  Each leg times on the device (CUDA events around CUDA-graph
# replays, max over ranks) and carries its roofline fraction, an oracle check
# of sampled outputs and an oracle CPU baseline.
L2_BYTES = 126e6


def capture_graph(fn, dev):
    """CUDA graph of fn() (one warm-up run on a side stream first)."""
    import torch
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize(dev)
    return g


def timed_replays(run, reps, barrier, warm=2):
    """Device ms of `reps` calls of run() between two events (after `warm`
    untimed calls), with a barrier + synchronize on both sides."""
    import torch
    for _ in range(warm):
        run()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    a.record()
    for _ in range(reps):
        run()
    b.record()
    barrier()
    return a.elapsed_time(b)


def copies_for(bytes_per_launch: float) -> int:
    """Distinct buffer copies a rotation needs so that every launch reads
    operands that left the L2 (the rotation moves >= 2.5 x L2)."""
    return max(2, int(np.ceil(2.5 * L2_BYTES / bytes_per_launch)))


def decode_bytes(M, N, K):
    """Algorithmic bytes of one decode linear: W codes + block scales, X codes
    + group scales, bf16 Y."""
    return N * K + (N // 128) * (K // 128) * 4 + M * K + M * (K // 128) * 4 + 2 * M * N


def leg_decode(fp8, dev, barrier, args, hbm_peak):
    """Llama-3-8B decode linears (M in {1, 8, 32, 64}).  Every linear is timed
    as a graph of back-to-back launches, each on another copy of the
    quantized weights (distinct addresses, >= 2.5 x L2 per rotation), so each
    launch streams its weights from HBM as in a model whose layers all
    differ.  `layer` times one whole decoder layer per token count (4
    activation quantizations + q, k, v, o, gate+up, down) over 4 layers'
    weight copies."""
    import torch
    names = list(wl.LLAMA3_8B_LINEARS)
    wsets = {}
    for name in names:
        N, K = wl.LLAMA3_8B_LINEARS[name]
        w = wl.to_torch_bf16(wl.llama3_decode_w(name)).to(dev)
        q_w, s_w = fp8.quant_weight(w)
        del w
        R = copies_for(N * K)
        wsets[name] = [(q_w, s_w)] + [(q_w.clone(), s_w.clone()) for _ in range(R - 1)]
    torch.cuda.synchronize(dev)
    out, acts = {}, {}
    tot_bytes, tot_ms = 0.0, 0.0
    for M in wl.DECODE_M:
        for name in names:
            N, K = wl.LLAMA3_8B_LINEARS[name]
            xb = wl.llama3_decode_x(M, name)
            x = wl.to_torch_bf16(xb).to(dev)
            q_a, s_a = fp8.quant_act(x)
            y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(max(fp8.workspace_bytes(M, N, K), 16), dtype=torch.uint8, device=dev)
            cps = wsets[name]

            def run(q_a=q_a, s_a=s_a, y=y, ws=ws, cps=cps):
                for q_w, s_w in cps:
                    fp8.block_linear(q_a, s_a, q_w, s_w, y, ws)

            g = capture_graph(run, dev)
            reps = max(2, int(np.ceil(args.decode_launches / len(cps))))
            ms = timed_replays(g.replay, reps, barrier)
            del g
            launches = reps * len(cps)
            out[f"{name}_M{M}"] = dict(ms=ms, launches=launches, bytes=decode_bytes(M, N, K))
            acts[(name, M)] = dict(xb=xb, x=x, q_a=q_a, s_a=s_a, y=y, ws=ws)
    # whole layers: q, k, v share the attention input; o, gate+up and down
    # each quantize their own input
    layers = 4
    layer_out = {}
    for M in wl.DECODE_M:
        qa_bufs = {n: (torch.empty_like(acts[(n, M)]["q_a"]), torch.empty_like(acts[(n, M)]["s_a"]))
                   for n in names}
        # the layer writes its own outputs (the per-linear outputs above are
        # checked against the oracle afterwards)
        y_bufs = {n: torch.empty_like(acts[(n, M)]["y"]) for n in names}

        def layer_run(M=M, qa_bufs=qa_bufs, y_bufs=y_bufs):
            for l in range(layers):
                def lin(name, idx, xname):
                    cp = wsets[name][idx % len(wsets[name])]
                    fp8.block_linear(qa_bufs[xname][0], qa_bufs[xname][1], cp[0], cp[1], y_bufs[name],
                                     acts[(name, M)]["ws"])
                fp8.quant_act(acts[("qo", M)]["x"], *qa_bufs["qo"])
                lin("qo", 2 * l, "qo")
                lin("kv", 2 * l, "qo")
                lin("kv", 2 * l + 1, "qo")
                fp8.quant_act(acts[("kv", M)]["x"], *qa_bufs["kv"])
                lin("qo", 2 * l + 1, "kv")
                fp8.quant_act(acts[("gate_up", M)]["x"], *qa_bufs["gate_up"])
                lin("gate_up", l, "gate_up")
                fp8.quant_act(acts[("down", M)]["x"], *qa_bufs["down"])
                lin("down", l, "down")

        g = capture_graph(layer_run, dev)
        reps = max(2, args.decode_launches // 24)
        ms = timed_replays(g.replay, reps, barrier)
        del g
        wbytes = sum(decode_bytes(M, *wl.LLAMA3_8B_LINEARS[n]) for n in ("qo", "kv", "kv", "qo", "gate_up", "down"))
        qbytes = sum(M * K * 3 + M * (K // 128) * 4 for K in (4096, 4096, 4096, 14336))
        layer_out[f"M{M}"] = dict(ms=ms, reps=reps * layers, bytes=wbytes + qbytes)
    return out, layer_out, acts, wsets


def decode_oracle(acts, wsets, rows_per_linear=1):
    """The oracle on the decode linears: every M = 1 linear complete (the CPU
    baseline: activation quant + fp64 GEMM, weights' codes from the GPU) and
    `rows_per_linear` sampled rows of the M = 8, 32, 64 linears.  Returns
    (cpu_baseline dict, parity dict)."""
    import torch
    import oracle
    threads = os.cpu_count() or 1
    t_tot, b_tot, worst = 0.0, 0.0, 0.0
    g = np.random.default_rng(5)
    for (name, M), a in acts.items():
        q_w, s_w = wsets[name][0]
        qw = q_w.view(torch.uint8).cpu().numpy()
        sw = s_w.cpu().numpy()
        N, K = qw.shape
        rows = np.arange(M) if M == 1 else np.sort(g.choice(M, rows_per_linear, replace=False))
        xs = np.ascontiguousarray(a["xb"][rows])
        t0 = time.perf_counter()
        qa, sa = oracle.quant_act(xs, nthreads=threads)
        R = oracle.block_linear(qa, sa, qw, sw, nthreads=threads)
        dt = time.perf_counter() - t0
        if M == 1:
            t_tot += dt
            b_tot += decode_bytes(1, N, K)
        Y = a["y"][torch.as_tensor(rows, device=a["y"].device)].float().cpu().numpy()
        worst = max(worst, within_tolerance(Y, R))
    cpu = {"value": b_tot / t_tot / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
           "seconds": t_tot,
           "sample": "the four Llama-3-8B decode linears at M = 1, complete (activation quant + "
                     "fp64 block-scaled GEMM; weights quantized before timing); GB/s of the same "
                     "algorithmic bytes as the GPU figure"}
    par = {"rows": f"all rows at M = 1, {rows_per_linear} sampled row(s) at M = 8, 32, 64, all N",
           "within_tolerance": worst <= 1.0, "worst_bound_ratio": worst}
    return cpu, par


def leg_gemm_workload(fp8, dev, barrier, args, lins):
    """One large-M workload (e.g. the DeepSeek-V3 MLP): the step = per linear
    quant_act + block_linear, graph-replayed; the GEMMs' own rate from a pass
    with events around them; the fused entry point on the same inputs, with
    a bit-identity check against the two-call output."""
    import torch
    items = []
    for label, xb, wb in lins:
        M, K = xb.shape
        N = wb.shape[0]
        x = wl.to_torch_bf16(xb).to(dev)
        w = wl.to_torch_bf16(wb).to(dev)
        q_w, s_w = fp8.quant_weight(w)
        del w
        items.append(dict(label=label, xb=xb, x=x, q_w=q_w, s_w=s_w,
                          q_a=torch.empty((M, K), dtype=torch.float8_e4m3fn, device=dev),
                          s_a=torch.empty((M, K // 128), dtype=torch.float32, device=dev),
                          y=torch.empty((M, N), dtype=torch.bfloat16, device=dev), M=M, N=N, K=K))

    def step(ev=None):
        for i, it in enumerate(items):
            fp8.quant_act(it["x"], it["q_a"], it["s_a"])
            if ev is not None:
                ev[2 * i].record()
            fp8.block_linear(it["q_a"], it["s_a"], it["q_w"], it["s_w"], it["y"])
            if ev is not None:
                ev[2 * i + 1].record()

    n = len(items)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * n)] for _ in range(args.steps)]
    step()
    barrier()
    for k in range(args.steps):
        step(evs[k])
    barrier()
    gemm_ms = sum(e[2 * i].elapsed_time(e[2 * i + 1]) for e in evs for i in range(n))
    y_ref = [it["y"].clone() for it in items]

    # The two-call step and the fused entry point (with its workspace, and
    # in-GEMM without) are timed in alternating rounds, so that the clock
    # drift of a long power-capped run does not favour whichever runs first.
    def fused_fn(in_kernel):
        def fused():
            for it in items:
                fp8.block_linear_fused(it["x"], it["q_w"], it["s_w"], it["y"], in_kernel=in_kernel)
        return fused

    out = {}
    graphs = {"two_call": capture_graph(step, dev)}
    for key, in_kernel in (("fused", False), ("fused_ik", True)):
        for it in items:
            it["y"].zero_()
        graphs[key] = capture_graph(fused_fn(in_kernel), dev)
        graphs[key].replay()
        torch.cuda.synchronize(dev)
        out[key + "_same"] = all(torch.equal(r.view(torch.int16), it["y"].view(torch.int16))
                                 for r, it in zip(y_ref, items))
    rounds = max(1, min(4, args.steps))
    per = [max(1, args.steps // rounds)] * rounds
    per[-1] += args.steps - sum(per)
    tot = {k: 0.0 for k in graphs}
    for r in range(rounds):
        for k, g in graphs.items():
            tot[k] += timed_replays(g.replay, per[r], barrier)
    ms = tot["two_call"]
    out["fused_ms"], out["fused_ik_ms"] = tot["fused"], tot["fused_ik"]
    del graphs
    flops = sum(2 * it["M"] * it["N"] * it["K"] for it in items)
    return items, dict(ms=ms, gemm_ms=gemm_ms, fused_ms=out["fused_ms"], fused_ik_ms=out["fused_ik_ms"],
                       flops=flops, identical=out["fused_same"], identical_ik=out["fused_ik_same"])


def rows_oracle_check(items, rows_per_linear, seed=0):
    """Oracle on `rows_per_linear` random rows of every linear (it quantizes
    those rows of the same input bits itself; weights: the GPU's codes, held
    bit-exact to the oracle by the tests).  Returns (cpu_baseline, parity)."""
    import torch
    import oracle
    threads = os.cpu_count() or 1
    t_tot, f_tot, worst = 0.0, 0.0, 0.0
    for i, it in enumerate(items):
        g = np.random.default_rng([seed, i])
        rows = np.sort(g.choice(it["M"], min(rows_per_linear, it["M"]), replace=False))
        qw = it["q_w"].view(torch.uint8).cpu().numpy()
        sw = it["s_w"].cpu().numpy()
        xs = np.ascontiguousarray(it["xb"][rows])
        t0 = time.perf_counter()
        qa, sa = oracle.quant_act(xs, nthreads=threads)
        R = oracle.block_linear(qa, sa, qw, sw, nthreads=threads)
        t_tot += time.perf_counter() - t0
        f_tot += 2.0 * len(rows) * it["N"] * it["K"]
        Y = it["y"][torch.as_tensor(rows, device=it["y"].device)].float().cpu().numpy()
        worst = max(worst, within_tolerance(Y, R))
    desc = (f"{rows_per_linear} random rows per linear ({', '.join(it['label'] for it in items)}), "
            "all N columns; activation quant + fp64 GEMM of those rows; weights quantized before timing")
    return ({"value": f_tot / t_tot / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
             "sample": desc, "seconds": t_tot},
            {"rows_per_linear": rows_per_linear, "within_tolerance": worst <= 1.0,
             "worst_bound_ratio": worst})


def leg_sweep(fp8, dev, barrier, args):
    """Sweep X [M, 7168], M = 512 .. 16384, against W [2048, 7168]: per M the
    activation quantizer's GB/s, the unfused GEMM's and the fused entry
    point's TFLOP/s.  Every launch reads another copy of its operands
    (>= 2.5 x L2 per rotation), so small M is not served from the L2."""
    import torch
    wb = wl.sweep_w()
    w = wl.to_torch_bf16(wb).to(dev)
    q_w0, s_w0 = fp8.quant_weight(w)
    del w
    K, N = wl.SWEEP_K, wl.SWEEP_N
    res, items = {}, []
    for M in wl.SWEEP_M:
        xb = wl.sweep_x(M)
        x0 = wl.to_torch_bf16(xb).to(dev)
        qbytes = M * K * 3 + M * (K // 128) * 4
        gbytes = M * K + N * K + 2 * M * N
        R = copies_for(min(qbytes, gbytes))
        xs = [x0] + [x0.clone() for _ in range(R - 1)]
        qs = [(torch.empty((M, K), dtype=torch.float8_e4m3fn, device=dev),
               torch.empty((M, K // 128), dtype=torch.float32, device=dev)) for _ in range(R)]
        ws = [(q_w0, s_w0)] + [(q_w0.clone(), s_w0.clone()) for _ in range(R - 1)]
        ys = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(R)]
        reps = max(2, int(np.ceil(args.sweep_launches / R)))

        def quant():
            for x, (q, s) in zip(xs, qs):
                fp8.quant_act(x, q, s)

        def gemm():
            for (q, s), (qw, sw), y in zip(qs, ws, ys):
                fp8.block_linear(q, s, qw, sw, y)

        yf = [torch.empty_like(y) for y in ys]
        yk = [torch.empty_like(y) for y in ys]

        def fused():
            for x, (qw, sw), y in zip(xs, ws, yf):
                fp8.block_linear_fused(x, qw, sw, y)

        def fused_ik():
            for x, (qw, sw), y in zip(xs, ws, yk):
                fp8.block_linear_fused(x, qw, sw, y, in_kernel=True)

        r = {}
        for key, fn in (("quant", quant), ("gemm", gemm), ("fused", fused), ("fused_ik", fused_ik)):
            g = capture_graph(fn, dev)
            r[key] = timed_replays(g.replay, reps, barrier) / (reps * R)
            del g
        torch.cuda.synchronize(dev)
        same = all(torch.equal(a.view(torch.int16), b.view(torch.int16)) for a, b in zip(ys, yf)) and \
            all(torch.equal(a.view(torch.int16), b.view(torch.int16)) for a, b in zip(ys, yk))
        res[f"M{M}"] = dict(quant_ms=r["quant"], gemm_ms=r["gemm"], fused_ms=r["fused"],
                            fused_ik_ms=r["fused_ik"], identical=same,
                            qbytes=qbytes, flops=2.0 * M * N * K, copies=R)
        items.append(dict(label=f"M{M}", xb=xb, q_w=q_w0, s_w=s_w0, y=ys[0], M=M, N=N, K=K))
        del xs, qs, ws, yf, yk
    return res, items


def leg_tiny(fp8, dev, barrier, args):
    """The tiny linear (X [32, 512], W [256, 512]): latency of one
    quant_act + block_linear, from a graph of back-to-back calls; the output
    is compared with the oracle element by element."""
    import torch
    import oracle
    xb, wb = wl.tiny()
    x = wl.to_torch_bf16(xb).to(dev)
    q_w, s_w = fp8.quant_weight(wl.to_torch_bf16(wb).to(dev))
    M, K = xb.shape
    N = wb.shape[0]
    q_a = torch.empty((M, K), dtype=torch.float8_e4m3fn, device=dev)
    s_a = torch.empty((M, K // 128), dtype=torch.float32, device=dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(fp8.workspace_bytes(M, N, K), 16), dtype=torch.uint8, device=dev)
    calls = 50

    def run():
        for _ in range(calls):
            fp8.quant_act(x, q_a, s_a)
            fp8.block_linear(q_a, s_a, q_w, s_w, y, ws)

    g = capture_graph(run, dev)
    ms = timed_replays(g.replay, 4, barrier) / (4 * calls)
    del g
    t0 = time.perf_counter()
    qa, sa = oracle.quant_act(xb)
    R = oracle.block_linear(qa, sa, q_w.view(torch.uint8).cpu().numpy(), s_w.cpu().numpy())
    cpu_s = time.perf_counter() - t0
    worst = within_tolerance(y.float().cpu().numpy(), R)
    codes_same = bool(np.array_equal(q_a.view(torch.uint8).cpu().numpy(), qa) and
                      np.array_equal(s_a.cpu().numpy().view(np.uint32), sa.view(np.uint32)))
    return dict(ms=ms, flops=2.0 * M * N * K, worst=worst, codes_same=codes_same, cpu_s=cpu_s)


# ----------------------------------------------------------------- GPU side

def legs_json(legs, world, args, hbm_peak, fp8_peak, peak_src):
    """JSON keys of the per-config legs (rank 0, after the max over ranks).
    The oracle checks and CPU baselines run only at N = 1 (replicas compute
    the same thing)."""
    out = {}
    cpu_ok = world == 1 and not args.no_cpu
    if "decode" in legs:
        out.update(decode_json(legs["decode"], cpu_ok, hbm_peak, peak_src))
    if "deepseek_mlp" in legs:
        out.update(deepseek_json(legs["deepseek_mlp"], world, args, cpu_ok, fp8_peak))
    if "sweep" in legs:
        out.update(sweep_json(legs["sweep"], cpu_ok, hbm_peak, fp8_peak))
    if "tiny" in legs:
        out.update(tiny_json(legs["tiny"], cpu_ok))
    if "deepseek_moe" in legs:
        out.update(moe_json(legs["deepseek_moe"], world, args, cpu_ok, fp8_peak, peak_src))
    return out


def decode_json(leg, cpu_ok, hbm_peak, peak_src):
    out = {}
    dec, lay, acts, wsets = leg
    lin = {}
    tb, tm = 0.0, 0.0
    for k, d in dec.items():
        us = d["ms"] * 1e3 / d["launches"]
        gbs = d["bytes"] / (us * 1e-6) / 1e9
        lin[k] = {"us": us, "GBps": gbs, "frac": gbs / hbm_peak, "bytes": d["bytes"]}
        tb += d["bytes"] * d["launches"]
        tm += d["ms"]
    agg = tb / (tm * 1e-3) / 1e9
    layer = {}
    for k, d in lay.items():
        us = d["ms"] * 1e3 / d["reps"]
        gbs = d["bytes"] / (us * 1e-6) / 1e9
        layer[k] = {"us_per_layer": us, "GBps": gbs, "frac": gbs / hbm_peak}
    dcpu, dpar = decode_oracle(acts, wsets) if cpu_ok else (None, None)
    out["decode"] = {
        "metric": "decode linear GB/s (algorithmic bytes: W codes + block scales, X codes + scales, Y)",
        "value": agg, "unit": "GB/s", "peak": hbm_peak, "frac": agg / hbm_peak,
        "peak_source": f"{peak_src} copy", "kernel": "decode_kernel",
        "linears": lin, "layer": layer,
        "config": {"workload": "llama3_decode", "M": list(wl.DECODE_M),
                   "linears": {n: list(v) for n, v in wl.LLAMA3_8B_LINEARS.items()},
                   "l2": "each launch reads another copy of the weights (a rotation moves >= 2.5 x L2)",
                   "launch": "CUDA graph of back-to-back launches (programmatic dependent launch)",
                   "layer": "one decoder layer = 4 activation quantizations + q, k, v, o, gate+up, down; "
                            "4 layers' weight copies per replay"},
        "cpu_baseline": dcpu, "parity": dpar}
    return out


def deepseek_json(leg, world, args, cpu_ok, fp8_peak):
    out = {}
    items, ds = leg
    tf = ds["flops"] * args.steps / (ds["gemm_ms"] * 1e-3) / 1e12
    step_tf = whole_job_rate(world, ds["flops"], args.steps, ds["ms"]) / 1e12
    dcpu, dpar = rows_oracle_check(items, 4) if cpu_ok else (None, None)
    out["deepseek_mlp"] = {
        "value": step_tf, "unit": "TFLOP/s", "ms_per_step": ds["ms"] / args.steps,
        "config": {"workload": "deepseek_mlp",
                   "linears": {it["label"]: [it["M"], it["N"], it["K"]] for it in items},
                   "l2": "no flush: a step's inputs exceed the 126 MB L2"},
        "gemm": {"kernel": "gemm_prefill_kernel", "achieved": tf, "peak": fp8_peak, "unit": "TFLOP/s",
                 "frac": tf / fp8_peak, "ms_per_launch": ds["gemm_ms"] / (args.steps * len(items)),
                 "traffic": recorded_traffic("gemm_prefill_kernel", "deepseek_mlp")},
        "fused": {"value": whole_job_rate(world, ds["flops"], args.steps, ds["fused_ms"]) / 1e12,
                  "vs_two_call": ds["ms"] / ds["fused_ms"], "identical_to_two_call": ds["identical"],
                  "in_kernel": {"value": whole_job_rate(world, ds["flops"], args.steps, ds["fused_ik_ms"]) / 1e12,
                                "vs_two_call": ds["ms"] / ds["fused_ik_ms"],
                                "identical_to_two_call": ds["identical_ik"]}},
        "cpu_baseline": dcpu, "parity": dpar}
    return out


def sweep_json(leg, cpu_ok, hbm_peak, fp8_peak):
    out = {}
    sw, sitems = leg
    per = {}
    for k, d in sw.items():
        q_gbs = d["qbytes"] / (d["quant_ms"] * 1e-3) / 1e9
        g_tf = d["flops"] / (d["gemm_ms"] * 1e-3) / 1e12
        f_tf = d["flops"] / (d["fused_ms"] * 1e-3) / 1e12
        per[k] = {"act_quant_GBps": q_gbs, "act_quant_frac": q_gbs / hbm_peak,
                  "gemm_TFLOPs": g_tf, "gemm_frac": g_tf / fp8_peak,
                  "fused_TFLOPs": f_tf, "fused_vs_two_call": (d["quant_ms"] + d["gemm_ms"]) / d["fused_ms"],
                  "fused_in_kernel_vs_two_call": (d["quant_ms"] + d["gemm_ms"]) / d["fused_ik_ms"],
                  "identical_to_two_call": d["identical"], "copies": d["copies"]}
    scpu, spar = rows_oracle_check(sitems, 4, seed=1) if cpu_ok else (None, None)
    out["sweep"] = {
        "unit": {"act_quant": "GB/s", "gemm": "TFLOP/s"}, "hbm_peak": hbm_peak, "fp8_peak": fp8_peak,
        "config": {"workload": "sweep", "M": list(wl.SWEEP_M), "N": wl.SWEEP_N, "K": wl.SWEEP_K,
                   "l2": "each launch reads another copy of its operands (a rotation moves >= 2.5 x L2)"},
        "per_M": per, "cpu_baseline": scpu, "parity": spar}
    return out


def tiny_json(t, cpu_ok):
    out = {}
    out["tiny"] = {"us_per_linear": t["ms"] * 1e3, "unit": "us (quant_act + block_linear)",
                   "TFLOPs": t["flops"] / (t["ms"] * 1e-3) / 1e12,
                   "config": {"workload": "tiny", "M": 32, "N": 256, "K": 512,
                              "launch": "CUDA graph of 50 back-to-back calls"},
                   "parity": {"all_elements": True, "within_tolerance": t["worst"] <= 1.0,
                              "worst_bound_ratio": t["worst"], "codes_and_scales_bit_exact": t["codes_same"]},
                   "cpu_baseline": {"value": t["cpu_s"] * 1e6, "unit": "us", "kind": "oracle",
                                    "cores": 1, "sample": "the whole tiny linear"} if cpu_ok else None}
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist

    import fine_grained_block_token_b200 as fp8

    world, rank, local = rank_info()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    hbm_peak, bf16_peak, peak_src = peaks()
    fp8_peak = bf16_peak * FP8_OVER_BF16

    lins = workload_linears(args.workload)
    items = []
    for label, xb, wb in lins:
        M, K = xb.shape
        N = wb.shape[0]
        x = wl.to_torch_bf16(xb).to(dev)
        w = wl.to_torch_bf16(wb).to(dev)
        q_w, s_w = fp8.quant_weight(w)
        del w
        q_a = torch.empty((M, K), dtype=torch.float8_e4m3fn, device=dev)
        s_a = torch.empty((M, K // 128), dtype=torch.float32, device=dev)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ws_n = fp8.workspace_bytes(M, N, K)
        ws = torch.empty(max(ws_n, 16), dtype=torch.uint8, device=dev)
        items.append(dict(label=label, xb=xb, x=x, q_w=q_w, s_w=s_w, q_a=q_a, s_a=s_a, y=y, ws=ws,
                          M=M, N=N, K=K))
    torch.cuda.synchronize()
    flops_step = sum(2 * it["M"] * it["N"] * it["K"] for it in items)
    act_bytes_step = sum(it["M"] * it["K"] * (2 + 1) + it["M"] * (it["K"] // 128) * 4 for it in items)
    gemm_flops_step = flops_step

    def step(ev=None):
        for i, it in enumerate(items):
            if ev is not None:
                ev[4 * i].record()
            fp8.quant_act(it["x"], it["q_a"], it["s_a"])
            if ev is not None:
                ev[4 * i + 1].record()
                ev[4 * i + 2].record()
            fp8.block_linear(it["q_a"], it["s_a"], it["q_w"], it["s_w"], it["y"], it["ws"])
            if ev is not None:
                ev[4 * i + 3].record()

    for _ in range(args.warmup):
        step()
    fp8.check()

    # The timed steps replay a CUDA graph of one step: the library's launches
    # (tensor-map set-up, workspace clears, kernels) are captured once, so the
    # host's launch rate drops out of the device time.  --eager times the
    # launches one by one instead.
    def capture(fn):
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            fn()
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        torch.cuda.synchronize(dev)
        return g

    graph = None if args.eager else capture(step)
    run_step = (lambda: graph.replay()) if graph is not None else step

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.3)

    # ---- device-timed region: K whole steps, nothing else on the stream
    n = len(items)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier()
    t_start.record()
    for k in range(args.steps):
        run_step()
    t_end.record()
    barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    fp8.check()

    # ---- the same K steps again with events around every kernel, for the
    # per-kernel rates (the event records themselves cost a few us each,
    # which matters next to decode-sized kernels, hence the separate pass)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4 * n)] for _ in range(args.steps)]
    barrier()
    for k in range(args.steps):
        step(evs[k])
    barrier()
    gemm_ms = sum(e[4 * i + 2].elapsed_time(e[4 * i + 3]) for e in evs for i in range(n))
    fp8.check()

    # ---- the activation quantizer's own rate: a graph of back-to-back
    # quantizations of the step's inputs (no events between kernels; the
    # step's inputs exceed the L2, so every launch reads X from HBM)
    aq_per_graph = 10

    def quant_only():
        for _ in range(aq_per_graph):
            for it in items:
                fp8.quant_act(it["x"], it["q_a"], it["s_a"])

    aq_graph = capture_graph(quant_only, dev)
    aq_reps = max(2, args.steps // 5)
    act_ms = timed_replays(aq_graph.replay, aq_reps, barrier)
    del aq_graph
    act_steps = aq_per_graph * aq_reps

    # ---- end to end: pinned host inputs in, outputs back, every step
    host_x = [wl.to_torch_bf16(it["xb"]).pin_memory() for it in items]
    host_y = [torch.empty((it["M"], it["N"]), dtype=torch.bfloat16).pin_memory() for it in items]
    h2d = sum(t.numel() * 2 for t in host_x)
    d2h = sum(t.numel() * 2 for t in host_y)

    def e2e_compute(xs, ys):
        for it, x, y in zip(items, xs, ys):
            fp8.quant_act(x, it["q_a"], it["s_a"])
            fp8.block_linear(it["q_a"], it["s_a"], it["q_w"], it["s_w"], y, it["ws"])

    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    e2e_ms = pipelined_e2e(items, host_x, host_y, e2e_compute, e2e_steps, min(args.warmup, 3),
                           barrier, dev)
    # ---- the fused entry point (bf16 activations in one call) on the same
    # inputs and steps, with its workspace (staged codes) and without it
    # (quantization inside the GEMM's tiles, prefill sizes only); its output
    # must equal the two-call one
    y_ref = [it["y"].clone() for it in items]
    fws = []
    for it in items:
        nb = fp8.fused_workspace_bytes(it["M"], it["N"], it["K"])
        fws.append(torch.empty(max(nb, 16), dtype=torch.uint8, device=dev))

    def time_fused(in_kernel):
        def fused_step():
            for it, w in zip(items, fws):
                if in_kernel:
                    fp8.block_linear_fused(it["x"], it["q_w"], it["s_w"], it["y"], in_kernel=True)
                else:
                    fp8.block_linear_fused(it["x"], it["q_w"], it["s_w"], it["y"], w)

        for _ in range(min(args.warmup, 3)):
            fused_step()
        torch.cuda.synchronize()
        fgraph = None if args.eager else capture(fused_step)
        run_fused = (lambda: fgraph.replay()) if fgraph is not None else fused_step
        for it in items:
            it["y"].zero_()
        run_fused()
        torch.cuda.synchronize()
        identical = all(torch.equal(r.view(torch.int16), it["y"].view(torch.int16))
                        for r, it in zip(y_ref, items))
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        barrier()
        a.record()
        for _ in range(args.steps):
            run_fused()
        b.record()
        barrier()
        ms = a.elapsed_time(b)
        del fgraph
        return ms, identical

    fused_ms, fused_identical = time_fused(False)
    fused_ik_ms, fused_ik_identical = (None, None) if decode_workload(args.workload) else time_fused(True)

    # ---- the scale-format variants on the same inputs, each one step =
    # its activation quantization + its GEMM per linear, timed like the
    # headline step (graph replay), then a pass with events around the GEMMs:
    #   ue8m0  -- power-of-two scales on the tensor core's block-scaled MMA
    #   fp8r   -- one fp32 scale per activation row and weight row
    variants = {}
    if not decode_workload(args.workload):
        wbits = {lb: wb for lb, _, wb in lins}
        specs = {
            "ue8m0": dict(wq=fp8.quant_weight_ue8m0, aq=fp8.quant_act_ue8m0,
                          gemm=fp8.block_linear_ue8m0, kernel="gemm_ue8m0_pair_kernel",
                          ws=fp8.ue8m0_workspace_bytes,
                          s_a=lambda it: torch.empty((it["M"], it["K"] // 128),
                                                     dtype=torch.float8_e8m0fnu, device=dev)),
            "fp8r": dict(wq=fp8.quant_rowwise, aq=fp8.quant_rowwise,
                         gemm=fp8.linear_rowwise,
                         # CTA pairs above one 128-row tile (the prefill workloads)
                         kernel="gemm_rowwise_pair_kernel",
                         s_a=lambda it: torch.empty((it["M"],), dtype=torch.float32, device=dev)),
        }
        for name, sp in specs.items():
            v_items = []
            for it in items:
                w = wl.to_torch_bf16(wbits[it["label"]]).to(dev)
                q_wv, s_wv = sp["wq"](w)
                del w
                ws_n = sp["ws"](it["M"], it["N"], it["K"]) if "ws" in sp else 0
                v_items.append(dict(it=it, q_w=q_wv, s_w=s_wv, q_a=torch.empty_like(it["q_a"]),
                                    s_a=sp["s_a"](it), y=torch.empty_like(it["y"]),
                                    ws=torch.empty(max(ws_n, 16), dtype=torch.uint8, device=dev)
                                    if ws_n else None))

            def v_step(ev=None, v_items=v_items, sp=sp):
                for i, u in enumerate(v_items):
                    sp["aq"](u["it"]["x"], u["q_a"], u["s_a"])
                    if ev is not None:
                        ev[2 * i].record()
                    if u["ws"] is not None:
                        sp["gemm"](u["q_a"], u["s_a"], u["q_w"], u["s_w"], u["y"], workspace=u["ws"])
                    else:
                        sp["gemm"](u["q_a"], u["s_a"], u["q_w"], u["s_w"], u["y"])
                    if ev is not None:
                        ev[2 * i + 1].record()

            for _ in range(min(args.warmup, 3)):
                v_step()
            torch.cuda.synchronize()
            v_graph = None if args.eager else capture(v_step)
            run_v = (lambda: v_graph.replay()) if v_graph is not None else v_step
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            barrier()
            a.record()
            for _ in range(args.steps):
                run_v()
            b.record()
            barrier()
            v_ms = a.elapsed_time(b)
            evv = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * n)] for _ in range(args.steps)]
            barrier()
            for k in range(args.steps):
                v_step(evv[k])
            barrier()
            v_gemm_ms = sum(e[2 * i].elapsed_time(e[2 * i + 1]) for e in evv for i in range(n))
            del v_graph
            variants[name] = dict(items=v_items, ms=v_ms, gemm_ms=v_gemm_ms, kernel=sp["kernel"])
    # ---- the other workloads of the build, on the same line
    legs = {}
    want = set(args.legs.split(",")) if args.legs else set()
    run_legs = args.workload == "llama3_prefill" and not args.no_legs and bool(want)
    if run_legs:
        if "decode" in want:
            legs["decode"] = leg_decode(fp8, dev, barrier, args, hbm_peak)
        if "deepseek_mlp" in want:
            legs["deepseek_mlp"] = leg_gemm_workload(fp8, dev, barrier, args,
                                                     workload_linears("deepseek_mlp"))
        if "sweep" in want:
            legs["sweep"] = leg_sweep(fp8, dev, barrier, args)
        if "tiny" in want:
            legs["tiny"] = leg_tiny(fp8, dev, barrier, args)
        if "deepseek_moe" in want:
            legs["deepseek_moe"] = leg_moe(fp8, dev, barrier, args)
    sampler.stop()
    fp8.check()

    # max over ranks (every device time below is the slowest rank's)
    vnames = sorted(variants)
    times = [elapsed_ms, e2e_ms, act_ms, gemm_ms, fused_ms, fused_ik_ms or 0.0] + \
        [variants[v][k] for v in vnames for k in ("ms", "gemm_ms")]
    leg_slots = []
    if "decode" in legs:
        dec, lay, _, _ = legs["decode"]
        for k in sorted(dec):
            leg_slots.append((dec[k], "ms"))
        for k in sorted(lay):
            leg_slots.append((lay[k], "ms"))
    if "deepseek_mlp" in legs:
        _, ds = legs["deepseek_mlp"]
        leg_slots += [(ds, "ms"), (ds, "gemm_ms"), (ds, "fused_ms"), (ds, "fused_ik_ms")]
    if "sweep" in legs:
        sw, _ = legs["sweep"]
        for k in sorted(sw):
            leg_slots += [(sw[k], "quant_ms"), (sw[k], "gemm_ms"), (sw[k], "fused_ms"), (sw[k], "fused_ik_ms")]
    if "tiny" in legs:
        leg_slots.append((legs["tiny"], "ms"))
    if "deepseek_moe" in legs:
        _, dm = legs["deepseek_moe"]
        leg_slots += [(dm, "ms"), (dm, "gemm_ms")]
    maxed = max_over_ranks(times + [d[k] for d, k in leg_slots], dev, world)
    elapsed_ms, e2e_ms, act_ms, gemm_ms, fused_ms, fused_ik_ms_max = maxed[:6]
    fused_ik_ms = fused_ik_ms_max if fused_ik_ms is not None else None
    for i, v in enumerate(vnames):
        variants[v]["ms"], variants[v]["gemm_ms"] = maxed[6 + 2 * i], maxed[7 + 2 * i]
    for (d, k), v in zip(leg_slots, maxed[len(times):]):
        d[k] = v

    ms_per_step = elapsed_ms / args.steps
    value = whole_job_rate(world, flops_step, args.steps, elapsed_ms) / 1e12
    e2e_value = whole_job_rate(world, flops_step, e2e_steps, e2e_ms) / 1e12
    gemm_tflops = gemm_flops_step * args.steps / (gemm_ms * 1e-3) / 1e12
    act_gbs = act_bytes_step * act_steps / (act_ms * 1e-3) / 1e9
    launches_per_step = 2 * n
    fused_value = whole_job_rate(world, flops_step, args.steps, fused_ms) / 1e12
    decode = args.workload == "llama3_decode"
    # decode linears are bound by streaming the weights: algorithmic bytes =
    # codes + block scales of W, codes + group scales of X, bf16 Y
    gemm_bytes_step = sum(it["N"] * it["K"] + (it["N"] // 128) * (it["K"] // 128) * 4 +
                          it["M"] * it["K"] + it["M"] * (it["K"] // 128) * 4 + 2 * it["M"] * it["N"]
                          for it in items)
    gemm_gbs = gemm_bytes_step * args.steps / (gemm_ms * 1e-3) / 1e9

    if rank == 0:
        parity = None
        cpu = None
        if world == 1 and not args.no_cpu:
            # CPU-baseline leg: the oracle on a bounded row sample of the same
            # input bits (it quantizes them itself); the GPU rows it covers
            # are also checked against its result.
            prepared = cpu_prepare(lins, args.cpu_rows)
            t, f, thr, outs = cpu_step(prepared)
            cpu = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
                   "sample": sample_desc(prepared), "seconds": t}
            worst = 0.0
            for it in items:
                rows, R = outs[it["label"]]
                Y = it["y"][torch.as_tensor(rows, device=dev)].float().cpu().numpy()
                worst = max(worst, within_tolerance(Y, R))
            parity = {"rows_per_linear": args.cpu_rows, "within_tolerance": worst <= 1.0,
                      "worst_bound_ratio": worst}
        variant_lines = {}
        for v in vnames:
            d = variants[v]
            tf = gemm_flops_step * args.steps / (d["gemm_ms"] * 1e-3) / 1e12
            variant_lines[v] = {
                "value": whole_job_rate(world, flops_step, args.steps, d["ms"]) / 1e12,
                "unit": "TFLOP/s", "ms_per_step": d["ms"] / args.steps,
                "vs_fp32_block_scales": ms_per_step / (d["ms"] / args.steps),
                "gemm": {"kernel": d["kernel"], "achieved": tf, "peak": fp8_peak, "unit": "TFLOP/s",
                         "frac": tf / fp8_peak, "ms_per_launch": d["gemm_ms"] / (args.steps * n),
                         "traffic": recorded_traffic(d["kernel"], args.workload)}}
            if world == 1 and not args.no_cpu:
                variant_lines[v]["parity"] = variant_parity(v, d["items"], lins, args.variant_rows, dev)
        traffic = recorded_traffic("gemm_prefill_kernel", args.workload)
        gemm_ms_per_launch = gemm_ms / (args.steps * n)
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3", "data": "synthetic",
            "config": {"workload": args.workload,
                       "linears": {it["label"]: [it["M"], it["N"], it["K"]] for it in items},
                       "l2": "no flush: inputs of a step exceed the 126 MB L2",
                       "parallelism": f"replicas x{world} (no data-path collective)",
                       "launch": "eager" if args.eager else "cuda_graph (one step captured, replayed)"},
            "roofline": ({"bound": "hbm", "achieved": gemm_gbs, "peak": hbm_peak,
                          "unit": "GB/s", "frac": gemm_gbs / hbm_peak, "traffic": None,
                          "kernel": "decode_kernel", "peak_source": f"{peak_src} copy",
                          "ms_per_launch": gemm_ms_per_launch,
                          "tflops": gemm_tflops} if decode else
                         {"bound": "tensor", "achieved": gemm_tflops, "peak": fp8_peak,
                          "unit": "TFLOP/s", "frac": gemm_tflops / fp8_peak,
                          "traffic": traffic,
                          "kernel": "gemm_prefill_kernel",
                          "peak_source": f"{peak_src} bf16 burst x {FP8_OVER_BF16} (nominal fp8/bf16)",
                          "ms_per_launch": gemm_ms_per_launch}),
            "act_quant": {"achieved": act_gbs, "peak": hbm_peak, "unit": "GB/s",
                          "frac": act_gbs / hbm_peak, "peak_source": f"{peak_src} copy",
                          "kernel": "act_quant32_kernel",
                          "timing": f"CUDA graph of {aq_per_graph} x the step's quantizations back to back, "
                                    f"{aq_reps} replays"},
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "schedule": "double-buffered: copy in, kernels, copy out on three streams"},
            "fused": {"value": fused_value, "unit": "TFLOP/s", "ms_per_step": fused_ms / args.steps,
                      "vs_two_call": ms_per_step / (fused_ms / args.steps),
                      "kernel": ("act_quant32_kernel into the workspace, then decode_kernel" if decode else
                                 "act_quant32_kernel into the workspace, then gemm_prefill_kernel"),
                      "identical_to_two_call": fused_identical,
                      "in_kernel": None if fused_ik_ms is None else {
                          "value": whole_job_rate(world, flops_step, args.steps, fused_ik_ms) / 1e12,
                          "ms_per_step": fused_ik_ms / args.steps,
                          "vs_two_call": ms_per_step / (fused_ik_ms / args.steps),
                          "kernel": "gemm_fused_kernel (no workspace: quantization in the GEMM's tiles)",
                          "identical_to_two_call": fused_ik_identical}},
            "ue8m0": variant_lines.get("ue8m0"),
            "fp8r": variant_lines.get("fp8r"),
            **(legs_json(legs, world, args, hbm_peak, fp8_peak, peak_src) if run_legs else {}),
            "gpu_launches": launches_per_step * args.steps,
            "clocks": sampler.summary(),
            "cpu_baseline": cpu,
            "parity": parity,
        }
        print(json.dumps(line))
    del graph   # released before the process group goes away
    variants.clear()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama3_prefill",
                    choices=["llama3_prefill", "deepseek_mlp", "llama3_decode", "sweep", "deepseek_moe"])
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--cpu-rows", type=int, default=32)
    ap.add_argument("--ref-rows", type=int, default=4)
    ap.add_argument("--variant-rows", type=int, default=4,
                    help="rows per linear of the ue8m0 / fp8r legs checked against the oracle")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--eager", action="store_true", help="launch every step's kernels one by one")
    ap.add_argument("--no-legs", action="store_true",
                    help="headline prefill step only (skip the decode, deepseek_mlp, sweep, tiny, deepseek_moe keys)")
    ap.add_argument("--legs", default="decode,deepseek_mlp,sweep,tiny,deepseek_moe",
                    help="comma-separated per-config legs to run with the prefill workload")
    ap.add_argument("--decode-launches", type=int, default=96,
                    help="timed launches per decode linear (rounded up to whole weight rotations)")
    ap.add_argument("--sweep-launches", type=int, default=12,
                    help="timed launches per sweep size and kernel (whole rotations)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)   # at least 3 untimed warm-up steps
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "deepseek_moe":
        return run_moe(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
