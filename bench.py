"""Benchmark: S²-Attn forward + backward useful TFLOP/s on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step = one pass of the whole hot path over one batch: s2attn_fwd, then
the three backward stages (prepare, dK/dV pass, dQ pass), on inputs resident
in HBM.  Default workload: B=1, H=32, N=32768, D=128, G=8192, strict variant,
bf16 Q/K/V/dO ~ N(0,1) with K doubled on 5% of positions.

Metric: useful causal TFLOP/s = 7·B·H·N·G·D per step (forward 2·B·H·N·G·D,
backward 2.5x that) / step time; N>1 runs one independent replica per GPU
(weak scaling, no collective on the data path) and reports the whole-job
aggregate over the max-over-ranks device time.  Rank 0 prints one JSON line.

--impl reference times the float64 CPU oracle (the only reference this
method has) on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "S²-Attn fwd+bwd useful TFLOP/s at 1 B200 and % of dense BF16 tensor peak"
UNIT = "TFLOP/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="long_n32768_g8192")
    ap.add_argument("--variant", type=int, default=None, help="0 strict, 1 rolled, 2 dense causal")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--doc-len", type=int, default=0,
                    help="pack documents of this many tokens (document mask); reports exact-pair TFLOP/s")
    ap.add_argument("--sp-emulate", type=int, default=0, metavar="W",
                    help="sequence parallelism: run W ranks' shards (halo exchange + rank kernels) in turn on this GPU")
    ap.add_argument("--sp", action="store_true",
                    help="sequence parallelism over the torchrun ranks: each GPU holds a G-aligned shard of the "
                         "sequence and exchanges the half-group halo over NCCL (strong scaling)")
    ap.add_argument("--recompute-dq", action="store_true",
                    help="dQ pass recomputes S and dP (8 MB workspace) instead of reading the stored dS")
    ap.add_argument("--rope", action="store_true",
                    help="start each step with the RoPE prologue (original positions, interpolation 1/4)")
    return ap.parse_args()


def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return {"bf16_burst": d["bf16_tflops"], "bf16_sustained": d["bf16_tflops_sustained"],
                "hbm_gbs": d["hbm_gbs"], "source": "measured"}
    return {"bf16_burst": 1590.0, "bf16_sustained": 1400.0, "hbm_gbs": 6650.0, "source": "fallback"}


def doc_pair_counts(w, variant, doc_len):
    """Visited pairs per head class under a document mask of back-to-back documents of
    doc_len tokens (strict or dense variant, no padding): every segment cut by the
    document boundaries is a causal triangle."""
    N, G = w.N, w.G
    tri = lambda L: L * (L + 1) // 2
    docs = set(range(0, N + 1, doc_len)) | {N}

    def pairs(group_cuts):
        c = sorted(docs | set(group_cuts))
        return sum(tri(b - a) for a, b in zip(c, c[1:]))

    if variant == 2:
        return pairs({0, N}), pairs({0, N})
    s = G // 2
    return pairs(set(range(0, N + 1, G))), pairs({0, N} | set(range(s, N, G)))


def stored_tile_pairs(w, variant, cls):
    """128x128 tile pairs (key tile <= query tile, both holding a valid row) of one
    head of class cls: the dS tiles the stored-dS backward writes and reads."""
    N, G, nv, T = w.N, w.G, w.valid, 128
    if variant == 2:
        segs = [(0, N)]
    elif cls == 1 and variant == 0:
        s = G // 2
        segs = [(0, s)] + [(s + k * G, G) for k in range(N // G - 1)] + [(N - s, s)]
    else:
        segs = [(k * G, G) for k in range(N // G)]  # rolled class 1: padding sits in the wrap group
    total = 0
    for start, length in segs:
        first = [(start + r * T + (G // 2 if variant == 1 and cls == 1 else 0)) % N for r in range(length // T)]
        valid = [x < nv for x in first]
        seen = 0
        for v in valid:  # pairs key tile <= query tile, both valid
            seen += v
            total += seen if v else 0
    return total


def pair_counts(w, variant):
    """Exact visited (query, key) pairs per head class: every segment is a causal
    triangle over its valid rows in segment order (the strict shifted class has the
    short head and tail groups, the rolled one the wrap group [N - s, N) + [0, s))."""
    N, G, nv = w.N, w.G, w.valid
    s = G // 2

    def seg_pairs(runs):
        total, seen = 0, 0
        for a, b in runs:  # runs in segment order
            n = max(0, min(b, nv) - a)
            # valid rows of this run follow `seen` earlier valid rows of the segment
            total += n * seen + n * (n + 1) // 2
            seen += n
        return total

    if variant == 2:
        c = seg_pairs([(0, N)])
        return c, c
    c0 = sum(seg_pairs([(a, a + G)]) for a in range(0, N, G))
    if variant == 0:
        segs = [[(0, s)]] + [[(a, a + G)] for a in range(s, N - s, G)] + [[(N - s, N)]]
    else:
        segs = [[(a, a + G)] for a in range(s, N - s, G)] + [[(N - s, N), (0, s)]]
    return c0, sum(seg_pairs(r) for r in segs)


# ---------------------------------------------------------------------------- clocks


class ClockSampler:
    """SM clock and throttle reasons sampled during the timed region.

    NVML is read every 10 ms from a background thread (read-only queries), so a
    timed region of a fraction of a second still gets dozens of samples;
    without NVML it falls back to nvidia-smi at its 200 ms floor."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_S = 0.010

    def __init__(self, gpu_index, uuid=None):
        self.gpu_index = gpu_index
        self.uuid = uuid
        self.proc = None
        self.path = None
        self.thread = None
        self.rows = []
        self.source = None

    def _nvml_handle(self):
        import pynvml

        pynvml.nvmlInit()
        if self.uuid:
            try:
                return pynvml.nvmlDeviceGetHandleByUUID(self.uuid)
            except pynvml.NVMLError:
                pass
        return pynvml.nvmlDeviceGetHandleByIndex(int(self.gpu_index))

    def _poll(self, handle):
        import pynvml

        R = pynvml
        bits = (("hw", R.nvmlClocksEventReasonHwSlowdown), ("hwt", R.nvmlClocksEventReasonHwThermalSlowdown),
                ("swt", R.nvmlClocksEventReasonSwThermalSlowdown), ("swp", R.nvmlClocksEventReasonSwPowerCap))
        mx = float(pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM))
        while not self._stop.is_set():
            try:
                sm = float(pynvml.nvmlDeviceGetClockInfo(handle, pynvml.NVML_CLOCK_SM))
                reasons = pynvml.nvmlDeviceGetCurrentClocksEventReasons(handle)
                power = pynvml.nvmlDeviceGetPowerUsage(handle) / 1000.0
            except pynvml.NVMLError:
                break
            row = dict(sm=sm, max=mx, power=power)
            for key, bit in bits:
                row[key] = "Active" if reasons & bit else "Not Active"
            self.rows.append(row)
            self._stop.wait(self.PERIOD_S)

    def __enter__(self):
        import threading

        try:
            handle = self._nvml_handle()
            self._stop = threading.Event()
            self.thread = threading.Thread(target=self._poll, args=(handle,), daemon=True)
            self.thread.start()
            self.source = "nvml every %d ms" % round(self.PERIOD_S * 1e3)
            return self
        except Exception:  # no NVML: nvidia-smi instead
            self.thread = None
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            self.source = "nvidia-smi every 200 ms"
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self._stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = list(self.rows)
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append(dict(sm=float(parts[1]), max=float(parts[2]), power=float(parts[3]),
                                     hw=parts[5], hwt=parts[6], swt=parts[7], swp=parts[8]))
                except ValueError:
                    continue
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        reasons = set()
        counts = {}
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                              ("swp", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
                    counts[name] = counts.get(name, 0) + 1
        sms = sorted(r["sm"] for r in rows)
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(r["max"] for r in rows),
                "sm_mhz_p10": sms[len(sms) // 10], "sm_mhz_p90": sms[(9 * len(sms)) // 10],
                "reasons": sorted(reasons), "reason_samples": counts, "samples": len(rows),
                "source": self.source, "power_w_max": max(r["power"] for r in rows)}


def _gpu_ids(local_rank):
    """(nvidia-smi index, NVML UUID) of this rank's GPU."""
    import torch

    phys = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
    index = phys[local_rank] if len(phys) > local_rank and phys[local_rank] else str(local_rank)
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(local_rank).uuid)
    except Exception:
        uuid = None
    return index, uuid


# ---------------------------------------------------------------------------- CPU oracle leg


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_sample(x, w, variant, rows_per_window):
    """Run the oracle on the last `rows_per_window` query rows of the first
    full group of every head: once forward only, once forward + backward (the
    oracle's backward recomputes each row's forward, so the backward's time is
    the difference).  Returns a dict: seconds (fwd, bwd, total = fwd + bwd),
    useful FLOPs of the sample on the metric's formula (fwd, bwd, total),
    threads, description."""
    import oracle

    G = w.G
    r0, r1 = G - rows_per_window, G
    t0 = time.perf_counter()
    oracle.attention(x["q"], x["k"], x["v"], G=G, variant=variant, n_valid=w.n_valid, rows=(r0, r1))
    t_fwd = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant, n_valid=w.n_valid, rows=(r0, r1))
    t_both = time.perf_counter() - t0
    t_bwd = max(t_both - t_fwd, 1e-9)
    # exact pairs of the sample (rows r0..r1 of every head), priced at 4·D (forward)
    # and 10·D (backward) per pair, then scaled by the metric's formula / exact ratio
    pc = pair_counts(w, variant)
    exact_pairs = 0
    for h in range(w.H):
        cls = 1 if (h >= w.H // 2 and variant != 2) else 0
        for i in range(r0, r1):
            lo = _row_lo(i, G, variant, cls, w.N)
            exact_pairs += i - lo + 1
    exact_pairs *= w.B
    ratio = 1.0
    if pc is not None:
        ratio = w.formula_flops(passes="fwd+bwd") / (w.B * (w.H // 2) * (pc[0] + pc[1]) * 14 * w.D)
    desc = ("oracle on query rows [%d, %d) of all %d heads of the workload's inputs (%d visited pairs), forward "
            "alone then forward + backward, priced on the metric's formula" % (r0, r1, w.B * w.H, exact_pairs))
    return {"s_fwd": t_fwd, "s_bwd": t_bwd, "s_total": t_fwd + t_bwd,
            "flops_fwd": exact_pairs * 4 * w.D * ratio, "flops_bwd": exact_pairs * 10 * w.D * ratio,
            "flops_total": exact_pairs * 14 * w.D * ratio, "threads": oracle.num_threads(), "desc": desc}


def cpu_baseline_line(smp):
    """The cpu_baseline object of a JSON line from one oracle_sample result."""
    return {"value": smp["flops_total"] / smp["s_total"] / 1e12, "unit": UNIT, "cores": smp["threads"],
            "kind": "oracle", "sample": smp["desc"], "cpu_model": cpu_model(),
            "seconds": {"fwd": smp["s_fwd"], "bwd": smp["s_bwd"], "total": smp["s_total"]},
            "tflops": {"fwd": smp["flops_fwd"] / smp["s_fwd"] / 1e12, "bwd": smp["flops_bwd"] / smp["s_bwd"] / 1e12}}


def _row_lo(i, G, variant, cls, N):
    s = G // 2
    if variant == 2:
        return 0
    if cls == 0:
        return (i // G) * G
    if i < s:
        return 0
    return s + ((i - s) // G) * G


def run_reference(args, rank, world):
    import torch  # noqa: F401

    from shifted_sparse_attention_b200 import synthetic

    if rank != 0:
        return
    w = synthetic.WORKLOADS[args.workload]
    variant = w.variants[0] if args.variant is None else args.variant
    x = synthetic.draw(w.B, w.N, w.H, w.D, seed=w.seed, sharpen_k=w.sharpen_k)
    rows = 16  # a ~1-2 s sample per step on a 16-core host
    for _ in range(args.warmup):
        oracle_sample(x, w, variant, rows)
    acc = None
    for _ in range(args.steps):
        smp = oracle_sample(x, w, variant, rows)
        if acc is None:
            acc = dict(smp)
        else:
            for key in ("s_fwd", "s_bwd", "s_total", "flops_fwd", "flops_bwd", "flops_total"):
                acc[key] += smp[key]
    cpu = cpu_baseline_line(acc)
    value = cpu["value"]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": acc["s_total"] / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config(w, variant),
        "cpu_baseline": cpu,
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _config(w, variant):
    return {"workload": w.name, "B": w.B, "N": w.N, "H": w.H, "D": w.D, "G": w.G, "shift": w.G // 2,
            "group_ratio": w.G / w.N, "n_valid": w.valid,
            "variant": {0: "strict", 1: "rolled", 2: "dense_causal"}[variant],
            "l2": _l2_note(w)}


def _fits_l2(w):
    return 4 * w.B * w.N * w.H * w.D * 2 <= 126e6


def _l2_note(w):
    """How a step's inputs relate to the 126 MB L2 (the timing rule: flush, or inputs larger than L2)."""
    each = w.B * w.N * w.H * w.D * 2
    if each > 126e6:
        return "inputs larger than L2 (each of Q/K/V/dO is %d MiB > 126 MB)" % (each >> 20)
    if 4 * each > 126e6:
        return ("inputs larger than L2 together (Q/K/V/dO %d MiB each, %d MiB in all > 126 MB; each pass streams "
                "all of them)" % (each >> 20, 4 * each >> 20))
    return ("inputs fit in L2 (%d MiB in all): L2 flushed before every step by a 256 MiB write outside the "
            "step's events" % (4 * each >> 20))


def _src_hash(name):
    return hashlib.sha256((ROOT / "shifted_sparse_attention_b200" / "csrc" / name).read_bytes()).hexdigest()[:16]


def _traffic(kernel, src, workload):
    """Per-launch DRAM bytes from the committed ncu summary, if taken on this exact
    kernel source and workload."""
    p = ROOT / "profiles" / "traffic.json"
    if not p.exists():
        return None
    t = json.loads(p.read_text())
    d = t.get(kernel)
    if not d or d.get("source_sha256_16") != _src_hash(src) or t.get("_workload") != workload:
        return None
    return d.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------- multi-rank host logic


def combine_ranks(ms, per, clocks, device):
    """Max over ranks of the timed region and of each kernel's time; clock
    summaries gathered to every rank (median of the ranks' medians, union of
    throttle reasons).  Works on any process group (nccl on GPUs, gloo on CPU)."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size()
    keys = list(per)
    t = torch.tensor([ms] + [per[k] for k in keys], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t[0].item())
    per = {k: float(t[1 + i].item()) for i, k in enumerate(keys)}
    gathered = [None] * world
    dist.all_gather_object(gathered, clocks)
    meds = [c["sm_mhz"] for c in gathered if c.get("sm_mhz") is not None]
    clocks = {"sm_mhz": statistics.median(meds) if meds else None,
              "sm_max_mhz": max((c.get("sm_max_mhz") or 0) for c in gathered) or None,
              "reasons": sorted(set(r for c in gathered for r in c.get("reasons", []))),
              "per_rank_sm_mhz": meds}
    return ms, per, clocks


def job_tflops(world, flops_per_rank_step, ms_step_max):
    """Whole-job throughput: every rank's useful FLOPs over the slowest rank's time."""
    return world * flops_per_rank_step / (ms_step_max * 1e-3) / 1e12


# ---------------------------------------------------------------------------- our arm


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from shifted_sparse_attention_b200 import binding as s2
    from shifted_sparse_attention_b200 import synthetic

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = synthetic.WORKLOADS[args.workload]
    variant = w.variants[0] if args.variant is None else args.variant
    B, N, H, D, G = w.B, w.N, w.H, w.D, w.G
    x = synthetic.draw(B, N, H, D, seed=w.seed + rank, sharpen_k=w.sharpen_k)
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "dout"))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    grads = (torch.empty_like(q), torch.empty_like(q), torch.empty_like(q))
    stored = not args.recompute_dq
    ws_bytes = (s2.s2attn_bwd_ds_workspace_size(B, N, H, D, G, variant) if stored
                else s2.s2attn_bwd_workspace_size(B, N, H, D))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    nv = w.n_valid
    docs = None
    if args.doc_len:
        if variant == 1 or w.valid != N:
            raise SystemExit("--doc-len supports the strict and dense variants without padding")
        ids = (torch.arange(N, device=dev, dtype=torch.int32) // args.doc_len).expand(B, N).contiguous()
        docs = s2.doc_bounds(ids)
    # RoPE prologue: rotate the step's raw Q/K at original positions (restarting per
    # packed document) with interpolation factor 1/4 into separate buffers
    q_in, k_in = q, k
    positions = None
    if args.rope:
        q_in, k_in = torch.empty_like(q), torch.empty_like(k)
        if args.doc_len:
            positions = (torch.arange(N, device=dev, dtype=torch.int32) % args.doc_len).expand(B, N).contiguous()

    nvtx = torch.cuda.nvtx  # ranges name each stage on a profiler's timeline

    def step(ev=None):
        if args.rope:
            if ev is not None:
                ev[5].record(stream)
            nvtx.range_push("s2 rope")
            s2.rope(q, k, positions, scale=0.25, out=(q_in, k_in))
            nvtx.range_pop()
        if ev is not None:
            ev[0].record(stream)
        nvtx.range_push("s2 forward")
        s2.forward(q_in, k_in, v, G, variant, nv, out=o, lse=lse, docs=docs)
        nvtx.range_pop()
        if ev is not None:
            ev[1].record(stream)
        nvtx.range_push("s2 backward")
        s2.backward(q_in, k_in, v, o, do, lse, G, variant, nv, grads=grads, workspace=ws, stages=s2.S2_BWD_PREPARE,
                    docs=docs, stored_ds=stored)
        if ev is not None:
            ev[2].record(stream)
        s2.backward(q_in, k_in, v, o, do, lse, G, variant, nv, grads=grads, workspace=ws, stages=s2.S2_BWD_DKDV,
                    docs=docs, stored_ds=stored)
        if ev is not None:
            ev[3].record(stream)
        s2.backward(q_in, k_in, v, o, do, lse, G, variant, nv, grads=grads, workspace=ws, stages=s2.S2_BWD_DQ,
                    docs=docs, stored_ds=stored)
        nvtx.range_pop()
        if ev is not None:
            ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    s2.check_status()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # inputs that fit in L2 together are flushed out of it before every step (a
    # 256 MiB write outside the step's events; the step time is then the sum of
    # the steps' own event spans)
    flush = _fits_l2(w)
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if flush else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(*_gpu_ids(local_rank)) as clk:
        time.sleep(0.2)  # let the sampler start before the timed region
        start.record(stream)
        for i in range(args.steps):
            if flush:
                flush_buf.zero_()
            step(evs[i])
        end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    s2.check_status()
    first = 5 if args.rope else 0
    ms = sum(e[first].elapsed_time(e[4]) for e in evs) if flush else start.elapsed_time(end)
    stages = (("fwd", 0, 1), ("bwd_prepare", 1, 2), ("bwd_dkdv", 2, 3), ("bwd_dq", 3, 4)) + (
        (("rope", 5, 0),) if args.rope else ())
    samples = {name: [e[a].elapsed_time(e[b]) for e in evs] for name, a, b in stages}
    per = {name: sum(t) / args.steps for name, t in samples.items()}
    # this rank's spread over the timed steps: median and minimum per pass
    per_spread = {name: {"median": statistics.median(t), "min": min(t)} for name, t in samples.items()}
    clocks = clk.summary()

    # e2e: the same step through the public API from pinned host buffers, copies included.
    # Every step copies its four inputs host -> device and its four results (o, dq,
    # dk, dv) device -> host.  The copies run on their own streams against two sets
    # of device buffers, so step i's results travel back while step i + 1 computes
    # and step i + 2's inputs arrive (the two directions of the link run at once);
    # the forward starts once q, k, v have landed (dout's copy overlaps it) and o
    # leaves right after the forward.  The timed region spans the first input copy
    # to the last result copy; 16 steps keep the pipeline's fill and drain (one
    # input copy, one step, one result copy) a small part of it.
    e2e = None
    if not args.no_e2e:
        e_steps = max(2, min(args.steps, 16))
        names_in, names_out = ("q", "k", "v", "dout"), ("o", "dq", "dk", "dv")
        host_in = {n: t.cpu().pin_memory() for n, t in (("q", q), ("k", k), ("v", v), ("dout", do))}
        host_out = [{n: torch.empty(q.shape, dtype=q.dtype, pin_memory=True) for n in names_out} for _ in range(2)]
        bufs = []
        for b in range(2):
            d = {n: (torch.empty_like(q) if b else t) for n, t in (("q", q), ("k", k), ("v", v), ("dout", do))}
            if args.rope:
                d["q_in"], d["k_in"] = torch.empty_like(q), torch.empty_like(k)
            d["o"] = torch.empty_like(q) if b else o
            d["lse"] = torch.empty_like(lse) if b else lse
            d["dq"], d["dk"], d["dv"] = (tuple(torch.empty_like(q) for _ in range(3)) if b else grads)
            bufs.append(d)
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev_qkv = [torch.cuda.Event() for _ in range(2)]
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_fwd = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_read = [torch.cuda.Event() for _ in range(2)]
        for e in ev_done + ev_read:
            e.record(stream)

        def e2e_step(i):
            b = i % 2
            d = bufs[b]
            s_in.wait_event(ev_done[b])  # step i - 2 no longer reads this buffer set
            with torch.cuda.stream(s_in):
                for n in ("q", "k", "v"):
                    d[n].copy_(host_in[n], non_blocking=True)
                ev_qkv[b].record(s_in)
                d["dout"].copy_(host_in["dout"], non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_qkv[b])
            stream.wait_event(ev_read[b])  # step i - 2's results have left this buffer set
            qi, ki = d["q"], d["k"]
            if args.rope:
                s2.rope(d["q"], d["k"], positions, scale=0.25, out=(d["q_in"], d["k_in"]))
                qi, ki = d["q_in"], d["k_in"]
            s2.forward(qi, ki, d["v"], G, variant, nv, out=d["o"], lse=d["lse"], docs=docs)
            ev_fwd[b].record(stream)
            stream.wait_event(ev_in[b])
            s2.backward(qi, ki, d["v"], d["o"], d["dout"], d["lse"], G, variant, nv, grads=(d["dq"], d["dk"], d["dv"]),
                        workspace=ws, docs=docs, stored_ds=stored)
            ev_done[b].record(stream)
            s_out.wait_event(ev_fwd[b])
            with torch.cuda.stream(s_out):
                host_out[b]["o"].copy_(d["o"], non_blocking=True)
            s_out.wait_event(ev_done[b])
            with torch.cuda.stream(s_out):
                for n in ("dq", "dk", "dv"):
                    host_out[b][n].copy_(d[n], non_blocking=True)
                ev_read[b].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        a, bev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s_in)
        stream.wait_event(a)
        s_out.wait_event(a)
        for i in range(e_steps):
            e2e_step(i)
        s_out.wait_stream(stream)
        bev.record(s_out)
        torch.cuda.synchronize()
        e2e_ms = a.elapsed_time(bev) / e_steps
        if world > 1:
            t = torch.tensor([e2e_ms], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e2e_ms = float(t.item())
        nbytes = q.numel() * q.element_size()
        e2e = {"value": world * w.formula_flops(passes="fwd+bwd") / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": 4 * nbytes, "d2h_bytes_per_step": 4 * nbytes, "ms_per_step": e2e_ms,
               "steps": e_steps, "overlap": "copies on two streams, two device buffer sets"}
        s2.check_status()

    if world > 1:
        ms, per, clocks = combine_ranks(ms, per, clocks, dev)

    # CPU oracle leg (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.doc_len:
        # 640 rows of every head: about 15 s of oracle work on the long workload
        cpu = cpu_baseline_line(oracle_sample({n: x[n] for n in x}, w, variant, min(640, w.G)))

    if rank != 0:
        return
    pk = peaks()
    ms_step = ms / args.steps
    pc = doc_pair_counts(w, variant, args.doc_len) if args.doc_len else pair_counts(w, variant)
    if pc is not None:
        pairs = w.B * (w.H // 2) * (pc[0] + pc[1])
    else:
        pairs = None
    # the metric's formula counts the grouping's causal work; under a document mask
    # the useful work is the exact visited pairs (14·D FLOPs each, forward + backward)
    flops_step = pairs * 14 * D if args.doc_len else w.formula_flops(passes="fwd+bwd")
    value = job_tflops(world, flops_step, ms_step)
    if e2e is not None and args.doc_len:
        e2e["value"] = world * flops_step / (e2e["ms_per_step"] * 1e-3) / 1e12
    # Algorithmic FLOPs per visited pair: forward 4·D (Q K^T, P V); dK/dV pass 8·D
    # (S, dP, dV, dK); dQ pass 2·D (dQ only: with the stored dS it reads dS, with the
    # recomputing form its S and dP products are overhead, not credited).
    per_pair = {"fwd": 4 * D, "bwd_dkdv": 8 * D, "bwd_dq": 2 * D}
    share = {"fwd": 1.0, "bwd_dkdv": 0.8, "bwd_dq": 0.2}
    knames = {"fwd": "s2_fwd_kernel", "bwd_dkdv": "s2_bwd_dkdv_kernel",
              "bwd_dq": "s2_bwd_dq_ds_kernel" if stored else "s2_bwd_dq_kernel"}
    srcs = {"fwd": "s2_fwd.cu", "bwd_dkdv": "s2_bwd.cu", "bwd_dq": "s2_bwd.cu"}
    # The peak a fraction is taken against: the burst figure (cuBLAS timed alone)
    # unless the timed region is as long as the sustained measurement's 4 s loop.
    timed_s = ms / 1e3
    sustained = timed_s >= 4.0
    peak = pk["bf16_sustained"] if sustained else pk["bf16_burst"]
    peak_kind = ("bf16 sustained: timed region %.2f s, as long as the sustained measurement's loop" % timed_s
                 if sustained else "bf16 burst: timed region %.2f s, shorter than the sustained measurement's "
                 "4 s loop" % timed_s) + ", %s" % pk["source"]
    kern = {}
    for kname in ("fwd", "bwd_dkdv", "bwd_dq"):
        algo_k = (pairs * per_pair[kname] if pairs is not None else
                  share[kname] * w.formula_flops(passes="fwd" if kname == "fwd" else "bwd"))
        ach = algo_k / (per[kname] * 1e-3) / 1e12
        kern[kname] = {"kernel": knames[kname], "avg_launch_ms": per[kname], "algorithmic_flops_per_launch": algo_k,
                       "achieved_tflops": ach, "frac": ach / peak}
    # dominant kernel: the longest of the forward, the dK/dV pass and the dQ pass
    dom = max(("fwd", "bwd_dkdv", "bwd_dq"), key=lambda k: per[k])
    roof = {"bound": "tensor", "kernel": knames[dom],
            "achieved": kern[dom]["achieved_tflops"], "peak": peak, "unit": "TFLOP/s",
            "frac": kern[dom]["achieved_tflops"] / peak, "peak_kind": peak_kind,
            "traffic": _traffic(knames[dom], srcs[dom], args.workload),
            "algorithmic_flops_per_launch": kern[dom]["algorithmic_flops_per_launch"], "avg_launch_ms": per[dom],
            "per_kernel": kern}
    sm = clocks.get("sm_mhz")
    if sm:
        # time x clock: the step in millions of SM cycles at the median clock seen
        clocks["step_mcycles_at_median"] = ms_step * 1e-3 * sm
    line = {
        "metric": METRIC + (" (document mask: exact visited pairs)" if args.doc_len else ""),
        "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(_config(w, variant), parallelism="replicas%d" % world if world > 1 else "single",
                       **({"doc_len": args.doc_len} if args.doc_len else {})),
        "pct_of_peak": {"bf16_burst": value / world / pk["bf16_burst"],
                        "bf16_sustained": value / world / pk["bf16_sustained"],
                        "nominal_2250": value / world / 2250.0},
        "kernel_ms": per,
        "kernel_ms_rank0_spread": per_spread,
        "useful_flops_per_step": flops_step,
        "exact_pair_tflops": (world * pairs * 14 * D / (ms_step * 1e-3) / 1e12) if pairs else None,
        "clocks": clocks,
        "e2e": e2e,
        "gpu_launches": (5 if args.rope else 4) * args.steps,
        "roofline": roof,
        "cpu_baseline": cpu,
    }
    line["config"]["backward"] = ("stored dS (dQ pass reads the dK/dV pass's dS tiles; workspace %.2f GB)"
                                  % (ws_bytes / 1e9) if stored else "recomputing dQ pass (workspace %.1f MB)"
                                  % (ws_bytes / 1e6))
    if w.valid != w.N and not args.doc_len:
        # raw throughput prices the padded length (what the kernels' shapes are),
        # effective the valid length (the metric); their ratio is the useful share
        raw_flops = 7.0 * w.B * w.H * w.N * w.G * D
        line["raw_vs_effective"] = {"raw_tflops_padded_n": world * raw_flops / (ms_step * 1e-3) / 1e12,
                                    "effective_tflops_n_valid": value, "effective_ratio": w.valid / w.N,
                                    "padded_n": w.N, "n_valid": w.valid}
    if pairs and not args.doc_len:
        # executed MMA work over the exact useful work: every visited 128 x 128 tile is
        # multiplied in full, so the excess is the masked half of the diagonal tiles
        tp = w.B * (w.H // 2) * (stored_tile_pairs(w, variant, 0) + stored_tile_pairs(w, variant, 1))
        line["executed_over_useful"] = tp * 128 * 128 / pairs
    if stored and not args.doc_len:
        # the stored-dS dQ pass is HBM-bound: it reads one 32 KB dS tile per computed
        # tile pair, the K tiles and writes dq
        tiles = w.B * (w.H // 2) * (stored_tile_pairs(w, variant, 0) + stored_tile_pairs(w, variant, 1))
        dq_bytes = tiles * 128 * 128 * 2 + 2 * q.numel() * q.element_size()
        ach = dq_bytes / (per["bwd_dq"] * 1e-3) / 1e9
        line["dq_roofline"] = {"bound": "hbm", "kernel": "s2_bwd_dq_ds_kernel", "achieved": ach, "peak": pk["hbm_gbs"],
                               "unit": "GB/s", "frac": ach / pk["hbm_gbs"], "algorithmic_bytes_per_launch": dq_bytes,
                               "stored_ds_tiles": tiles, "avg_launch_ms": per["bwd_dq"],
                               "traffic": _traffic("s2_bwd_dq_ds_kernel", "s2_bwd.cu", args.workload)}
    if args.rope:
        # HBM-bound prologue: reads and writes Q and K once (plus the positions)
        rope_bytes = 2 * 2 * q.numel() * q.element_size() + (positions.numel() * 4 if positions is not None else 0)
        ach = rope_bytes / (per["rope"] * 1e-3) / 1e9
        line["config"]["rope"] = {"scale": 0.25, "base": 10000.0,
                                  "positions": "restart per document" if positions is not None else "0..N-1"}
        line["rope_roofline"] = {"bound": "hbm", "kernel": "s2_rope_kernel", "achieved": ach, "peak": pk["hbm_gbs"],
                                 "unit": "GB/s", "frac": ach / pk["hbm_gbs"], "algorithmic_bytes_per_launch": rope_bytes,
                                 "avg_launch_ms": per["rope"],
                                 "traffic": _traffic("s2_rope_kernel", "s2_rope.cu", args.workload)}
    print(json.dumps(line), flush=True)


def sp_layout(N, G, n_valid, world):
    """Shard length and each rank's valid rows when a sequence of N (padded) rows,
    n_valid of them valid, is cut into `world` G-aligned shards: rank r holds
    original positions [rL, rL + L).  Padding may sit only on the last rank
    (the rank kernels' rule), so every other rank must be full."""
    if world < 1 or N % (world * G):
        raise ValueError("N=%d is not a multiple of world x G = %d x %d" % (N, world, G))
    L = N // world
    valid = [max(0, min(L, n_valid - r * L)) for r in range(world)]
    if any(v != L for v in valid[:-1]) or valid[-1] < 1:
        raise ValueError("the padding of n_valid=%d does not fall on the last of %d shards of %d rows" % (
            n_valid, world, L))
    return L, valid


def run_sp(args, rank, world, local_rank):
    """Sequence parallelism over the torchrun ranks ("4.1.2 · LongLoRA:
    用S²-Attn完成长上下文微调" §1.1, Sequence Parallel通信).  Each rank holds the
    G-aligned shard [rL, rL + L) of the workload in extended buffers (halo
    rows first).  One step per rank: the K/V halo exchange (pack, NCCL
    send/receive with both neighbours, unpack), the rank's forward and its
    stored-dS backward, and the halo rows' gradients back to their owner.
    value = the whole sequence's useful FLOPs / the slowest rank's step time
    (strong scaling: the total work is fixed as ranks are added)."""
    import torch
    import torch.distributed as dist

    from shifted_sparse_attention_b200 import binding as s2
    from shifted_sparse_attention_b200 import sp
    from shifted_sparse_attention_b200 import synthetic

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = synthetic.WORKLOADS[args.workload]
    variant = w.variants[0] if args.variant is None else args.variant
    if variant not in (0, 1):
        raise SystemExit("--sp runs the strict and rolled variants")
    B, N, H, D, G = w.B, w.N, w.H, w.D, w.G
    L, valid = sp_layout(N, G, w.valid, world)
    s = G // 2
    nv = valid[rank]
    x = synthetic.draw(B, N, H, D, seed=w.seed, sharpen_k=w.sharpen_k)
    t = {}
    for name in ("q", "k", "v", "dout"):
        e = sp.extended(B, L, H, D, G, dev)
        e.zero_()
        sp.shard(e, G).copy_(x[name][:, rank * L:(rank + 1) * L])
        t[name] = e
    del x
    attn = sp.SequenceParallelS2Attn(G, variant)
    o = torch.empty_like(t["q"])
    lse = torch.empty((B, H, s + L), dtype=torch.float32, device=dev)
    grads = tuple(torch.empty_like(t["q"]) for _ in range(3))
    ws_bytes = s2.s2attn_sp_ds_workspace_size(B, L, H, D, G, variant, rank, world)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        attn.exchange_kv(t["k"], t["v"])
        if ev is not None:
            ev[1].record(stream)
        attn.forward(t["q"], t["k"], t["v"], n_valid=nv, out=o, lse=lse, exchange=False)
        if ev is not None:
            ev[2].record(stream)
        attn.backward(t["q"], t["k"], t["v"], o, t["dout"], lse, n_valid=nv, grads=grads, workspace=ws,
                      exchange=False, stored_ds=True)
        if ev is not None:
            ev[3].record(stream)
        attn.exchange_grad(grads[1], grads[2])
        if ev is not None:
            ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    s2.check_status()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(*_gpu_ids(local_rank)) as clk:
        time.sleep(0.2)
        for i in range(args.steps):
            step(evs[i])
        torch.cuda.synchronize()
    dist.barrier()
    s2.check_status()
    ms = sum(e[0].elapsed_time(e[4]) for e in evs)
    parts = (("halo_kv", 0, 1), ("fwd", 1, 2), ("bwd", 2, 3), ("halo_grad", 3, 4))
    per = {name: sum(e[a].elapsed_time(e[b]) for e in evs) / args.steps for name, a, b in parts}
    ms, per, clocks = combine_ranks(ms, per, clk.summary(), dev)
    if rank != 0:
        return
    pk = peaks()
    ms_step = ms / args.steps
    flops = w.formula_flops(passes="fwd+bwd")
    value = flops / (ms_step * 1e-3) / 1e12
    to0, frm0 = sp.peers(0, world, variant)
    line = {
        "metric": METRIC + " (sequence parallel over %d GPUs)" % world,
        "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": dict(_config(w, variant), parallelism="sp%d" % world, shard_rows=L,
                       backward="stored dS", halo="NCCL point-to-point, %d bytes per direction"
                       % s2.s2attn_sp_halo_bytes(B, H, D, G)),
        "pct_of_peak": {"bf16_burst": value / world / pk["bf16_burst"],
                        "bf16_sustained": value / world / pk["bf16_sustained"]},
        "stage_ms_max_over_ranks": per,
        "clocks": clocks,
        # per step and rank: halo pack/unpack kernels where the rank sends/receives,
        # the forward, the backward's three stages
        "gpu_launches": args.steps * sum(
            4 + (2 if sp.peers(r, world, variant)[0] is not None else 0)
            + (2 if sp.peers(r, world, variant)[1] is not None else 0) for r in range(world)),
    }
    print(json.dumps(line), flush=True)


def run_sp_emulated(args):
    """Sequence-parallel step of W ranks, run one rank after another on this GPU.

    Each rank holds a G-aligned shard of L = N / W rows of the workload in
    extended buffers; per step and rank: K/V halo from the previous rank
    (pack + unpack kernels, the message handed over in memory where the
    collective layer would send it), the rank's forward and backward, and the
    halo gradients back (pack + accumulate).  value = the whole sequence's
    useful FLOPs / the summed device time of all ranks (comparable with the
    single-GPU line); per_rank_ms is what each GPU of a W-GPU job would spend
    on kernels, without the transfer itself (estimated from the halo bytes at
    the measured 770 GB/s peer bandwidth)."""
    import torch

    from shifted_sparse_attention_b200 import binding as s2
    from shifted_sparse_attention_b200 import sp
    from shifted_sparse_attention_b200 import synthetic

    torch.cuda.set_device(0)
    w = synthetic.WORKLOADS[args.workload]
    variant = w.variants[0] if args.variant is None else args.variant
    B, N, H, D, G, W = w.B, w.N, w.H, w.D, w.G, args.sp_emulate
    if N % (W * G) or w.valid != N or variant not in (0, 1):
        raise SystemExit("--sp-emulate needs N divisible by W·G, no padding, strict or rolled")
    L, s = N // W, G // 2
    x = synthetic.draw(B, N, H, D, seed=w.seed, sharpen_k=w.sharpen_k)
    ops = sp.HaloOps()
    ranks = []
    for r in range(W):
        t = {}
        for name in ("q", "k", "v", "dout"):
            e = sp.extended(B, L, H, D, G, "cuda")
            e.zero_()
            sp.shard(e, G).copy_(x[name][:, r * L:(r + 1) * L])
            t[name] = e
        t["o"] = torch.empty_like(t["q"])
        t["lse"] = torch.empty((B, H, s + L), dtype=torch.float32, device="cuda")
        t["g"] = tuple(torch.empty_like(t["q"]) for _ in range(3))
        ws_bytes = (s2.s2attn_bwd_workspace_size(B, s + L, H, D) if args.recompute_dq
                    else s2.s2attn_sp_ds_workspace_size(B, L, H, D, G, variant, r, W))
        t["ws"] = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        ranks.append(t)
    del x
    msg = torch.empty((2, B, s, H // 2, D), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()

    def rank_step(r, ev=None):
        t = ranks[r]
        to, frm = sp.peers(r, W, variant)
        if ev is not None:
            ev[0].record(stream)
        if frm is not None:
            f = ranks[frm]
            ops.pack(f["k"], f["v"], msg, B, L, H, D, G, s2.S2_SP_KV)
            ops.unpack(msg, t["k"], t["v"], B, L, H, D, G, s2.S2_SP_KV)
        if ev is not None:
            ev[1].record(stream)
        s2._check(s2.s2attn_sp_fwd(t["q"], t["k"], t["v"], t["o"], t["lse"], B, L, H, D, G, L, variant, r, W))
        dq, dk, dv = t["g"]
        s2._check(s2.s2attn_sp_bwd_stages(t["q"], t["k"], t["v"], t["o"], t["dout"], t["lse"], dq, dk, dv, B, L, H,
                                          D, G, L, variant, r, W, t["ws"], t["ws"].numel(),
                                          s2.S2_BWD_ALL if args.recompute_dq else s2.S2_BWD_ALL_DS))
        if ev is not None:
            ev[2].record(stream)
        if frm is not None:
            f = ranks[frm]
            ops.pack(dk, dv, msg, B, L, H, D, G, s2.S2_SP_GRAD)
            ops.unpack(msg, f["g"][1], f["g"][2], B, L, H, D, G, s2.S2_SP_GRAD)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        for r in range(W):
            rank_step(r)
    torch.cuda.synchronize()
    s2.check_status()
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(W)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(*_gpu_ids(0)) as clk:
        time.sleep(0.6)
        start.record(stream)
        for i in range(args.steps):
            for r in range(W):
                rank_step(r, evs[i][r])
        end.record(stream)
        torch.cuda.synchronize()
    s2.check_status()
    ms_step = start.elapsed_time(end) / args.steps
    per_rank = [sum(e[r][0].elapsed_time(e[r][3]) for e in evs) / args.steps for r in range(W)]
    halo = [sum(e[r][0].elapsed_time(e[r][1]) + e[r][2].elapsed_time(e[r][3]) for e in evs) / args.steps
            for r in range(W)]
    flops = w.formula_flops(passes="fwd+bwd")
    pk = peaks()
    v_kv = s2.s2attn_sp_halo_bytes(B, H, D, G)
    value = flops / (ms_step * 1e-3) / 1e12
    line = {
        "metric": METRIC + " (sequence parallel, ranks emulated in turn on one GPU)",
        "value": value, "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": dict(_config(w, variant), parallelism="sp%d-emulated" % W, shard_rows=L,
                       backward="recomputing dQ pass" if args.recompute_dq else "stored dS"),
        "pct_of_peak": {"bf16_burst": value / pk["bf16_burst"], "bf16_sustained": value / pk["bf16_sustained"]},
        "sp": {"world": W, "per_rank_ms": per_rank, "halo_kernels_ms": halo,
               "halo_bytes_per_direction": v_kv,
               "halo_transfer_us_at_770GBps": v_kv / 770e9 * 1e6,
               "ideal_w_gpu_step_ms": max(per_rank) + 2 * v_kv / 770e9 * 1e3},
        "clocks": clk.summary(),
        "gpu_launches": args.steps * sum((6 if sp.peers(r, W, variant)[1] is not None else 2) + 2 for r in range(W)),
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.sp_emulate:
        if world > 1:
            raise SystemExit("--sp-emulate runs on one GPU")
        run_sp_emulated(args)
        return
    if world > 1 or args.sp:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        if world == 1:  # --sp on one GPU: a process group of one rank
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("MASTER_PORT", "29531")
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.sp:
            run_sp(args, rank, world, local_rank)
        else:
            run_ours(args, rank, world, local_rank)
    finally:
        if world > 1 or args.sp:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
