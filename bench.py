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
    ap.add_argument("--fwd-pairs", type=int, default=None, choices=[0, 1],
                    help="forward over CTA pairs (tcgen05 cta_group::2) on or off")
    ap.add_argument("--dkdv-half", type=int, default=None, choices=[0, 1],
                    help="dK/dV pass over half query tiles with double-buffered scores, on or off")
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
    """Exact visited (query, key) pairs per head class, closed forms of the grouping."""
    N, G, nv = w.N, w.G, w.valid
    tri = lambda L: L * (L + 1) // 2
    if nv != N:
        return None
    s, M = G // 2, N // G
    if variant == 2:
        return tri(N), tri(N)
    c0 = M * tri(G)
    c1 = c0 if variant == 1 else 2 * tri(s) + (M - 1) * tri(G)
    return c0, c1


# ---------------------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
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
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                              ("swp", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in rows), "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows),
                "power_w_max": max(r["power"] for r in rows)}


# ---------------------------------------------------------------------------- CPU oracle leg


def oracle_sample(x, w, variant, rows_per_window):
    """Run the oracle on the last `rows_per_window` query rows of the first
    full group of every head (fwd + bwd); return (seconds, useful FLOPs of the
    sample on the metric's formula, threads, description)."""
    import oracle

    G = w.G
    r0, r1 = G - rows_per_window, G
    t0 = time.perf_counter()
    oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant, n_valid=w.n_valid, rows=(r0, r1))
    dt = time.perf_counter() - t0
    # exact pairs of the sample (rows r0..r1 of every head), priced at 14·D per pair
    # (4D forward + 10D backward), then scaled by the metric's formula / exact ratio
    pc = pair_counts(w, variant)
    exact_pairs = 0
    for h in range(w.H):
        cls = 1 if (h >= w.H // 2 and variant != 2) else 0
        for i in range(r0, r1):
            lo = _row_lo(i, G, variant, cls, w.N)
            exact_pairs += i - lo + 1
    exact_pairs *= w.B
    flops_exact = exact_pairs * 14 * w.D
    ratio = 1.0
    if pc is not None:
        ratio = w.formula_flops(passes="fwd+bwd") / (w.B * (w.H // 2) * (pc[0] + pc[1]) * 14 * w.D)
    desc = ("oracle fwd+bwd on query rows [%d, %d) of all %d heads of the workload's inputs "
            "(%d visited pairs), priced on the metric's formula" % (r0, r1, w.B * w.H, exact_pairs))
    return dt, flops_exact * ratio, oracle.num_threads(), desc


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
    total_t, total_f = 0.0, 0.0
    for _ in range(args.steps):
        dt, fl, threads, desc = oracle_sample(x, w, variant, rows)
        total_t += dt
        total_f += fl
    value = total_f / total_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_t / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config(w, variant),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _config(w, variant):
    return {"workload": w.name, "B": w.B, "N": w.N, "H": w.H, "D": w.D, "G": w.G, "shift": w.G // 2,
            "group_ratio": w.G / w.N, "n_valid": w.valid,
            "variant": {0: "strict", 1: "rolled", 2: "dense_causal"}[variant],
            "l2": _l2_note(w)}


def _l2_note(w):
    """How a step's inputs relate to the 126 MB L2 (the timing rule: flush, or inputs larger than L2)."""
    each = w.B * w.N * w.H * w.D * 2
    if each > 126e6:
        return "inputs larger than L2 (each of Q/K/V/dO is %d MiB > 126 MB)" % (each >> 20)
    if 4 * each > 126e6:
        return ("inputs larger than L2 together (Q/K/V/dO %d MiB each, %d MiB in all > 126 MB; each pass streams "
                "all of them)" % (each >> 20, 4 * each >> 20))
    return "inputs fit in L2 (%d MiB in all) and are not flushed between steps: not a timing workload" % (
        4 * each >> 20)


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
    if args.fwd_pairs is not None:
        s2.set_fwd_pairs(bool(args.fwd_pairs))
    if args.dkdv_half is not None:
        s2.set_dkdv_half(bool(args.dkdv_half))
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
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    phys = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
    gpu_index = phys[local_rank] if len(phys) > local_rank and phys[local_rank] else str(local_rank)
    with ClockSampler(gpu_index) as clk:
        time.sleep(0.6)  # let nvidia-smi start sampling before the timed region
        start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    s2.check_status()
    ms = start.elapsed_time(end)
    stages = (("fwd", 0, 1), ("bwd_prepare", 1, 2), ("bwd_dkdv", 2, 3), ("bwd_dq", 3, 4)) + (
        (("rope", 5, 0),) if args.rope else ())
    samples = {name: [e[a].elapsed_time(e[b]) for e in evs] for name, a, b in stages}
    per = {name: sum(t) / args.steps for name, t in samples.items()}
    # this rank's spread over the timed steps (the survey's protocol: median and minimum per pass)
    per_spread = {name: {"median": statistics.median(t), "min": min(t)} for name, t in samples.items()}
    clocks = clk.summary()

    # e2e: the same step through the public API from pinned host buffers, copies included.
    # Every step copies its four inputs host -> device and its four results (o, dq,
    # dk, dv) device -> host.  The copies run on their own streams against two sets
    # of device buffers, so step i's results travel back while step i + 1 computes
    # and step i + 2's inputs arrive (the two directions of the link run at once);
    # the timed region spans the first input copy to the last result copy.
    e2e = None
    if not args.no_e2e:
        e_steps = max(2, min(args.steps, 6))
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
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_read = [torch.cuda.Event() for _ in range(2)]
        for e in ev_done + ev_read:
            e.record(stream)

        def e2e_step(i):
            b = i % 2
            d = bufs[b]
            s_in.wait_event(ev_done[b])  # step i - 2 no longer reads this buffer set
            with torch.cuda.stream(s_in):
                for n in names_in:
                    d[n].copy_(host_in[n], non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_read[b])  # step i - 2's results have left this buffer set
            qi, ki = d["q"], d["k"]
            if args.rope:
                s2.rope(d["q"], d["k"], positions, scale=0.25, out=(d["q_in"], d["k_in"]))
                qi, ki = d["q_in"], d["k_in"]
            s2.forward(qi, ki, d["v"], G, variant, nv, out=d["o"], lse=d["lse"], docs=docs)
            s2.backward(qi, ki, d["v"], d["o"], d["dout"], d["lse"], G, variant, nv, grads=(d["dq"], d["dk"], d["dv"]),
                        workspace=ws, docs=docs, stored_ds=stored)
            ev_done[b].record(stream)
            s_out.wait_event(ev_done[b])
            with torch.cuda.stream(s_out):
                for n in names_out:
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
        dt, fl, threads, desc = oracle_sample({n: x[n] for n in x}, w, variant, 256)
        cpu = {"value": fl / dt / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc,
               "seconds": dt}

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
    # dominant kernel: the longest of the forward, the dK/dV pass and the dQ pass.
    # Algorithmic FLOPs per visited pair: forward 4·D (Q K^T, P V); dK/dV pass
    # 8·D (S, dP, dV, dK); dQ pass 2·D (dQ only: its S and dP are recomputed).
    dom = max(("fwd", "bwd_dkdv", "bwd_dq"), key=lambda k: per[k])
    per_pair = {"fwd": 4 * D, "bwd_dkdv": 8 * D, "bwd_dq": 2 * D}[dom]
    share = {"fwd": 1.0, "bwd_dkdv": 0.8, "bwd_dq": 0.2}[dom]
    algo = pairs * per_pair if pairs is not None else share * w.formula_flops(passes="fwd" if dom == "fwd" else "bwd")
    achieved = algo / (per[dom] * 1e-3) / 1e12
    src = {"fwd": "s2_fwd.cu", "bwd_dkdv": "s2_bwd.cu", "bwd_dq": "s2_bwd.cu"}[dom]
    kname = {"fwd": "s2_fwd_kernel", "bwd_dkdv": "s2_bwd_dkdv_kernel",
             "bwd_dq": "s2_bwd_dq_ds_kernel" if stored else "s2_bwd_dq_kernel"}[dom]
    roof = {"bound": "tensor", "kernel": kname,
            "achieved": achieved, "peak": pk["bf16_sustained"], "unit": "TFLOP/s",
            "frac": achieved / pk["bf16_sustained"],
            "peak_kind": "bf16 sustained (kernel timed inside a long step loop), %s" % pk["source"],
            "traffic": _traffic(kname, src, args.workload),
            "algorithmic_flops_per_launch": algo, "avg_launch_ms": per[dom]}
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
    with ClockSampler(os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")[0] or "0") as clk:
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
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
