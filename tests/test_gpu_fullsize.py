"""Parity at the workloads' full sizes, on sampled outputs (needs a B200).

Each workload runs through the C ABI exactly as bench.py launches it (one
forward, then the backward's three stages, with the stored-dS dQ pass as
bench.py times it, and again with the recomputing dQ pass) on the full
seeded inputs.  The float64 oracle then recomputes windows of 64 query rows
for a few heads of each class: at segment starts, at the end of every
segment (where the window also holds every query that sees the window's
keys, so dK and dV are complete there), around the shifted boundaries and
around the ragged valid length.

Tolerances take no value from the CUDA output.  The gradient bound is scaled
by the tensor's max-norm, taken as the oracle's largest |value| over all the
windows of the workload (at most the true max-norm, so the check is at least
as strict as the rule).  Two more checks cover the whole tensors:

* on the sampled windows, the GPU tensor's max-norm agrees with the oracle's
  within the 1e-2 bound;
* every segment of every head satisfies two identities of the gradient
  formula ("4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §3): the softmax rows sum
  to one, so the sum of dV over a segment's keys equals the sum of dO over
  its valid queries, and sum_j dS_ij = g_i·o_i - Delta_i = 0, so dK sums to
  zero over a segment.  The residual per segment and column must stay within
  the mean bound applied to that segment (1e-3 x max-norm x its key count).
"""
from __future__ import annotations

import functools

import numpy as np
import pytest
import torch

import oracle
from shifted_sparse_attention_b200 import binding as s2
from shifted_sparse_attention_b200 import synthetic
from tests.seg_layout import segments
from tests.tolerance import G_MAX, G_MEAN, check_grad, check_lse, check_o, to_np

pytestmark = pytest.mark.gpu

W = 64  # rows per window


@functools.lru_cache(maxsize=1)
def _inputs(B, N, H, D, seed, sharpen):
    return synthetic.draw(B, N, H, D, seed=seed, sharpen_k=sharpen)


def _segments(w, variant, cls):
    return segments(w.N, w.G, variant, cls)


def _windows(w, variant, cls):
    """(r0, r1, grads_complete) windows of original positions for one head class."""
    N, G, nv = w.N, w.G, w.valid
    s = G // 2
    out = []
    if variant == 2:  # one causal segment: only the last window holds all queries of its keys
        starts = [0, N // 2]
    elif cls == 0:
        starts = [0, G]
    elif variant == 0:  # strict shifted: short head [0, s), groups [s + kG, s + kG + G), tail [N - s, N)
        starts = [0, s, s + G]
    else:  # rolled shifted: the wrap group is [N - s, N) then [0, s)
        starts = [N - s, s, s + G]
    for a in starts:
        out.append((a, a + W, False))
    for seg in _segments(w, variant, cls):  # the last rows of every segment: complete dK, dV
        e = seg[-1][1]
        out.append((e - W, e, True))
    if nv < N:  # the ragged boundary: last valid rows (complete grads) and first padded rows
        out.append((nv - W, nv, True))
        out.append((nv - W // 2, nv + W // 2, False))
    out = [(max(0, a), min(N, b), c) for a, b, c in out if b - a > 0 and a < nv]
    return sorted(set(out))


@functools.lru_cache(maxsize=64)
def _oracle_window(name, variant, r0, r1, bhs):
    w = synthetic.WORKLOADS[name]
    x = _inputs(w.B, w.N, w.H, w.D, w.seed, w.sharpen_k)
    return oracle.attention_window(x["q"], x["k"], x["v"], x["dout"], G=w.G, variant=variant, rows=(r0, r1),
                                   heads=list(bhs), n_valid=w.n_valid)


def _check_segment_identities(w, variant, x, dk, dv, ref_max):
    """Per segment of every head: sum of dV over its keys = sum of dO over its valid
    queries, and the sum of dK over its keys = 0 (float64 sums of the bf16 values)."""
    nv = w.valid
    g = x["dout"].double()
    g[:, nv:] = 0  # loss mask: padded rows carry no output gradient
    dkf, dvf = dk.double(), dv.double()
    worst = {"dk": 0.0, "dv": 0.0}
    for h in range(w.H):
        cls = 0 if variant == 2 else int(h >= w.H // 2)
        for seg in _segments(w, variant, cls):
            n_keys = sum(max(0, min(b, nv) - a) for a, b in seg)
            if n_keys == 0:
                continue
            sdv = sum(dvf[:, a:b, h].sum(1) for a, b in seg)
            sg = sum(g[:, a:b, h].sum(1) for a, b in seg)
            sdk = sum(dkf[:, a:b, h].sum(1) for a, b in seg)
            for name, r in (("dv", (sdv - sg).abs().max().item()), ("dk", sdk.abs().max().item())):
                bound = n_keys * G_MEAN * ref_max[name]
                worst[name] = max(worst[name], r / (n_keys * ref_max[name]))
                assert r <= bound, "%s segment identity: residual %.4g > %.4g (head %d, segment %s)" % (
                    name, r, bound, h, seg)
    return worst


def _check_workload(name, variant, stored=True):
    w = synthetic.WORKLOADS[name]
    x = _inputs(w.B, w.N, w.H, w.D, w.seed, w.sharpen_k)
    dev = {n: t.cuda() for n, t in x.items()}
    o, lse = s2.forward(dev["q"], dev["k"], dev["v"], w.G, variant, w.n_valid)
    dq, dk, dv = s2.backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, w.G, variant, w.n_valid,
                             stored_ds=stored)
    torch.cuda.synchronize()
    s2.check_status()
    del dev
    res = {n: t.cpu() for n, t in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv))}
    del o, lse, dq, dk, dv
    torch.cuda.empty_cache()
    for n in ("o", "dq", "dk", "dv"):
        assert torch.isfinite(res[n]).all(), "%s holds a non-finite value" % n

    H, B = w.H, w.B
    if variant == 2:
        head_sets = {0: [0, H - 1]}
    else:
        head_sets = {0: [0, H // 2 - 1], 1: [H // 2, H - 1]}
    # every oracle window first: the gradient scale is the oracle's maximum over all of them
    jobs = []
    for cls, hs in head_sets.items():
        bhs = tuple((B - 1 if i % 2 else 0) * H + h for i, h in enumerate(hs))
        for r0, r1, complete in _windows(w, variant, cls):
            jobs.append((bhs, r0, r1, complete, _oracle_window(name, variant, r0, r1, bhs)))
    ref_max = {"dq": 0.0, "dk": 0.0, "dv": 0.0}
    for bhs, r0, r1, complete, ref in jobs:
        nv_rows = max(0, min(r1, w.valid) - r0)
        ref_max["dq"] = max(ref_max["dq"], float(np.abs(ref["dq"][:, :nv_rows]).max()) if nv_rows else 0.0)
        if complete:
            for n in ("dk", "dv"):
                ref_max[n] = max(ref_max[n], float(np.abs(ref[n]).max()))
    assert all(v > 0 for v in ref_max.values()), ref_max

    gpu_max = {"dq": 0.0, "dk": 0.0, "dv": 0.0}
    for bhs, r0, r1, complete, ref in jobs:
        for t, bh in enumerate(bhs):
            b, h = divmod(bh, H)
            where = "%s variant %d head %d rows [%d, %d)" % (name, variant, h, r0, r1)
            check_o(res["o"][b, r0:r1, h], ref["o"][t], where)
            check_lse(res["lse"][b, h, r0:r1], ref["lse"][t], where)
            nv_rows = max(0, min(r1, w.valid) - r0)
            if nv_rows:
                got = to_np(res["dq"][b, r0:r0 + nv_rows, h])
                check_grad("dq", got, ref["dq"][t][:nv_rows], where, ref_max["dq"])
                gpu_max["dq"] = max(gpu_max["dq"], float(np.abs(got).max()))
            if r1 > w.valid:
                assert (to_np(res["dq"][b, max(r0, w.valid):r1, h]) == 0).all(), where
                assert (to_np(res["dk"][b, max(r0, w.valid):r1, h]) == 0).all(), where
            if complete:
                for n in ("dk", "dv"):
                    got = to_np(res[n][b, r0:r1, h])
                    check_grad(n, got, ref[n][t], where, ref_max[n])
                    gpu_max[n] = max(gpu_max[n], float(np.abs(got).max()))
    # the max-norm itself, over the same elements
    for n in ref_max:
        assert abs(gpu_max[n] - ref_max[n]) <= G_MAX * ref_max[n], (n, gpu_max[n], ref_max[n])
    _check_segment_identities(w, variant, x, res["dk"], res["dv"], ref_max)


PATHS = pytest.mark.parametrize("stored", [True, False], ids=["stored_ds", "recompute"])


@PATHS
@pytest.mark.parametrize("variant", [0, 1])
def test_llama7b_layer_n8192_g2048(variant, stored):
    _check_workload("llama7b_n8192_g2048", variant, stored)


@PATHS
def test_long_context_n32768_g8192(stored):
    _check_workload("long_n32768_g8192", 0, stored)


@PATHS
def test_long_context_head_dim_64(stored):
    _check_workload("long_n32768_g8192_d64", 0, stored)


@PATHS
@pytest.mark.parametrize("name", ["sweep_n12288_g6144", "sweep_n12288_g3072", "sweep_n12288_g2048",
                                  "sweep_n12288_g1536"])
def test_group_ratio_sweep(name, stored):
    _check_workload(name, 0, stored)


@PATHS
def test_group_ratio_sweep_full_causal(stored):
    _check_workload("sweep_n12288_full", 2, stored)


@PATHS
def test_ragged_tail_n100000(stored):
    _check_workload("ragged_n100000_g8192", 0, stored)


def test_tensors_beyond_2_31_elements():
    """Maximum sizes: B1 N131072 H132 D128 G8192, 2.2e9 elements (4.4 GB) per
    tensor, so any element offset kept in 32 bits would wrap.  The forward and
    the recomputing backward (the stored dS would need about 140 GB here) run
    through the C ABI; the oracle checks windows of the first and last heads of
    each class at the start, in the middle and at the end of the sequence, where
    the offsets are largest."""
    B, N, H, D, G, variant = 1, 131072, 132, 128, 8192, 0
    assert B * N * H * D > 2 ** 31
    x = synthetic.draw(B, N, H, D, seed=31)
    dev = {n: t.cuda() for n, t in x.items()}
    o, lse = s2.forward(dev["q"], dev["k"], dev["v"], G, variant)
    dq, dk, dv = s2.backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, G, variant)
    torch.cuda.synchronize()
    s2.check_status()
    for name, t in (("o", o), ("dq", dq), ("dk", dk), ("dv", dv)):
        assert bool(torch.isfinite(t).all()), name
    s = G // 2
    heads = (0, H // 2 - 1, H // 2, H - 1)
    # class-0 segment ends at multiples of G; class-1 (strict) at s + kG and at N
    windows = [(0, W, False), (N // 2 - W, N // 2, True), (N // 2 + s - W, N // 2 + s, True), (N - W, N, True)]
    jobs, ref_max = [], {"dq": 0.0, "dk": 0.0, "dv": 0.0}
    for r0, r1, at_end in windows:
        ref = oracle.attention_window(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant, rows=(r0, r1),
                                      heads=list(heads))
        jobs.append((r0, r1, at_end, ref))
        ref_max["dq"] = max(ref_max["dq"], float(np.abs(ref["dq"]).max()))
        for t, h in enumerate(heads):
            cls = int(h >= H // 2)
            seg_end = (r1 % G == 0) if cls == 0 else (r1 == N or (r1 - s) % G == 0)
            if at_end and seg_end:
                for n in ("dk", "dv"):
                    ref_max[n] = max(ref_max[n], float(np.abs(ref[n][t]).max()))
    assert all(v > 0 for v in ref_max.values()), ref_max
    for r0, r1, at_end, ref in jobs:
        for t, h in enumerate(heads):
            where = "N131072 H132 head %d rows [%d, %d)" % (h, r0, r1)
            check_o(o[0, r0:r1, h], ref["o"][t], where)
            check_lse(lse[0, h, r0:r1], ref["lse"][t], where)
            check_grad("dq", to_np(dq[0, r0:r1, h]), ref["dq"][t], where, ref_max["dq"])
            cls = int(h >= H // 2)
            seg_end = (r1 % G == 0) if cls == 0 else (r1 == N or (r1 - s) % G == 0)
            if at_end and seg_end:  # every query that sees these keys lies in the window
                for n, g in (("dk", dk), ("dv", dv)):
                    check_grad(n, to_np(g[0, r0:r1, h]), ref[n][t], where, ref_max[n])


@PATHS
def test_long_context_packed_documents(stored):
    """The long-context workload packed with documents of 4096 tokens (the step
    bench.py --doc-len 4096 times), both backward forms, against the oracle under
    the same document mask: windows at document starts (o, lse, dq) and at
    document ends, where every query that sees the window's keys lies in the
    window (dk, dv complete as well)."""
    name, doc_len = "long_n32768_g8192", 4096
    w = synthetic.WORKLOADS[name]
    x = _inputs(w.B, w.N, w.H, w.D, w.seed, w.sharpen_k)
    ids = np.tile((np.arange(w.N) // doc_len).astype(np.int32), (w.B, 1))
    dev = {n: t.cuda() for n, t in x.items()}
    docs = s2.doc_bounds(torch.from_numpy(ids).cuda())
    o, lse = s2.forward(dev["q"], dev["k"], dev["v"], w.G, 0, docs=docs)
    dq, dk, dv = s2.backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, w.G, 0, docs=docs, stored_ds=stored)
    torch.cuda.synchronize()
    s2.check_status()
    H = w.H
    heads = (0, H // 2 - 1, H // 2, H - 1)
    windows = [(0, W, False), (3 * doc_len, 3 * doc_len + W, False), (2 * doc_len - W, 2 * doc_len, True),
               (5 * doc_len - W, 5 * doc_len, True), (w.N - W, w.N, True)]
    jobs, ref_max = [], {"dq": 0.0, "dk": 0.0, "dv": 0.0}
    for r0, r1, at_end in windows:
        ref = oracle.attention_window(x["q"], x["k"], x["v"], x["dout"], G=w.G, variant=0, rows=(r0, r1),
                                      heads=list(heads), doc=ids)
        jobs.append((r0, r1, at_end, ref))
        ref_max["dq"] = max(ref_max["dq"], float(np.abs(ref["dq"]).max()))
        if at_end:
            for n in ("dk", "dv"):
                ref_max[n] = max(ref_max[n], float(np.abs(ref[n]).max()))
    for r0, r1, at_end, ref in jobs:
        for t, h in enumerate(heads):
            where = "%s documents of %d head %d rows [%d, %d)" % (name, doc_len, h, r0, r1)
            check_o(o[0, r0:r1, h], ref["o"][t], where)
            check_lse(lse[0, h, r0:r1], ref["lse"][t], where)
            check_grad("dq", to_np(dq[0, r0:r1, h]), ref["dq"][t], where, ref_max["dq"])
            if at_end:
                for n, g in (("dk", dk), ("dv", dv)):
                    check_grad(n, to_np(g[0, r0:r1, h]), ref[n][t], where, ref_max[n])
