"""The bounds-checked build, libs2attn_debug.so (needs a B200).

Built from the same sources with -DS2_DEBUG_BOUNDS: before each access the
attention kernels check the tile origins they compute against [0, N) and the
plan's row ranges, their TMA row coordinates and stored indices against the
tensors, the stored-dS slots against the workspace and the TMEM columns
against the 512 allocated.  A violation is recorded (first one wins), the
access is skipped and the kernel gives up without a trap.

Checked here: the small parity cases of the other GPU tests (forward, both
backward forms, padding, one-group sequences, document masks, the emulated
sequence-parallel ranks, the plain entry points without n_valid) and 32
seeded random shapes run through
the debug build with no violation recorded, give results bit for bit equal to
the normal build's, and match the float64 oracle.  The recording path itself
is exercised by the probe entry point, which runs the same check on a chosen
value and touches no memory on its result.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from shifted_sparse_attention_b200 import binding as s2
from shifted_sparse_attention_b200 import synthetic
from tests import test_gpu_sp as sp_cases
from tests.tolerance import check_grad, check_lse, check_o, to_np

pytestmark = pytest.mark.gpu

STRICT, ROLLED, DENSE = 0, 1, 2


def _no_violation():
    assert s2.bounds_report() == (0, 0, 0, 0)
    s2.check_status()


def _run(dev, G, variant, nv, docs=None):
    o, lse = s2.forward(dev["q"], dev["k"], dev["v"], G, variant, nv, docs=docs)
    rec = s2.backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, G, variant, nv, docs=docs)
    sto = s2.backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, G, variant, nv, docs=docs, stored_ds=True)
    torch.cuda.synchronize()
    return (o, lse) + tuple(rec) + tuple(sto)


def _debug_and_release(x, G, variant, nv, docs=None):
    dev = {n: t.cuda() for n, t in x.items()}
    with s2.debug_library() as D:
        assert D.s2attn_debug_bounds_checked() == 1
        _no_violation()
        dbg = _run(dev, G, variant, nv, docs)
        _no_violation()
    rel = _run(dev, G, variant, nv, docs)
    s2.check_status()
    names = ("o", "lse", "dq", "dk", "dv", "dq_ds", "dk_ds", "dv_ds")
    for name, a, b in zip(names, dbg, rel):
        assert torch.equal(a, b), name
    return dict(zip(names, dbg))


CASES = [
    # (B, N, H, D, G, variant, n_valid)
    (1, 1024, 8, 64, 256, STRICT, None),
    (1, 1024, 8, 64, 256, ROLLED, None),
    (2, 2048, 4, 128, 512, STRICT, 1900),
    (2, 2048, 4, 128, 512, ROLLED, 1283),
    (1, 2048, 4, 128, 2048, DENSE, None),
    (1, 1536, 4, 128, 768, DENSE, 1409),
    (1, 1536, 2, 128, 768, STRICT, 129),
    (1, 1024, 2, 128, 256, ROLLED, 1),       # a single valid row
    (1, 256, 2, 64, 256, STRICT, None),      # one group per sequence
    (1, 256, 2, 128, 256, ROLLED, 200),      # one group, padded, wrap onto itself
    (3, 1024, 6, 64, 512, STRICT, 777),
    (1, 4096, 2, 128, 4096, STRICT, 4000),   # G = N
    (1, 128, 2, 128, 128, DENSE, None),      # the smallest dense sequence
]


@pytest.mark.parametrize("B,N,H,D,G,variant,nv", CASES)
def test_debug_build_records_no_violation_and_matches(B, N, H, D, G, variant, nv):
    x = synthetic.draw(B, N, H, D, seed=5000 + N + G + variant)
    r = _debug_and_release(x, G, variant, nv)
    ref = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant, n_valid=nv)
    n = N if nv is None else nv
    where = str((B, N, H, D, G, variant, nv))
    check_o(r["o"][:, :n], ref["o"][:, :n], where)
    check_lse(r["lse"].cpu().numpy(), ref["lse"])
    for name in ("dq", "dk", "dv"):
        check_grad(name, to_np(r[name])[:, :n], ref[name][:, :n], where)
        check_grad(name, to_np(r[name + "_ds"])[:, :n], ref[name][:, :n], where + " stored dS")


@pytest.mark.parametrize("variant", [STRICT, ROLLED])
def test_debug_build_under_document_masks(variant):
    B, N, H, D, G = 2, 2048, 4, 128, 512
    ids = np.zeros((B, N), dtype=np.int32)
    for b, cuts in enumerate(([300, 700, 1024, 1500], [129, 256, 1800])):
        for c in cuts:
            ids[b, c:] += 1
    x = synthetic.draw(B, N, H, D, seed=51 + variant)
    docs = s2.doc_bounds(torch.from_numpy(ids).cuda())
    r = _debug_and_release(x, G, variant, None, docs)
    ref = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant, doc=ids)
    check_o(r["o"], ref["o"], "docs variant %d" % variant)
    for name in ("dq", "dk", "dv"):
        check_grad(name, to_np(r[name]), ref[name], "docs variant %d" % variant)


@pytest.mark.parametrize("stored", [False, True], ids=["recompute", "stored_ds"])
@pytest.mark.parametrize("B,H,D,G,W,L,variant,pad", [c for c in sp_cases.CASES if c[4] > 1])
def test_debug_build_sequence_parallel_ranks(B, H, D, G, W, L, variant, pad, stored):
    N = W * L
    x = synthetic.draw(B, N, H, D, seed=W * 100 + L + variant)
    with s2.debug_library():
        _no_violation()
        dbg = sp_cases._emulate(x, G, variant, W, L - pad, stored)
        _no_violation()
    rel = sp_cases._emulate(x, G, variant, W, L - pad, stored)
    for name, a, b in zip(("o", "lse", "dq", "dk", "dv"), dbg, rel):
        assert torch.equal(a, b), name


def test_debug_build_plain_entry_points():
    B, N, H, D, G = 1, 2048, 4, 128, 512
    x = synthetic.draw(B, N, H, D, seed=61)
    dev = {n: t.cuda() for n, t in x.items()}

    def plain():
        o = torch.empty_like(dev["q"])
        lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
        s2._check(s2.s2attn_fwd(dev["q"], dev["k"], dev["v"], o, lse, B, N, H, D, G, STRICT))
        ws = torch.empty(s2.s2attn_bwd_workspace_size(B, N, H, D), dtype=torch.uint8, device="cuda")
        g = tuple(torch.empty_like(o) for _ in range(3))
        s2._check(s2.s2attn_bwd(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, *g, B, N, H, D, G, STRICT,
                                ws, ws.numel()))
        torch.cuda.synchronize()
        return (o, lse) + g

    with s2.debug_library():
        dbg = plain()
        _no_violation()
    rel = plain()
    for a, b in zip(dbg, rel):
        assert torch.equal(a, b)


def test_probe_records_the_first_violation_without_a_fault():
    # the normal build compiles the check out: nothing is recorded
    assert s2.s2attn_debug_bounds_probe(5, 0, 4) == s2.S2_OK
    assert s2.bounds_report() == (0, 0, 0, 0)
    s2.check_status()
    with s2.debug_library():
        _no_violation()
        assert s2.s2attn_debug_bounds_probe(3, 0, 4) == s2.S2_OK  # inside: nothing recorded
        _no_violation()
        assert s2.s2attn_debug_bounds_probe(5, 0, 4) == s2.S2_OK
        assert s2.s2attn_debug_bounds_probe(-1, 0, 4) == s2.S2_OK  # a later one keeps the first record
        assert s2.bounds_report() == (14, 5, 0, 4)
        assert s2.bounds_report() == (14, 5, 0, 4)  # reading does not clear
        with pytest.raises(s2.S2AttnError) as e:
            s2.check_status()
        assert e.value.code == s2.S2_ERR_BOUNDS
        assert "site 14" in str(e.value) and "value 5 outside [0, 4)" in str(e.value)
        _no_violation()  # the check cleared it
        assert s2.s2attn_debug_bounds_probe(1, 2, 1) == s2.S2_ERR_INVALID_ARG
        # the context keeps working after a recorded violation
        x = synthetic.draw(1, 1024, 4, 128, seed=3)
        o, lse = s2.forward(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), 256)
        torch.cuda.synchronize()
        _no_violation()
        assert torch.isfinite(o).all()


@pytest.mark.parametrize("seed", range(100, 132))
def test_debug_build_on_random_shapes(seed):
    """Seeded random shapes, padding and document cuts (the fuzz test's generator,
    other seeds) through the debug build: no violation, bitwise the normal
    build's results, and the oracle's within the parity tolerances."""
    from tests.test_gpu_fuzz import _case

    B, N, H, D, G, variant, nv, ids = _case(seed)
    where = str((seed, B, N, H, D, G, variant, nv, ids is not None))
    x = synthetic.draw(B, N, H, D, seed=9000 + seed)
    docs = s2.doc_bounds(torch.from_numpy(ids).cuda()) if ids is not None else None
    r = _debug_and_release(x, G, variant, nv, docs)
    ref = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant, n_valid=nv, doc=ids)
    n = N if nv is None else nv
    check_o(r["o"][:, :n], ref["o"][:, :n], where)
    check_lse(r["lse"].cpu().numpy(), ref["lse"], where)
    for name in ("dq", "dk", "dv"):
        check_grad(name, to_np(r[name])[:, :n], ref[name][:, :n], where)
        check_grad(name, to_np(r[name + "_ds"])[:, :n], ref[name][:, :n], where + " stored dS")
