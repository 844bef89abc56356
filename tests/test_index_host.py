"""CPU checks of the kernels' scheduler (s2_index.cuh) and of the C ABI host layer.

The scheduler header is compiled with g++ into a small host harness that walks
work units, key tiles and column limits exactly as the kernels do; the pairs
it visits must equal the oracle's explicit matrices A^(0), A^(1) (every pair
once, nothing else), and every query row must be owned by exactly one unit.
"""
from __future__ import annotations

import ctypes
import re
import subprocess
from pathlib import Path

import numpy as np
import pytest

import oracle

ROOT = Path(__file__).resolve().parent.parent
CSRC = ROOT / "shifted_sparse_attention_b200" / "csrc"
HARNESS = Path(__file__).resolve().parent / "native" / "index_harness.cpp"


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    out = tmp_path_factory.mktemp("harness") / "libindex_harness.so"
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-I", str(CSRC), str(HARNESS),
                           "-o", str(out)])
    L = ctypes.CDLL(str(out))
    L.s2h_visit.argtypes = [ctypes.c_int] * 5 + [ctypes.c_void_p, ctypes.c_void_p]
    L.s2h_visit.restype = ctypes.c_int
    L.s2h_visit_bwd.argtypes = [ctypes.c_int] * 5 + [ctypes.c_void_p, ctypes.c_void_p]
    L.s2h_visit_bwd.restype = ctypes.c_int
    L.s2h_plan.argtypes = [ctypes.c_int] * 6 + [ctypes.c_void_p]
    L.s2h_visit_docs.argtypes = [ctypes.c_int] * 5 + [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    L.s2h_visit_docs.restype = ctypes.c_int
    L.s2h_visit_sp.argtypes = [ctypes.c_int] * 8 + [ctypes.c_void_p]
    L.s2h_visit_sp.restype = ctypes.c_int
    L.s2h_ds_slots.argtypes = [ctypes.c_int] * 6 + [ctypes.c_void_p] * 3
    L.s2h_ds_slots.restype = ctypes.c_longlong
    return L


def _visit(L, N, G, nv, variant, cls, backward=False):
    vis = np.zeros((N, N), dtype=np.uint8)
    cover = np.zeros(N, dtype=np.int32)
    fn = L.s2h_visit_bwd if backward else L.s2h_visit
    fn(N, G, nv, variant, cls, vis.ctypes.data, cover.ctypes.data)
    return vis, cover


CASES = [(N, G) for N in (256, 512, 768, 1024, 1536, 2048) for G in (256, 512, 768, 1024) if N % G == 0]


@pytest.mark.parametrize("N,G", CASES)
@pytest.mark.parametrize("variant", [0, 1])
def test_scheduler_visits_exactly_the_oracle_pairs(harness, N, G, variant):
    for nv in sorted({N, N - 1, N - 127, N - 128, N - G // 2 - 3, 1, 129, (N * 3) // 5}):
        if nv < 1:
            continue
        for cls in (0, 1):
            A = oracle.adjacency(N, G, nv, variant, cls)
            for backward in (False, True):
                vis, cover = _visit(harness, N, G, nv, variant, cls, backward)
                where = str((N, G, nv, variant, cls, "bwd" if backward else "fwd"))
                assert (cover == 1).all(), where
                assert vis.max() <= 1, "a pair was computed twice " + where
                np.testing.assert_array_equal(vis.astype(bool), A, err_msg=where)


@pytest.mark.parametrize("N", [128, 256, 640, 1024])
def test_scheduler_dense_causal(harness, N):
    for nv in (N, N - 5, 1):
        for backward in (False, True):
            vis, cover = _visit(harness, N, N, nv, 2, 0, backward)
            assert (cover == 1).all()
            np.testing.assert_array_equal(vis.astype(bool), oracle.adjacency(N, N, nv, 2, 0))


def _bounds_of(ids):
    """Per-position [first, one past last] of each maximal run of equal IDs (reference for the kernels' input)."""
    N = len(ids)
    b = np.zeros((N, 2), dtype=np.int32)
    start = 0
    for x in range(1, N + 1):
        if x == N or ids[x] != ids[x - 1]:
            b[start:x] = (start, x)
            start = x
    return b


def _doc_layouts(N, G):
    """Document boundaries inside groups, on original and on shifted group boundaries, short
    documents spanning several tiles, and one document."""
    s = G // 2
    cuts = [
        [N],
        [5, N],
        [G, N],
        [s, G + s, N],
        [100, 300, 301, G + s + 7, N],
        list(range(97, N, 97)) + [N],
        [1, 2, 3, N - 3, N],
    ]
    out = []
    for c in cuts:
        c = sorted(set(x for x in c if 0 < x <= N))
        ids = np.zeros(N, dtype=np.int32)
        for d, (a, b) in enumerate(zip([0] + c, c)):
            ids[a:b] = d
        out.append(ids)
    return out


@pytest.mark.parametrize("N,G", [(512, 256), (1024, 512), (1536, 512), (2048, 1024)])
@pytest.mark.parametrize("variant", [0, 1, 2])
def test_scheduler_under_document_masks_visits_exactly_the_oracle_pairs(harness, N, G, variant):
    if variant == 2:
        G = N
    for ids in _doc_layouts(N, G):
        bounds = np.ascontiguousarray(_bounds_of(ids))
        same = ids[:, None] == ids[None, :]
        for nv in (N, N - 77):
            for cls in ((0,) if variant == 2 else (0, 1)):
                A = oracle.adjacency(N, G, nv, variant, cls) & same
                assert oracle.pair_count_docs(N, G, nv, variant, cls, ids) == A.sum()
                for which in (0, 1, 2):
                    vis = np.zeros((N, N), dtype=np.uint8)
                    harness.s2h_visit_docs(N, G, nv, variant, cls, bounds.ctypes.data, which, vis.ctypes.data)
                    where = str((N, G, nv, variant, cls, which, ids[::97][:6]))
                    assert vis.max() <= 1, "a pair was computed twice " + where
                    np.testing.assert_array_equal(vis.astype(bool), A, err_msg=where)


@pytest.mark.parametrize("seed", range(24))
def test_scheduler_under_random_document_layouts(harness, seed):
    # random shape, valid length and document cuts (any position, any count) for all three traversals
    r = np.random.default_rng(7000 + seed)
    variant = int(r.integers(0, 3))
    G = 256 * int(r.integers(1, 5))
    N = G * int(r.integers(1, 3 if variant == 2 else 4))
    if variant == 2:
        G = N
    nv = N if r.random() < 0.4 else int(r.integers(1, N + 1))
    ids = np.zeros(N, dtype=np.int32)
    for c in r.choice(np.arange(1, N), size=int(r.integers(0, 12)), replace=False):
        ids[c:] += 1
    bounds = np.ascontiguousarray(_bounds_of(ids))
    same = ids[:, None] == ids[None, :]
    for cls in ((0,) if variant == 2 else (0, 1)):
        A = oracle.adjacency(N, G, nv, variant, cls) & same
        for which in (0, 1, 2):
            vis = np.zeros((N, N), dtype=np.uint8)
            harness.s2h_visit_docs(N, G, nv, variant, cls, bounds.ctypes.data, which, vis.ctypes.data)
            where = str((seed, N, G, nv, variant, cls, which))
            assert vis.max() <= 1, "a pair was computed twice " + where
            np.testing.assert_array_equal(vis.astype(bool), A, err_msg=where)


def test_dq_traversal_without_documents(harness):
    for N, G, variant in ((1024, 512, 0), (1024, 512, 1), (768, 768, 2)):
        for nv in (N, N - 200):
            for cls in ((0,) if variant == 2 else (0, 1)):
                vis = np.zeros((N, N), dtype=np.uint8)
                harness.s2h_visit_docs(N, G, nv, variant, cls, None, 2, vis.ctypes.data)
                assert vis.max() <= 1
                np.testing.assert_array_equal(vis.astype(bool), oracle.adjacency(N, G, nv, variant, cls))


def test_grid_sizes_of_the_workloads(harness):
    out = np.zeros(5, dtype=np.int32)
    # long-context workload: 4 unshifted segments of 32 units, 5 strict shifted segments
    harness.s2h_plan(1, 32768, 32, 8192, 32768, 0, out.ctypes.data)
    assert out.tolist() == [32 * 5 * 32, 4, 5, 32, 32]
    harness.s2h_plan(1, 1024, 8, 256, 1024, 0, out.ctypes.data)
    assert out.tolist() == [8 * 5 * 1, 4, 5, 1, 1]


# ---------------------------------------------------------------- C ABI host layer (no GPU needed)


@pytest.fixture(scope="module")
def abi():
    from shifted_sparse_attention_b200 import build
    build.build()
    from shifted_sparse_attention_b200 import binding
    return binding


def test_library_exports_every_declared_symbol(abi):
    header = (ROOT / "include" / "s2attn.h").read_text()
    declared = set(re.findall(r"\b(s2attn_\w+)\s*\(", header))
    assert declared == set(abi.SIGNATURES), declared ^ set(abi.SIGNATURES)
    nm = subprocess.run(["nm", "-D", "--defined-only", str(abi.LIB_PATH)], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (s2attn_\w+)", nm))
    assert declared <= exported, declared - exported
    L = abi.lib()
    for name in declared:
        assert hasattr(L, name)
    assert L.s2attn_version() == 201
    assert L.s2attn_debug_bounds_checked() == 0


def test_debug_library_exports_the_same_symbols_with_checks_compiled_in(abi):
    """libs2attn_debug.so is the same ABI; only the kernels carry the bounds checks."""
    header = (ROOT / "include" / "s2attn.h").read_text()
    declared = set(re.findall(r"\b(s2attn_\w+)\s*\(", header))
    nm = subprocess.run(["nm", "-D", "--defined-only", str(abi.DEBUG_LIB_PATH)], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (s2attn_\w+)", nm))
    assert declared <= exported, declared - exported
    with abi.debug_library() as D:
        assert D.s2attn_version() == 201
        assert D.s2attn_debug_bounds_checked() == 1
        assert abi.lib() is D
    assert abi.lib().s2attn_debug_bounds_checked() == 0
    # host validation is shared: a bad shape fails before any launch in both builds
    fake = 1 << 20
    with abi.debug_library() as D:
        rc = D.s2attn_fwd_v(fake, fake, fake, fake, fake, 1, 1000, 8, 64, 256, 1000, 0, None)
    assert rc == abi.S2_ERR_SHAPE


def test_host_validation_rejects_bad_shapes_before_any_launch(abi):
    L = abi.lib()
    fake = 1 << 20  # never dereferenced: validation fails first
    cases = [
        (dict(H=3), abi.S2_ERR_SHAPE),           # odd head count
        (dict(G=255), abi.S2_ERR_SHAPE),         # odd group
        (dict(N=1000), abi.S2_ERR_SHAPE),        # N not a multiple of G
        (dict(nv=0), abi.S2_ERR_SHAPE),
        (dict(nv=1025), abi.S2_ERR_SHAPE),
        (dict(D=96), abi.S2_ERR_UNSUPPORTED),
        (dict(G=128), abi.S2_ERR_UNSUPPORTED),   # shift 64 is not a multiple of 128
        (dict(variant=7), abi.S2_ERR_INVALID_ARG),
    ]
    for over, code in cases:
        a = dict(B=1, N=1024, H=8, D=64, G=256, nv=1024, variant=0)
        a.update(over)
        rc = L.s2attn_fwd_v(fake, fake, fake, fake, fake, a["B"], a["N"], a["H"], a["D"], a["G"], a["nv"],
                            a["variant"], None)
        assert rc == code, (over, rc, abi.s2attn_last_error())
        assert abi.s2attn_last_error()
    rc = L.s2attn_fwd_v(None, fake, fake, fake, fake, 1, 1024, 8, 64, 256, 1024, 0, None)
    assert rc == abi.S2_ERR_INVALID_ARG
    rc = L.s2attn_fwd_v(fake + 8, fake, fake, fake, fake, 1, 1024, 8, 64, 256, 1024, 0, None)
    assert rc == abi.S2_ERR_INVALID_ARG  # misaligned
    ws = L.s2attn_bwd_workspace_size(1, 1024, 8, 64)
    assert ws == 2 * 1024 * 8 * 4  # two float32 row statistics; no dq accumulator
    rc = L.s2attn_bwd_v(*([fake] * 9), 1, 1024, 8, 64, 256, 1024, 0, fake, ws - 1, None)
    assert rc == abi.S2_ERR_INVALID_ARG  # workspace too small
    rc = L.s2attn_debug_adjacency(1024, 256, 1024, 0, 2, 0, fake, None)
    assert rc == abi.S2_ERR_INVALID_ARG


def test_tensor_api_refuses_cpu_tensors(abi):
    import torch
    q = torch.zeros(1, 1024, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        abi.forward(q, q, q, 256)


def test_rope_host_validation(abi):
    L = abi.lib()
    fake = 1 << 20
    rc = L.s2attn_rope(fake, fake, fake, fake, None, 1, 16, 2, 96, 10000.0, 1.0, None)
    assert rc == abi.S2_ERR_UNSUPPORTED  # D outside {64, 128}
    rc = L.s2attn_rope(fake, fake, fake, fake, None, 1, 16, 2, 128, 1.0, 1.0, None)
    assert rc == abi.S2_ERR_INVALID_ARG  # base must exceed 1
    rc = L.s2attn_rope(fake, fake, fake, fake, None, 1, 16, 2, 128, 10000.0, 0.0, None)
    assert rc == abi.S2_ERR_INVALID_ARG  # scale must be positive
    rc = L.s2attn_rope(fake, None, fake, fake, None, 1, 16, 2, 128, 10000.0, 1.0, None)
    assert rc == abi.S2_ERR_INVALID_ARG
    rc = L.s2attn_rope(fake, fake, fake + 4, fake, None, 1, 16, 2, 128, 10000.0, 1.0, None)
    assert rc == abi.S2_ERR_INVALID_ARG  # misaligned output
    rc = L.s2attn_rope(fake, fake, fake, fake, fake + 2, 1, 16, 2, 128, 10000.0, 1.0, None)
    assert rc == abi.S2_ERR_INVALID_ARG  # misaligned positions
    rc = L.s2attn_rope(fake, fake, fake, fake, None, 0, 16, 2, 128, 10000.0, 1.0, None)
    assert rc == abi.S2_ERR_SHAPE


# ---------------------------------------------------------------- sequence parallelism
# "4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §1.1: with G-aligned shards and a
# half-group halo exchange, the multi-rank graph must equal the single-GPU one
# (the pages' single- vs multi-card comparison of visible sets): the union over
# ranks of the pairs each rank's kernels compute is exactly A^(0) / A^(1) of
# the whole sequence, every pair once, in the forward and in both backward passes.

SP_CASES = [(G, L // G, W) for G in (256, 512) for L in (G, 2 * G) for W in (1, 2, 3, 4)]


@pytest.mark.parametrize("G,per,W", SP_CASES)
@pytest.mark.parametrize("variant", [0, 1])
def test_sequence_parallel_union_is_the_single_gpu_graph(harness, G, per, W, variant):
    L = G * per
    N = W * L
    for nv_last in ([L] if variant == 1 else [L, L - 100, 1]):
        nv = (W - 1) * L + nv_last
        for cls in (0, 1):
            ref = oracle.adjacency(N, G, nv, variant, cls)
            for which in (0, 1, 2):
                vis = np.zeros((N, N), dtype=np.uint8)
                for r in range(W):
                    rc = harness.s2h_visit_sp(L, G, nv_last if r == W - 1 else L, variant, r, W, cls, which,
                                              vis.ctypes.data)
                    assert rc == 0, ("halo row without a global position", r)
                assert vis.max() <= 1, ("pair computed twice", which)
                np.testing.assert_array_equal(vis.astype(bool), ref, err_msg=str((W, L, cls, which, nv)))


def test_sequence_parallel_host_validation(abi):
    L = abi.lib()
    fake = 1 << 20
    base = dict(B=1, L=1024, H=8, D=128, G=256, nv=1024, variant=0, rank=0, world=2)
    cases = [
        (dict(variant=2), abi.S2_ERR_UNSUPPORTED),       # dense causal does not shard by halos
        (dict(variant=5), abi.S2_ERR_INVALID_ARG),
        (dict(rank=2), abi.S2_ERR_INVALID_ARG),
        (dict(world=0), abi.S2_ERR_INVALID_ARG),
        (dict(L=1000), abi.S2_ERR_SHAPE),                # shard not a multiple of G
        (dict(nv=1000), abi.S2_ERR_SHAPE),               # padding on a rank that is not the last
        (dict(nv=1000, rank=1, variant=1), abi.S2_ERR_UNSUPPORTED),  # ROLLED needs no padding
    ]
    for over, code in cases:
        a = dict(base)
        a.update(over)
        rc = L.s2attn_sp_fwd(fake, fake, fake, fake, fake, a["B"], a["L"], a["H"], a["D"], a["G"], a["nv"],
                             a["variant"], a["rank"], a["world"], None)
        assert rc == code, (over, rc, abi.s2attn_last_error())
        rc = L.s2attn_sp_bwd(*([fake] * 9), a["B"], a["L"], a["H"], a["D"], a["G"], a["nv"], a["variant"], a["rank"],
                             a["world"], fake, 1 << 30, None)
        assert rc == code, (over, rc, abi.s2attn_last_error())
    assert L.s2attn_sp_halo_bytes(2, 32, 128, 8192) == 2 * 2 * 16 * 4096 * 128 * 2  # V_KV, K and V
    rc = L.s2attn_sp_halo_pack(fake, fake, fake, 1, 1024, 8, 128, 256, 7, None)
    assert rc == abi.S2_ERR_INVALID_ARG
    rc = L.s2attn_sp_halo_unpack(fake, fake, fake + 8, 1, 1024, 8, 128, 256, 0, None)
    assert rc == abi.S2_ERR_INVALID_ARG


# ---------------------------------------------------------------- stored dS
# The dK/dV pass writes one dS tile per computed tile pair and the dQ pass
# reads exactly those tiles: every written slot once, the read set equal to the
# written set (also under document masks and padding), all inside the workspace.

def _tri(n):
    return n * (n + 1) // 2


def _ds_head_tiles(N, G, variant):
    if variant == 2:
        return _tri(N // 128)
    s = G // 2
    c0 = (N // G) * _tri(G // 128)
    c1 = c0 if variant == 1 else 2 * _tri(s // 128) + (N // G - 1) * _tri(G // 128)
    return max(c0, c1)


@pytest.mark.parametrize("N,G", [(1024, 256), (1536, 512), (2048, 1024), (1024, 1024)])
@pytest.mark.parametrize("variant", [0, 1, 2])
@pytest.mark.parametrize("docs", [False, True])
def test_stored_ds_slots_written_once_and_read_back(harness, N, G, variant, docs):
    B, H = 2, 4
    for nv in (N, N - 77):
        d = None
        if docs:
            ids = np.zeros((B, N), dtype=np.int32)
            ids[0, 300:] = 1
            ids[0, 700:] = 2
            ids[1, 129:] = 1
            d = np.zeros((B, N, 2), dtype=np.int32)
            for b in range(B):
                st = 0
                for x in range(1, N + 1):
                    if x == N or ids[b, x] != ids[b, x - 1]:
                        d[b, st:x] = (st, x)
                        st = x
        total = B * H * _ds_head_tiles(N, G, variant)
        w = np.zeros(total, dtype=np.int32)
        r = np.zeros(total, dtype=np.int32)
        got = harness.s2h_ds_slots(B, N, H, G, nv, variant, d.ctypes.data if d is not None else None,
                                   w.ctypes.data, r.ctypes.data)
        assert got == total
        assert w.max() == 1 and r.max() == 1
        np.testing.assert_array_equal(w, r)


def test_stored_ds_workspace_size(abi):
    L = abi.lib()
    for (B, N, H, G, variant) in [(1, 32768, 32, 8192, 0), (2, 12288, 32, 12288, 2), (1, 8192, 32, 2048, 1),
                                  (1, 106496, 32, 8192, 0)]:
        got = L.s2attn_bwd_ds_workspace_size(B, N, H, 128, G, variant)
        assert got == 2 * B * H * N * 4 + B * H * _ds_head_tiles(N, G, variant) * 128 * 128 * 2
    assert L.s2attn_bwd_ds_workspace_size(1, 1000, 8, 128, 256, 0) == 0  # invalid shape
    fake = 1 << 20
    rc = L.s2attn_bwd_stages_v(*([fake] * 9), 1, 1024, 8, 64, 256, 1024, 0, fake, 1 << 30, 8, None)
    assert rc == abi.S2_ERR_INVALID_ARG  # the flag alone runs nothing
    ws = L.s2attn_bwd_ds_workspace_size(1, 1024, 8, 64, 256, 0)
    rc = L.s2attn_bwd_stages_v(*([fake] * 9), 1, 1024, 8, 64, 256, 1024, 0, fake, ws - 1, 15, None)
    assert rc == abi.S2_ERR_INVALID_ARG  # workspace too small for the stored dS


def test_bench_tile_pair_count_matches_the_kernels_traversal(harness):
    # bench.py prices the stored-dS dQ pass on a closed count of tile pairs; it must
    # equal the number of dS tiles the kernels' traversal writes
    import bench
    from types import SimpleNamespace

    for (N, G, nv, variant) in [(1024, 256, 1024, 0), (1536, 512, 1400, 0), (2048, 512, 2048, 1),
                                (2048, 1024, 1700, 1), (1024, 1024, 900, 2)]:
        B, H = 1, 2
        d = None
        total = B * H * _ds_head_tiles(N, G, variant)
        w = np.zeros(total, dtype=np.int32)
        r = np.zeros(total, dtype=np.int32)
        harness.s2h_ds_slots(B, N, H, G, nv, variant, d, w.ctypes.data, r.ctypes.data)
        wl = SimpleNamespace(N=N, G=G, valid=nv)
        counted = sum(bench.stored_tile_pairs(wl, variant, c) for c in ((0,) if variant == 2 else (0, 1)))
        if variant == 2:
            counted *= 2  # both heads of the dense graph are class 0
        assert int(w.sum()) == counted, (N, G, nv, variant, int(w.sum()), counted)


def test_bench_pair_count_matches_the_oracle():
    # bench.py prices exact-pair throughput (and the executed-over-useful ratio) on a
    # closed count of visible pairs per head class, padding included
    import bench
    from types import SimpleNamespace

    import oracle

    for (N, G, nv, variant) in [(1024, 256, 1024, 0), (1024, 256, 1000, 0), (2048, 512, 1283, 1),
                                (2048, 512, 300, 1), (1024, 1024, 900, 2), (4096, 1024, 4096, 1)]:
        c0, c1 = bench.pair_counts(SimpleNamespace(N=N, G=G, valid=nv), variant)
        assert c0 == oracle.pair_count(N, G, nv, variant, 0), (N, G, nv, variant)
        assert c1 == oracle.pair_count(N, G, nv, variant, 0 if variant == 2 else 1), (N, G, nv, variant)
