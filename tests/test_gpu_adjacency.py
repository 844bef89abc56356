"""Bit-exact adjacency dump of the kernels' scheduler against the oracle (needs a B200)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from shifted_sparse_attention_b200 import binding as s2

pytestmark = pytest.mark.gpu


def _bits_to_bool(bits: torch.Tensor, N: int) -> np.ndarray:
    w = bits.cpu().numpy().view(np.uint32)
    out = np.unpackbits(w.view(np.uint8), axis=1, bitorder="little")
    return out[:, :N].astype(bool)


@pytest.mark.parametrize("N,G", [(1024, 256), (2048, 512), (8192, 2048)])
@pytest.mark.parametrize("variant", [0, 1, 2])
def test_bitset_equals_oracle(N, G, variant):
    for nv in (N, N - 1, N - 200, N // 2 + 77):
        for cls in (0, 1):
            got = _bits_to_bool(s2.debug_adjacency(N, G, variant, cls, nv, fmt=0), N)
            A = oracle.adjacency(N, G, nv, variant, 0 if variant == 2 else cls)
            np.testing.assert_array_equal(got, A, err_msg=str((N, G, variant, nv, cls)))


def _intervals_from_row(row: np.ndarray):
    idx = np.nonzero(row)[0]
    if len(idx) == 0:
        return [-1, -1, -1, -1]
    cuts = np.nonzero(np.diff(idx) > 1)[0]
    parts = np.split(idx, cuts + 1)
    assert len(parts) <= 2
    iv = []
    # kernel order: in the rolled wrap group the tail part comes first
    for p in sorted(parts, key=lambda a: -a[0] if len(parts) == 2 else a[0]):
        iv += [int(p[0]), int(p[-1])]
    return iv + [-1, -1] * (2 - len(parts))


@pytest.mark.parametrize("N,G,nv,variant", [
    (32768, 8192, 32768, 0),
    (32768, 8192, 30001, 1),
    (106496, 8192, 100000, 0),
    (12288, 12288, 12288, 2),
])
def test_intervals_on_sampled_rows(N, G, nv, variant):
    rng = np.random.default_rng(N + variant)
    s = G // 2
    for cls in (0, 1):
        got = s2.debug_adjacency(N, G, variant, cls, nv, fmt=1).cpu().numpy()
        rows = set(rng.integers(0, N, 48).tolist())
        rows |= {0, 1, s - 1, s, s + 1, G - 1, G, N - s - 1, N - s, N - 1, nv - 1, min(nv, N - 1)}
        for i in sorted(r for r in rows if 0 <= r < N):
            ref = _intervals_from_row(oracle.adjacency_row(N, G, nv, variant, 0 if variant == 2 else cls, i))
            assert got[i].tolist() == ref, (N, G, nv, variant, cls, i, got[i].tolist(), ref)


def _runs(N, cuts):
    ids = np.zeros(N, dtype=np.int32)
    for c in cuts:
        ids[c:] += 1
    return ids


DOC_CASES = [
    # N, G, cuts (document starts), n_valid
    (1024, 256, [300, 700, 1000], 1024),
    (1024, 256, [128, 256, 384, 640], 1000),        # on tile, group and shifted-group boundaries
    (2048, 512, [1, 2, 3, 1500, 1501], 1900),        # one-position documents
    (2048, 512, [129, 1800], 1283),
    (2048, 2048, [500, 1024, 1900], 2048),
    (1536, 768, list(range(64, 1536, 64)), 1409),    # many short documents
]


@pytest.mark.parametrize("N,G,cuts,nv", DOC_CASES)
@pytest.mark.parametrize("variant", [0, 1, 2])
def test_bitset_under_documents_equals_oracle(N, G, cuts, nv, variant):
    if variant == 2:
        G = N
    ids = _runs(N, cuts)
    docs = s2.doc_bounds(torch.from_numpy(ids).reshape(1, N).cuda())
    for cls in (0, 1):
        got = _bits_to_bool(s2.debug_adjacency(N, G, variant, cls, nv, fmt=0, docs=docs), N)
        A = oracle.adjacency_docs(N, G, nv, variant, 0 if variant == 2 else cls, ids)
        np.testing.assert_array_equal(got, A, err_msg=str((N, G, cuts, nv, variant, cls)))


@pytest.mark.parametrize("variant", [0, 1])
def test_intervals_under_documents_on_sampled_rows(variant):
    N, G, nv = 32768, 8192, 30001
    rng = np.random.default_rng(7 + variant)
    cuts = sorted(set(rng.integers(1, N, 40).tolist()) | {4096, 8192, 12288})
    ids = _runs(N, cuts)
    docs = s2.doc_bounds(torch.from_numpy(ids).reshape(1, N).cuda())
    s = G // 2
    for cls in (0, 1):
        got = s2.debug_adjacency(N, G, variant, cls, nv, fmt=1, docs=docs).cpu().numpy()
        rows = set(rng.integers(0, N, 48).tolist()) | {0, s - 1, s, G, N - s, N - 1, nv - 1}
        rows |= {c for c in cuts} | {c - 1 for c in cuts}
        for i in sorted(r for r in rows if 0 <= r < N):
            ref = _intervals_from_row(oracle.adjacency_row_docs(N, G, nv, variant, cls, ids, i))
            assert got[i].tolist() == ref, (variant, cls, i, got[i].tolist(), ref)
