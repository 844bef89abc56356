"""Pins for the oracle's document mask (packed sequences).

"4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §1.1 ("因果mask与样本packing"): when
documents are packed into one sequence, attention also needs a document
mask, and the original and the shifted grouping use the same document-ID
constraint.  The same section gives the test: put document boundaries inside
a group, on an original group boundary and on a shifted boundary, change the
earlier document, and the later document's outputs must not move.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from shifted_sparse_attention_b200 import synthetic

STRICT, ROLLED, DENSE = oracle.STRICT, oracle.ROLLED, oracle.DENSE_CAUSAL


def _runs(lengths):
    """Per-position IDs of documents laid out back to back."""
    return np.concatenate([np.full(n, d, dtype=np.int32) for d, n in enumerate(lengths)])


def _sdpa_causal(q, k, v):
    o = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(1, 2), k.transpose(1, 2), v.transpose(1, 2), is_causal=True)
    return o.transpose(1, 2)


@pytest.mark.parametrize("variant", [STRICT, ROLLED, DENSE])
def test_leak_test_of_the_pages(variant):
    # N = 32, G = 8 (s = 4): boundaries at 5 (inside a group), 16 (original group
    # boundary) and 20 (shifted boundary).
    B, N, H, D, G = 1, 32, 4, 8, 8
    doc = _runs([5, 11, 4, 12])
    x = synthetic.draw(B, N, H, D, seed=41)
    ref = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant, doc=doc)
    for first, last in ((0, 5), (5, 16), (16, 20)):
        y = {n: t.clone() for n, t in x.items()}
        for n in ("q", "k", "v", "dout"):
            y[n][:, first:last] = (torch.randn_like(y[n][:, first:last].float()) * 3).to(torch.bfloat16)
        got = oracle.attention(y["q"], y["k"], y["v"], y["dout"], G=G, variant=variant, doc=doc)
        after = slice(last, N)
        # the later documents see nothing of the changed one: bit-identical outputs
        for name in ("o", "dq", "dk", "dv"):
            np.testing.assert_array_equal(got[name][:, after], ref[name][:, after])
        np.testing.assert_array_equal(got["lse"][:, :, after], ref["lse"][:, :, after])
    # without the mask the same change leaks into later documents (the test has teeth)
    if variant != ROLLED:
        plain = oracle.attention(x["q"], x["k"], x["v"], G=G, variant=variant)
        y = {n: t.clone() for n, t in x.items()}
        y["v"][:, 0:5] = (torch.randn_like(y["v"][:, 0:5].float()) * 3).to(torch.bfloat16)
        moved = oracle.attention(y["q"], y["k"], y["v"], G=G, variant=variant)
        assert not np.array_equal(moved["o"][:, 5:8], plain["o"][:, 5:8])


def test_dense_causal_with_documents_is_causal_attention_per_document():
    B, N, H, D = 2, 40, 2, 8
    lengths = [7, 13, 1, 19]
    doc = _runs(lengths)
    x = synthetic.draw(B, N, H, D, seed=43)
    res = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=N, variant=DENSE, doc=doc)
    q, k, v, g = (x[n].to(torch.float64).requires_grad_(True) for n in ("q", "k", "v", "dout"))
    outs, a = [], 0
    for n in lengths:
        outs.append(_sdpa_causal(q[:, a:a + n], k[:, a:a + n], v[:, a:a + n]))
        a += n
    o_ref = torch.cat(outs, dim=1)
    (o_ref * g).sum().backward()
    np.testing.assert_allclose(res["o"], o_ref.detach().numpy(), rtol=0, atol=1e-12)
    for name, t in (("dq", q), ("dk", k), ("dv", v)):
        np.testing.assert_allclose(res[name], t.grad.numpy(), rtol=0, atol=1e-12)


def test_one_document_is_no_mask():
    B, N, H, D, G = 1, 48, 4, 8, 16
    x = synthetic.draw(B, N, H, D, seed=44)
    for variant in (STRICT, ROLLED):
        a = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant)
        b = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant,
                             doc=np.full(N, 7, dtype=np.int32))
        for name in ("o", "lse", "dq", "dk", "dv"):
            np.testing.assert_array_equal(a[name], b[name])


@pytest.mark.parametrize("lengths", [[3, 9, 12], [16, 8], [1] * 8 + [16], [24], [5, 2, 9, 8]])
def test_pair_counts_with_documents(lengths):
    N, G = 24, 8
    doc = _runs(lengths)
    tri = lambda n: n * (n + 1) // 2
    # dense causal: every document is a causal triangle
    assert oracle.pair_count_docs(N, N, N, DENSE, 0, doc) == sum(tri(n) for n in lengths)
    # class 0: causal triangles of the intersections of documents and groups
    cuts = sorted(set(list(range(0, N + 1, G)) + list(np.cumsum([0] + lengths))))
    expect0 = sum(tri(b - a) for a, b in zip(cuts, cuts[1:]))
    assert oracle.pair_count_docs(N, G, N, STRICT, 0, doc) == expect0
    # class 1 strict: the same with the shifted cut points (short head and tail groups)
    s = G // 2
    cuts1 = sorted(set([0, N] + list(range(s, N, G)) + list(np.cumsum([0] + lengths))))
    expect1 = sum(tri(b - a) for a, b in zip(cuts1, cuts1[1:]))
    assert oracle.pair_count_docs(N, G, N, STRICT, 1, doc) == expect1
    # the mask only removes pairs
    for variant, cls in ((STRICT, 0), (STRICT, 1), (ROLLED, 1)):
        assert oracle.pair_count_docs(N, G, N, variant, cls, doc) <= oracle.pair_count(N, G, N, variant, cls)


def test_document_mask_applies_to_both_head_classes_and_the_window_entry():
    B, N, H, D, G = 1, 32, 4, 8, 8
    doc = _runs([6, 10, 16])
    x = synthetic.draw(B, N, H, D, seed=45)
    full = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=STRICT, doc=doc)
    win = oracle.attention_window(x["q"], x["k"], x["v"], x["dout"], G=G, variant=STRICT,
                                  rows=(0, N), heads=list(range(H)), doc=doc)
    np.testing.assert_allclose(win["o"], full["o"][0].transpose(1, 0, 2), rtol=0, atol=1e-14)
    # a shifted head (class 1) near position 6: without the mask, row 6 (first row of
    # document 1) would see 4 and 5 (shifted group [4, 12)); with it, only itself
    lse = full["lse"][0, H - 1, 6]
    qk = float((x["q"][0, 6, H - 1].double() @ x["k"][0, 6, H - 1].double()) / math.sqrt(D))
    assert abs(lse - qk) < 1e-12


@pytest.mark.parametrize("variant,cls", [(STRICT, 0), (STRICT, 1), (ROLLED, 1), (DENSE, 0)])
def test_adjacency_with_documents(variant, cls):
    """The document-masked matrix, pinned three ways: one document is no mask;
    one document per position leaves only the valid diagonal; documents laid
    out back to back give, for class 0 and the dense graph, causal triangles
    over the cuts of documents and groups, checked cell by cell."""
    N, G = 32, 8
    for nv in (N, 27):
        A = oracle.adjacency(N, G, nv, variant, cls)
        one = oracle.adjacency_docs(N, G, nv, variant, cls, np.zeros(N, dtype=np.int32))
        np.testing.assert_array_equal(one, A)
        single = oracle.adjacency_docs(N, G, nv, variant, cls, np.arange(N, dtype=np.int32))
        np.testing.assert_array_equal(single, np.diag(np.arange(N) < nv))
    lengths = [5, 3, 9, 8, 7]
    doc = _runs(lengths)
    got = oracle.adjacency_docs(N, G, N, variant, cls, doc)
    assert got.sum() == oracle.pair_count_docs(N, G, N, variant, cls, doc)
    for i in range(N):
        np.testing.assert_array_equal(oracle.adjacency_row_docs(N, G, N, variant, cls, doc, i), got[i])
    if variant == DENSE or cls == 0:
        bounds = np.cumsum([0] + lengths)
        cuts = sorted(set(bounds.tolist()) | (set() if variant == DENSE else set(range(0, N + 1, G))))
        expect = np.zeros((N, N), dtype=bool)
        for a, b in zip(cuts, cuts[1:]):
            for i in range(a, b):
                expect[i, a:i + 1] = True
        np.testing.assert_array_equal(got, expect)
