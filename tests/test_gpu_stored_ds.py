"""The stored-dS backward (S2_BWD_STORE_DS) against the float64 oracle and the
recomputing backward (needs a B200).

With the flag the dK/dV pass also writes every dS tile and the dQ pass
computes dq = dS·K/√D from them.  dk and dv come from the same kernel
arithmetic as without the flag (bitwise equal); dq differs from the
recomputing pass only by the rounding of its own S and dP products.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from shifted_sparse_attention_b200 import binding as s2
from shifted_sparse_attention_b200 import synthetic
from tests.tolerance import check_grad, to_np

pytestmark = pytest.mark.gpu

STRICT, ROLLED, DENSE = 0, 1, 2

CASES = [
    # (B, N, H, D, G, variant, n_valid)
    (1, 1024, 8, 64, 256, STRICT, None),
    (1, 1024, 8, 64, 256, ROLLED, None),
    (2, 2048, 4, 128, 512, STRICT, 1900),
    (2, 2048, 4, 128, 512, ROLLED, 1283),
    (1, 2048, 4, 128, 2048, DENSE, None),
    (1, 1536, 4, 128, 768, DENSE, 1409),
    (1, 1536, 2, 128, 768, STRICT, 129),
    (1, 4096, 4, 128, 1024, STRICT, None),
    (1, 1024, 2, 128, 256, ROLLED, 1),       # a single valid row
    (1, 256, 2, 64, 256, STRICT, None),      # one group per sequence
    (3, 1024, 6, 64, 512, STRICT, 777),
]


def _both(x, G, variant, nv, docs=None):
    dev = {n: t.cuda() for n, t in x.items()}
    o, lse = s2.forward(dev["q"], dev["k"], dev["v"], G, variant, nv, docs=docs)
    rec = s2.backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, G, variant, nv, docs=docs)
    sto = s2.backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, G, variant, nv, docs=docs, stored_ds=True)
    torch.cuda.synchronize()
    s2.check_status()
    return rec, sto


@pytest.mark.parametrize("B,N,H,D,G,variant,nv", CASES)
def test_stored_ds_matches_oracle_and_recompute(B, N, H, D, G, variant, nv):
    x = synthetic.draw(B, N, H, D, seed=3000 + N + G + variant)
    rec, sto = _both(x, G, variant, nv)
    assert torch.equal(rec[1], sto[1]) and torch.equal(rec[2], sto[2])  # dk, dv
    ref = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant, n_valid=nv)
    n = N if nv is None else nv
    where = str((B, N, H, D, G, variant, nv))
    for name, g in zip(("dq", "dk", "dv"), sto):
        check_grad(name, to_np(g)[:, :n], ref[name][:, :n], where)
        if nv is not None:
            assert (to_np(g)[:, nv:] == 0).all(), (name, where)
    d = (sto[0].float() - rec[0].float()).abs().max().item() / rec[0].float().abs().max().item()
    assert d < 4e-3, d


@pytest.mark.parametrize("variant", [STRICT, ROLLED])
def test_stored_ds_under_document_masks(variant):
    B, N, H, D, G = 2, 2048, 4, 128, 512
    ids = np.zeros((B, N), dtype=np.int32)
    for b, cuts in enumerate(([300, 700, 1024, 1500], [129, 256, 1800])):
        for c in cuts:
            ids[b, c:] += 1
    x = synthetic.draw(B, N, H, D, seed=41 + variant)
    docs = s2.doc_bounds(torch.from_numpy(ids).cuda())
    rec, sto = _both(x, G, variant, None, docs)
    assert torch.equal(rec[1], sto[1]) and torch.equal(rec[2], sto[2])
    ref = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant, doc=ids)
    for name, g in zip(("dq", "dk", "dv"), sto):
        check_grad(name, to_np(g), ref[name], "docs variant %d" % variant)


def test_stored_ds_is_bitwise_reproducible():
    x = synthetic.draw(1, 8192, 8, 128, seed=77, sharpen_k=True)
    dev = {n: t.cuda() for n, t in x.items()}
    o, lse = s2.forward(dev["q"], dev["k"], dev["v"], 2048, STRICT)
    a = s2.backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, 2048, STRICT, stored_ds=True)
    b = s2.backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, 2048, STRICT, stored_ds=True)
    torch.cuda.synchronize()
    s2.check_status()
    for u, v in zip(a, b):
        assert torch.equal(u, v)
