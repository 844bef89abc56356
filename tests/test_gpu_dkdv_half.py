"""The dK/dV pass over half query tiles (S2_OPT_DKDV_HALF) against the float64
oracle and the default dK/dV pass (needs a B200)."""
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
    # (B, N, H, D, G, variant, n_valid, stored)
    (1, 1024, 8, 64, 256, STRICT, None, True),
    (2, 2048, 4, 128, 512, STRICT, 1900, True),
    (2, 2048, 4, 128, 512, ROLLED, 1283, False),
    (1, 2048, 4, 128, 2048, DENSE, None, True),
    (1, 1536, 2, 128, 768, STRICT, 129, False),
    (1, 1024, 2, 128, 256, ROLLED, 1, True),
    (3, 1024, 6, 64, 512, STRICT, 777, True),
]


def _grads(dev, G, variant, nv, stored, half, docs=None):
    s2.set_dkdv_half(half)
    try:
        o, lse = s2.forward(dev["q"], dev["k"], dev["v"], G, variant, nv, docs=docs)
        g = s2.backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, G, variant, nv, docs=docs,
                        stored_ds=stored)
        torch.cuda.synchronize()
        s2.check_status()
    finally:
        s2.set_dkdv_half(False)
    return g


@pytest.mark.parametrize("B,N,H,D,G,variant,nv,stored", CASES)
def test_half_tile_dkdv_matches_oracle_and_default(B, N, H, D, G, variant, nv, stored):
    x = synthetic.draw(B, N, H, D, seed=5000 + N + G + variant)
    dev = {n: t.cuda() for n, t in x.items()}
    g1 = _grads(dev, G, variant, nv, stored, False)
    g2 = _grads(dev, G, variant, nv, stored, True)
    ref = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant, n_valid=nv)
    n = N if nv is None else nv
    where = str((B, N, H, D, G, variant, nv, stored))
    for name, a, b in zip(("dq", "dk", "dv"), g2, g1):
        check_grad(name, to_np(a)[:, :n], ref[name][:, :n], where)
        d = (a.float() - b.float()).abs().max().item() / max(b.float().abs().max().item(), 1e-30)
        assert d < 4e-3, (name, d)
        if nv is not None:
            assert (to_np(a)[:, nv:] == 0).all()


def test_half_tile_dkdv_under_document_masks():
    B, N, H, D, G = 2, 2048, 4, 128, 512
    ids = np.zeros((B, N), dtype=np.int32)
    for b, cuts in enumerate(([300, 700, 1024, 1500], [129, 256, 1800])):
        for c in cuts:
            ids[b, c:] += 1
    x = synthetic.draw(B, N, H, D, seed=61)
    dev = {n: t.cuda() for n, t in x.items()}
    docs = s2.doc_bounds(torch.from_numpy(ids).cuda())
    g = _grads(dev, G, STRICT, None, True, True, docs)
    ref = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=STRICT, doc=ids)
    for name, a in zip(("dq", "dk", "dv"), g):
        check_grad(name, to_np(a), ref[name], "docs")


def test_half_tile_dkdv_long_context_matches_default():
    w = synthetic.WORKLOADS["long_n32768_g8192"]
    x = synthetic.draw(1, w.N, 4, w.D, seed=2, sharpen_k=True)
    dev = {n: t.cuda() for n, t in x.items()}
    g1 = _grads(dev, w.G, STRICT, None, True, False)
    g2 = _grads(dev, w.G, STRICT, None, True, True)
    for a, b in zip(g2, g1):
        d = (a.float() - b.float()).abs().max().item() / b.float().abs().max().item()
        assert d < 4e-3, d
