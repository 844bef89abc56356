"""Seeded random shapes through the whole path against the float64 oracle (needs a B200).

Each case draws B, H, D, G, N, n_valid, the variant and, for some cases,
document cuts from its own seed, within the library's constraints: H even,
G/2 a multiple of 128, N a multiple of G, D in {64, 128}.  The forward and
both forms of the backward (recomputing dQ, and dQ from the stored dS) are
checked against the oracle with the tolerances of the other parity tests.
The two forms must give bitwise the same dK and dV, and padded rows must be
exactly zero.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from shifted_sparse_attention_b200 import binding as s2
from shifted_sparse_attention_b200 import synthetic
from tests.tolerance import check_grad, check_lse, check_o, to_np

pytestmark = pytest.mark.gpu

DENSE = 2


def _case(seed: int):
    r = np.random.default_rng(seed)
    D = int(r.choice([64, 128]))
    G = 256 * int(r.integers(1, 5))  # 256 .. 1024: G/2 a multiple of 128
    variant = int(r.integers(0, 3))
    M = int(r.integers(1, 3 if variant == DENSE else 5))
    N = G * M
    H = int(r.choice([2, 4, 6]))
    B = int(r.integers(1, 3))
    nv = None if r.random() < 0.4 else int(r.integers(1, N + 1))
    ids = None
    if r.random() < 0.4:  # documents of random lengths, cut points anywhere
        cuts = np.sort(r.choice(np.arange(1, N), size=int(r.integers(1, 6)), replace=False))
        ids = np.zeros((B, N), dtype=np.int32)
        for c in cuts:
            ids[:, c:] += 1
    return B, N, H, D, G, variant, nv, ids


@pytest.mark.parametrize("seed", range(48))
def test_random_shapes_match_oracle(seed):
    B, N, H, D, G, variant, nv, ids = _case(seed)
    where = str((seed, B, N, H, D, G, variant, nv, ids is not None))
    x = synthetic.draw(B, N, H, D, seed=9000 + seed)
    dev = {n: t.cuda() for n, t in x.items()}
    docs = s2.doc_bounds(torch.from_numpy(ids).cuda()) if ids is not None else None
    o, lse = s2.forward(dev["q"], dev["k"], dev["v"], G, variant, nv, docs=docs)
    rec = s2.backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, G, variant, nv, docs=docs)
    sto = s2.backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, G, variant, nv, docs=docs,
                      stored_ds=True)
    torch.cuda.synchronize()
    s2.check_status()
    assert torch.equal(rec[1], sto[1]) and torch.equal(rec[2], sto[2]), where  # dk, dv

    ref = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant, n_valid=nv, doc=ids)
    check_o(o.cpu(), ref["o"], where)
    check_lse(lse.cpu(), ref["lse"], where)
    n = N if nv is None else nv
    for form, grads in (("recompute", rec), ("stored", sto)):
        for name, g in zip(("dq", "dk", "dv"), grads):
            g = to_np(g.cpu())
            check_grad(name, g[:, :n], ref[name][:, :n], where + " " + form)
            if nv is not None:
                assert (g[:, nv:] == 0).all(), (name, form, where)
    if nv is not None:
        assert (to_np(o.cpu())[:, nv:] == 0).all(), where
