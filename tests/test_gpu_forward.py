"""Forward parity of libs2attn.so against the float64 oracle (needs a B200)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from shifted_sparse_attention_b200 import binding as s2
from shifted_sparse_attention_b200 import synthetic
from tests.tolerance import check_lse, check_o, to_np

pytestmark = pytest.mark.gpu

STRICT, ROLLED, DENSE = 0, 1, 2


def _run(x, G, variant, nv=None):
    dev = {n: t.cuda() for n, t in x.items()}
    o, lse = s2.forward(dev["q"], dev["k"], dev["v"], G, variant, nv)
    s2.check_status()
    return o.cpu(), lse.cpu()


CASES = [
    # (B, N, H, D, G, variant, n_valid)
    (1, 1024, 8, 64, 256, STRICT, None),      # small workload, whole
    (1, 1024, 8, 64, 256, ROLLED, None),
    (1, 1024, 8, 64, 512, STRICT, 1000),
    (2, 2048, 4, 128, 512, STRICT, None),
    (2, 2048, 4, 128, 512, ROLLED, None),
    (2, 2048, 4, 128, 512, STRICT, 1900),      # ragged tail inside a tile
    (2, 2048, 4, 128, 512, ROLLED, 1283),      # ragged tail inside the wrap group
    (1, 2048, 4, 128, 2048, DENSE, None),
    (1, 1536, 4, 128, 768, DENSE, 1409),
    (1, 1536, 2, 128, 768, STRICT, 129),
    (1, 4096, 2, 128, 1024, ROLLED, 3000),
    # degenerate shapes: a single valid row, one group per sequence (G = N), the
    # smallest dense sequence, six heads, three batch rows
    (1, 1024, 2, 128, 256, STRICT, 1),
    (1, 1024, 2, 128, 256, ROLLED, 1),
    (1, 256, 2, 64, 256, STRICT, None),
    (1, 256, 2, 128, 256, ROLLED, 200),
    (1, 128, 2, 128, 128, DENSE, None),
    (3, 1024, 6, 64, 512, STRICT, 777),
]


@pytest.mark.parametrize("B,N,H,D,G,variant,nv", CASES)
def test_forward_matches_oracle(B, N, H, D, G, variant, nv):
    x = synthetic.draw(B, N, H, D, seed=1000 + N + G + variant)
    o, lse = _run(x, G, variant, nv)
    ref = oracle.attention(x["q"], x["k"], x["v"], G=G, variant=variant, n_valid=nv)
    where = str((B, N, H, D, G, variant, nv))
    check_o(o, ref["o"], where)
    check_lse(lse, ref["lse"], where)
    if nv is not None:
        assert (to_np(o)[:, nv:] == 0).all()


def test_forward_padding_values_do_not_matter():
    B, N, H, D, G, nv = 1, 2048, 4, 128, 512, 1700
    x = synthetic.draw(B, N, H, D, seed=7)
    y = {n: t.clone() for n, t in x.items()}
    for n in ("q", "k", "v"):
        y[n][:, nv:] = torch.randn_like(y[n][:, nv:].float()).to(torch.bfloat16) * 9
    for variant in (STRICT, ROLLED):
        oa, la = _run(x, G, variant, nv)
        ob, lb = _run(y, G, variant, nv)
        assert torch.equal(oa, ob) and torch.equal(la, lb)


def test_forward_sharpened_keys_small():
    # the long-context workload's K x2 on 5% of positions, at a size the oracle finishes quickly
    x = synthetic.draw(1, 2048, 4, 128, seed=3, sharpen_k=True)
    o, lse = _run(x, 1024, STRICT)
    ref = oracle.attention(x["q"], x["k"], x["v"], G=1024, variant=STRICT)
    check_o(o, ref["o"])
    check_lse(lse, ref["lse"])


def test_forward_adjacency_through_the_numeric_kernel():
    # Q = K = 0 makes P uniform over the visible set; V one-hot over a block of D
    # keys turns "key j visible from row i" into O[i, j - block] != 0.
    N, G, D, H = 1024, 256, 64, 2
    for variant in (STRICT, ROLLED):
        for nv in (N, 901):
            got = np.zeros((2, N, N), dtype=bool)
            z = torch.zeros(1, N, H, D, dtype=torch.bfloat16, device="cuda")
            for blk in range(N // D):
                v = torch.zeros(1, N, H, D, dtype=torch.bfloat16, device="cuda")
                idx = torch.arange(D, device="cuda")
                v[0, blk * D + idx, :, idx] = 1
                o, _ = s2.forward(z, z, v, G, variant, nv)
                got[:, :, blk * D:(blk + 1) * D] = (o[0].float().cpu().numpy() != 0).transpose(1, 0, 2)
            for cls in (0, 1):
                A = oracle.adjacency(N, G, nv, variant, cls)
                np.testing.assert_array_equal(got[cls], A, err_msg=str((variant, nv, cls)))
