"""The forward over CTA pairs (S2_OPT_FWD_PAIRS, tcgen05 cta_group::2) against
the float64 oracle and the single-CTA forward (needs a B200).

Each cluster of two CTAs owns four query tiles; a pair's products span both
CTAs.  The cases cover segments whose tile count is not a multiple of four
(absent tiles in a cluster), short STRICT head and tail groups, the rolled
wrap group, padding inside a tile and in whole tiles, and dense causal.
"""
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


@pytest.fixture
def pairs():
    s2.set_fwd_pairs(True)
    yield
    s2.set_fwd_pairs(False)


def _both(x, G, variant, nv):
    dev = {n: t.cuda() for n, t in x.items()}
    s2.set_fwd_pairs(False)
    o1, l1 = s2.forward(dev["q"], dev["k"], dev["v"], G, variant, nv)
    s2.set_fwd_pairs(True)
    o2, l2 = s2.forward(dev["q"], dev["k"], dev["v"], G, variant, nv)
    torch.cuda.synchronize()
    s2.check_status()
    return (o1, l1), (o2, l2)


CASES = [
    # (B, N, H, D, G, variant, n_valid)
    (1, 1024, 2, 128, 512, STRICT, None),      # 4 tiles per group; short head / tail of 2 tiles
    (1, 1024, 4, 128, 256, STRICT, None),      # 2 tiles per group: half-empty clusters
    (1, 1536, 2, 128, 768, STRICT, None),      # 6 tiles per group
    (2, 2048, 4, 128, 512, ROLLED, None),
    (2, 2048, 4, 128, 512, STRICT, 1900),      # ragged tail inside a tile
    (1, 4096, 2, 128, 1024, ROLLED, 3000),     # padding in the wrap group
    (1, 2048, 2, 128, 2048, DENSE, None),
    (1, 1536, 4, 128, 768, DENSE, 1409),
    (1, 1536, 2, 128, 768, STRICT, 129),       # one valid tile
]


@pytest.mark.parametrize("B,N,H,D,G,variant,nv", CASES)
def test_pair_forward_matches_oracle_and_single_cta(pairs, B, N, H, D, G, variant, nv):
    x = synthetic.draw(B, N, H, D, seed=4000 + N + G + variant)
    (o1, l1), (o2, l2) = _both(x, G, variant, nv)
    ref = oracle.attention(x["q"], x["k"], x["v"], G=G, variant=variant, n_valid=nv)
    where = str((B, N, H, D, G, variant, nv))
    check_o(o2.cpu(), ref["o"], where)
    check_lse(l2.cpu().numpy(), ref["lse"], where)
    d = (o2.float() - o1.float()).abs().max().item()
    assert d < 2e-2, d  # same products in another summation order, bf16 output
    n = N if nv is None else nv
    assert (to_np(o2)[:, n:] == 0).all()


def test_pair_forward_long_context_matches_single_cta(pairs):
    w = synthetic.WORKLOADS["long_n32768_g8192"]
    x = synthetic.draw(1, w.N, 8, w.D, seed=1, sharpen_k=True)
    (o1, l1), (o2, l2) = _both(x, w.G, STRICT, None)
    assert (o2.float() - o1.float()).abs().max().item() < 2e-2
    assert (l2 - l1).abs().max().item() < 2e-3
