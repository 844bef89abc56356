"""The training / inference graph gap on the GPU (needs a B200).

"4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §3: switching from the S² graph
to the full causal graph scales every in-group weight by Z_s / (Z_s + Z_out),
which is exp(lse_S2 - lse_full); §2.1 asks for the gap bucketed by the query's
distance to its group boundary.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from shifted_sparse_attention_b200 import binding as s2
from shifted_sparse_attention_b200 import synthetic

pytestmark = pytest.mark.gpu

STRICT, ROLLED, DENSE = 0, 1, 2


def _local(N, G, variant, cls, i):
    """Position of row i inside its S² segment, from the grouping's definition."""
    s = G // 2
    if cls == 0:
        return i % G
    if variant == STRICT:
        if i < s:
            return i
        if i >= N - s:
            return i - (N - s)
        return (i - s) % G
    return ((i - s) % N) % G  # rolled index (i - s) mod N, position inside its group


def _stats_ref(rho, dist, N, H, G, variant, nv):
    out = np.zeros((2, s2.S2_GAP_BUCKETS, 4))
    acc = {}
    for h in range(H):
        cls = 1 if h >= H // 2 else 0
        for i in range(nv):
            k = int(math.floor(math.log2(_local(N, G, variant, cls, i) + 1)))
            acc.setdefault((cls, k), []).append((rho[:, h, i], dist[:, h, i]))
    for (cls, k), v in acc.items():
        r = np.concatenate([a for a, _ in v])
        d = np.concatenate([b for _, b in v])
        out[cls, k] = (len(r), r.mean(), r.min(), d.mean())
    return out


@pytest.mark.parametrize("B,N,H,D,G,variant,nv", [
    (1, 2048, 4, 128, 512, STRICT, None),
    (2, 2048, 4, 128, 512, ROLLED, 1900),
    (1, 1024, 8, 64, 256, STRICT, 1000),
])
def test_graph_gap_matches_oracle(B, N, H, D, G, variant, nv):
    x = synthetic.draw(B, N, H, D, seed=900 + N + variant, with_dout=False)
    n = N if nv is None else nv
    rho, dist, stats = (t.cpu().numpy() for t in s2.graph_gap(*(x[c].cuda() for c in "qkv"), G, variant, nv))
    a = oracle.attention(x["q"], x["k"], x["v"], G=G, variant=variant, n_valid=nv)
    f = oracle.attention(x["q"], x["k"], x["v"], G=N, variant=DENSE, n_valid=nv)
    rho_ref = np.exp(a["lse"][:, :, :n] - f["lse"][:, :, :n])
    dist_ref = np.linalg.norm(a["o"] - f["o"], axis=-1).transpose(0, 2, 1)[:, :, :n]
    assert np.abs(rho[:, :, :n] - rho_ref).max() <= 1e-2 * rho_ref.max()
    assert np.abs(dist[:, :, :n] - dist_ref).mean() <= 1e-2
    assert (rho[:, :, n:] == 0).all() and (dist[:, :, n:] == 0).all()
    ref = _stats_ref(rho_ref, dist_ref, N, H, G, variant, n)
    np.testing.assert_array_equal(stats[..., 0], ref[..., 0])  # row counts per class and bucket
    used = ref[..., 0] > 0
    assert np.abs(stats[..., 1][used] - ref[..., 1][used]).max() < 1e-2
    assert np.abs(stats[..., 2][used] - ref[..., 2][used]).max() < 1e-2
    assert np.abs(stats[..., 3][used] - ref[..., 3][used]).max() < 2e-2
    if variant == STRICT:  # S_i ⊂ F_i: the in-group share never exceeds 1
        assert rho[:, :, :n].max() <= 1.0 + 1e-5


@pytest.mark.parametrize("variant", [STRICT, ROLLED])
def test_graph_gap_uniform_logits_closed_form(variant):
    # Q = 0: every visible logit is 0, so Z_s = |S_i| and Z_s + Z_out = |F_i| = i + 1
    B, N, H, D, G = 1, 2048, 4, 128, 512
    x = synthetic.draw(B, N, H, D, seed=5, with_dout=False)
    x["q"].zero_()
    rho, _, stats = (t.cpu().numpy() for t in s2.graph_gap(*(x[c].cuda() for c in "qkv"), G, variant))
    s = G // 2
    for h in range(H):
        cls = 1 if h >= H // 2 else 0
        i = np.arange(N)
        if cls == 1 and variant == ROLLED:
            size_s = np.array([_local(N, G, variant, 1, t) + 1 for t in i])  # the rolled group may reach past i
        else:
            size_s = np.array([_local(N, G, variant, cls, t) + 1 for t in i])
        np.testing.assert_allclose(rho[0, h], size_s / (i + 1), rtol=1e-5)
    # class-0 rows of the first group see their whole history: rho = 1 there
    np.testing.assert_allclose(rho[0, : H // 2, :G], 1.0, rtol=1e-6)
    assert stats[0, 0, 0] == (H // 2) * (N // G)  # bucket 0 = the first row of every class-0 group
