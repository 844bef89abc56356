"""Rotary position prologue on the GPU (needs a B200).

"4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §1.1 ("RoPE使用原始位置"): Q and K
are rotated at each token's original position ID with position interpolation
p -> p·scale.  The kernel is compared with the float64 reference
(oracle/rope.py) on the same bf16 inputs: it forms angles in float64,
rotates in float32 and rounds once to bf16, so every element lies within
half a bf16 ulp of the exact rotation plus a float32 term, and almost every
element equals the exact rotation rounded to bf16.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import rope as rope_ref
from shifted_sparse_attention_b200 import binding as s2

pytestmark = pytest.mark.gpu


def _inputs(B, N, H, D, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, N, H, D, generator=g).to(torch.bfloat16)
    k = torch.randn(B, N, H, D, generator=g).to(torch.bfloat16)
    return q, k


def _check(got, x, positions, base, scale):
    """got (bf16, device) against the float64 rotation of x (bf16, host)."""
    ref = rope_ref.rope(x, positions, base=base, scale=scale)
    g = got.float().cpu().double().numpy()
    xd = x.double().numpy()
    D = xd.shape[-1]
    pair = np.abs(xd[..., : D // 2]) + np.abs(xd[..., D // 2:])
    slack = 1e-6 * np.concatenate([pair, pair], axis=-1)
    bound = 2.0 ** -8 * (np.abs(ref) + slack) + slack
    err = np.abs(g - ref)
    assert (err <= bound).all(), float((err - bound).max())
    # the exact result rounded to bf16 is hit except at near-ties
    ref_bf16 = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
    assert (g != ref_bf16).mean() < 2e-3


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("B,N,H", [(1, 1, 1), (2, 1003, 5), (1, 4096, 8)])
def test_rope_default_positions(B, N, H, D):
    q, k = _inputs(B, N, H, D, seed=N + D)
    qo, ko = s2.rope(q.cuda(), k.cuda())
    torch.cuda.synchronize()
    _check(qo, q, None, 10000.0, 1.0)
    _check(ko, k, None, 10000.0, 1.0)


@pytest.mark.parametrize("D", [64, 128])
def test_rope_packed_positions_and_interpolation(D):
    # positions restart at each packed document; interpolation factor L0/L1 = 1/4
    B, N, H = 2, 3000, 4
    rng = np.random.default_rng(D)
    pos = np.zeros((B, N), dtype=np.int32)
    for b in range(B):
        cuts = np.sort(rng.choice(np.arange(1, N), size=5, replace=False))
        start = 0
        for c in list(cuts) + [N]:
            pos[b, start:c] = np.arange(c - start)
            start = c
    q, k = _inputs(B, N, H, D, seed=3 + D)
    qo, ko = s2.rope(q.cuda(), k.cuda(), torch.from_numpy(pos).cuda(), base=500000.0, scale=0.25)
    torch.cuda.synchronize()
    _check(qo, q, pos, 500000.0, 0.25)
    _check(ko, k, pos, 500000.0, 0.25)


def test_rope_large_positions():
    # angles near 10^6 rad: a float32 angle would lose the rotation entirely
    B, N, H, D = 1, 8, 2, 128
    pos = np.array([[0, 1, 2, 8191, 32767, 65535, 99999, 1000000]], dtype=np.int32)
    q, k = _inputs(B, N, H, D, seed=11)
    qo, ko = s2.rope(q.cuda(), k.cuda(), torch.from_numpy(pos).cuda())
    torch.cuda.synchronize()
    _check(qo, q, pos, 10000.0, 1.0)
    _check(ko, k, pos, 10000.0, 1.0)


def test_rope_in_place_matches_out_of_place():
    q, k = _inputs(2, 2048, 4, 128, seed=5)
    qo, ko = s2.rope(q.cuda(), k.cuda(), scale=0.5)
    qi, ki = q.cuda(), k.cuda()
    qr, kr = s2.rope(qi, ki, scale=0.5, inplace=True)
    torch.cuda.synchronize()
    assert qr.data_ptr() == qi.data_ptr() and kr.data_ptr() == ki.data_ptr()
    assert torch.equal(qi, qo) and torch.equal(ki, ko)


def test_rope_positions_travel_with_their_tokens():
    # rotating a shifted copy at its tokens' original positions, then shifting back,
    # is bit-identical to rotating in place: the rotation never sees the grouping
    B, N, H, D, G = 1, 4096, 4, 128, 1024
    q, k = _inputs(B, N, H, D, seed=9)
    pos = torch.arange(N, dtype=torch.int32).expand(B, N).contiguous()
    qa, ka = s2.rope(q.cuda(), k.cuda())
    qs = torch.roll(q, -G // 2, dims=1).contiguous().cuda()
    ks = torch.roll(k, -G // 2, dims=1).contiguous().cuda()
    ps = torch.roll(pos, -G // 2, dims=1).contiguous().cuda()
    qb, kb = s2.rope(qs, ks, ps)
    torch.cuda.synchronize()
    assert torch.equal(torch.roll(qb, G // 2, dims=1), qa)
    assert torch.equal(torch.roll(kb, G // 2, dims=1), ka)


def test_rope_then_attention_sees_relative_positions():
    # shifting every position by a constant leaves the S² forward unchanged up to rounding
    B, N, H, D, G = 1, 2048, 4, 128, 512
    q, k = _inputs(B, N, H, D, seed=13)
    v = torch.randn(B, N, H, D, generator=torch.Generator().manual_seed(14)).to(torch.bfloat16).cuda()
    outs = []
    for off in (0, 4096):
        pos = (torch.arange(N, dtype=torch.int32) + off).expand(B, N).contiguous().cuda()
        qr, kr = s2.rope(q.cuda(), k.cuda(), pos)
        o, _ = s2.forward(qr, kr, v, G, 0)
        outs.append(o.float())
    s2.check_status()
    assert (outs[0] - outs[1]).abs().max().item() < 3e-2
