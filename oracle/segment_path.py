"""Second, independent route to S²-Attn for self-checking the oracle.

TEST INFRASTRUCTURE ONLY.

"4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §1 asks for two references that
must agree: the explicit (i, j) mask (``s2_oracle.c``) and the route the
authors' code takes -- shift the second half of the heads, reshape the
sequence into groups that become batch rows, run ordinary causal attention in
each group, inverse-shift the outputs.  This module is that second route, in
plain PyTorch float64 on the CPU, with gradients from autograd:

* heads [0, H/2): reshape [B, N, ...] -> [B, M, G, ...], causal per group;
* heads [H/2, H), strict variant: slice into the short head segment [0, s),
  the full groups [s + kG, s + kG + G) and the short tail [N - s, N), causal
  per slice (the "staggered cumulative lengths" of §1);
* heads [H/2, H), rolled variant: torch.roll by -s along the sequence,
  reshape into groups with the in-group triangular mask, roll back by +s;
* dense-causal variant: one causal attention over [0, N).

Padding (§1): positions >= n_valid are masked as keys; their query rows give
o = 0, lse = -inf and receive no gradient.
"""
from __future__ import annotations

import math

import torch

STRICT, ROLLED, DENSE_CAUSAL = 0, 1, 2


def _causal_block(q, k, v, pos, n_valid):
    """Causal softmax attention over one ordered segment.

    q, k, v: [B, L, h, D] float64; pos: [L] original positions of the rows.
    Returns o [B, L, h, D] and lse [B, h, L].
    """
    B, L, h, D = q.shape
    scale = 1.0 / math.sqrt(D)
    s = torch.einsum("bihd,bjhd->bhij", q, k) * scale
    tri = torch.ones(L, L, dtype=torch.bool).tril()
    key_ok = (pos < n_valid)[None, :]
    row_ok = (pos < n_valid)[:, None]
    allowed = tri & key_ok & row_ok
    s = s.masked_fill(~allowed, float("-inf"))
    lse = torch.logsumexp(s, dim=-1)  # -inf on fully masked rows
    safe_lse = torch.where(torch.isfinite(lse), lse, torch.zeros_like(lse))
    p = torch.exp(s - safe_lse[..., None])  # exp(-inf) = 0 on masked entries
    o = torch.einsum("bhij,bjhd->bihd", p, v)
    return o, lse


def _segments(N, G, variant, head_class):
    """Ordered lists of original positions, one per segment."""
    s = G // 2
    if variant == DENSE_CAUSAL:
        return [torch.arange(N)]
    if head_class == 0:
        return [torch.arange(a, a + G) for a in range(0, N, G)]
    if variant == STRICT:
        segs = [torch.arange(0, s)]
        segs += [torch.arange(a, a + G) for a in range(s, N - s, G)]
        segs.append(torch.arange(N - s, N))
        return segs
    # rolled: rolled[t] = orig[(t + s) mod N], then groups of G in rolled order
    rolled = torch.roll(torch.arange(N), -s)
    return [rolled[a:a + G] for a in range(0, N, G)]


def forward(q, k, v, *, G, variant, n_valid=None):
    """S²-Attn forward by the shift/reshape route.  q, k, v: [B, N, H, D] float64."""
    B, N, H, D = q.shape
    nv = N if n_valid is None else n_valid
    o = torch.zeros_like(q)
    lse = torch.full((B, H, N), float("-inf"), dtype=q.dtype)
    halves = [(0, H // 2, 0), (H // 2, H, 1)]
    for h0, h1, cls in halves:
        for seg in _segments(N, G, variant, cls):
            ob, lb = _causal_block(q[:, seg, h0:h1], k[:, seg, h0:h1], v[:, seg, h0:h1], seg, nv)
            o = o.index_put((torch.arange(B)[:, None, None], seg[None, :, None],
                             torch.arange(h0, h1)[None, None, :]), ob)
            lse = lse.index_put((torch.arange(B)[:, None, None], torch.arange(h0, h1)[None, :, None],
                                 seg[None, None, :]), lb)
    valid_rows = (torch.arange(N) < nv)[None, :, None, None]
    o = torch.where(valid_rows, o, torch.zeros_like(o))
    return o, lse


def forward_backward(q, k, v, dout, *, G, variant, n_valid=None):
    """Forward plus gradients of L = sum over valid rows of dout·o."""
    q = q.detach().clone().requires_grad_(True)
    k = k.detach().clone().requires_grad_(True)
    v = v.detach().clone().requires_grad_(True)
    o, lse = forward(q, k, v, G=G, variant=variant, n_valid=n_valid)
    N = q.shape[1]
    nv = N if n_valid is None else n_valid
    mask = (torch.arange(N) < nv)[None, :, None, None].to(q.dtype)
    (o * dout * mask).sum().backward()
    return o.detach(), lse.detach(), q.grad, k.grad, v.grad
