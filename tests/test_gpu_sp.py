"""Sequence-parallel S²-Attn on one GPU (needs a B200): the ranks run in turn.

"4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §1.1: a sequence simulated on one
card and on several cards must give the same visible sets, outputs and
gradients.  Here W ranks are emulated one after another on one GPU: each rank
gets its shard in an extended buffer, the halo rows arrive through the halo
kernels with the message handed over in memory (the transfer the collective
layer does between GPUs), and the rank calls s2attn_sp_fwd / s2attn_sp_bwd.
No kernel waits on another rank, so running them in sequence is exact.

Checked: O, lse and dQ of every row are bitwise the single-GPU results on
the whole sequence; dK, dV bitwise except on the s rows in front of each
shard boundary (two partial sums, one extra rounding), which are held to the
oracle's tolerances; all of it against the float64 oracle at small sizes.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from shifted_sparse_attention_b200 import binding as s2
from shifted_sparse_attention_b200 import sp
from shifted_sparse_attention_b200 import synthetic
from tests.tolerance import check_grad, check_lse, check_o, to_np

pytestmark = pytest.mark.gpu


def _emulate(x, G, variant, W, nv_last, stored=False):
    """Run the W ranks in turn; returns global (o, lse, dq, dk, dv)."""
    B, N, H, D = x["q"].shape
    L, s = N // W, G // 2
    ops = sp.HaloOps()
    ext = {}
    for name in ("q", "k", "v", "dout"):
        bufs = []
        for r in range(W):
            e = sp.extended(B, L, H, D, G, "cuda")
            e.fill_(1.0e4)  # halo rows that are never read as keys must not matter
            sp.shard(e, G).copy_(x[name][:, r * L:(r + 1) * L])
            bufs.append(e)
        ext[name] = bufs
    msg = torch.empty((2, B, s, H // 2, D), dtype=torch.bfloat16, device="cuda")
    for r in range(W):  # K/V halo: rank r receives from the rank before it
        to, frm = sp.peers(r, W, variant)
        if frm is not None:
            ops.pack(ext["k"][frm], ext["v"][frm], msg, B, L, H, D, G, s2.S2_SP_KV)
            ops.unpack(msg, ext["k"][r], ext["v"][r], B, L, H, D, G, s2.S2_SP_KV)
    outs = []
    for r in range(W):
        nv = nv_last if r == W - 1 else L
        o = torch.empty_like(ext["q"][r])
        lse = torch.empty((B, H, s + L), dtype=torch.float32, device="cuda")
        s2._check(s2.s2attn_sp_fwd(ext["q"][r], ext["k"][r], ext["v"][r], o, lse, B, L, H, D, G, nv, variant, r, W))
        dq, dk, dv = (torch.empty_like(o) for _ in range(3))
        if stored:
            ws = torch.empty(s2.s2attn_sp_ds_workspace_size(B, L, H, D, G, variant, r, W), dtype=torch.uint8,
                             device="cuda")
        else:
            ws = torch.empty(s2.s2attn_bwd_workspace_size(B, s + L, H, D), dtype=torch.uint8, device="cuda")
        s2._check(s2.s2attn_sp_bwd_stages(ext["q"][r], ext["k"][r], ext["v"][r], o, ext["dout"][r], lse, dq, dk, dv,
                                          B, L, H, D, G, nv, variant, r, W, ws, ws.numel(),
                                          s2.S2_BWD_ALL_DS if stored else s2.S2_BWD_ALL))
        outs.append(dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv))
    for r in range(W):  # halo gradients go back to the rank the halo came from
        to, frm = sp.peers(r, W, variant)
        if frm is not None:
            ops.pack(outs[r]["dk"], outs[r]["dv"], msg, B, L, H, D, G, s2.S2_SP_GRAD)
            ops.unpack(msg, outs[frm]["dk"], outs[frm]["dv"], B, L, H, D, G, s2.S2_SP_GRAD)
    torch.cuda.synchronize()
    s2.check_status()
    cat = lambda n: torch.cat([sp.shard(outs[r][n], G) for r in range(W)], dim=1)
    lse = torch.cat([outs[r]["lse"][:, :, s:] for r in range(W)], dim=2)
    return cat("o"), lse, cat("dq"), cat("dk"), cat("dv")


def _single(x, G, variant, nv, stored=False):
    dev = {n: t.cuda() for n, t in x.items()}
    o, lse = s2.forward(dev["q"], dev["k"], dev["v"], G, variant, nv)
    dq, dk, dv = s2.backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, G, variant, nv, stored_ds=stored)
    torch.cuda.synchronize()
    s2.check_status()
    return o, lse, dq, dk, dv


def _boundary_rows(N, L, s, W, variant):
    rows = np.zeros(N, dtype=bool)
    for r in range(1, W):
        rows[r * L - s:r * L] = True
    if variant == 1:
        rows[N - s:] = True  # the ring: rank 0's halo is the last rank's tail
    return rows


CASES = [
    # B, H, D, G, W, L, variant, padding of the last rank
    (1, 4, 64, 256, 2, 512, 0, 0),
    (1, 4, 128, 256, 4, 512, 0, 0),
    (2, 2, 128, 512, 3, 512, 0, 100),
    (1, 4, 128, 256, 4, 512, 1, 0),
    (1, 2, 64, 512, 2, 1024, 1, 0),
    (1, 4, 128, 256, 1, 512, 0, 0),
    (1, 4, 128, 256, 1, 512, 1, 0),
]


@pytest.mark.parametrize("stored", [False, True], ids=["recompute", "stored_ds"])
@pytest.mark.parametrize("B,H,D,G,W,L,variant,pad", CASES)
def test_sequence_parallel_matches_single_gpu_and_oracle(B, H, D, G, W, L, variant, pad, stored):
    N, s = W * L, G // 2
    nv = N - pad
    x = synthetic.draw(B, N, H, D, seed=W * 100 + L + variant)
    o, lse, dq, dk, dv = _emulate(x, G, variant, W, L - pad, stored)
    o1, lse1, dq1, dk1, dv1 = _single(x, G, variant, nv, stored)
    assert torch.equal(o, o1)
    assert torch.equal(lse, lse1)
    assert torch.equal(dq, dq1)
    inner = torch.from_numpy(~_boundary_rows(N, L, s, W, variant)).cuda()
    assert torch.equal(dk[:, inner], dk1[:, inner]) and torch.equal(dv[:, inner], dv1[:, inner])
    # class-0 heads never cross a shard boundary: bitwise everywhere
    assert torch.equal(dk[:, :, : H // 2], dk1[:, :, : H // 2])
    ref = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant, n_valid=nv)
    check_o(o[:, :nv], ref["o"][:, :nv])
    check_lse(lse.cpu().numpy(), ref["lse"])
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        check_grad(name, g[:, :nv], ref[name][:, :nv])
    assert (to_np(dk[:, nv:]) == 0).all() and (to_np(dv[:, nv:]) == 0).all()


def test_sequence_parallel_long_shards_bitwise():
    # four ranks of L = 8192 (G = 4096): the single-GPU N = 32768 sequence, bitwise
    B, H, D, G, W, L = 1, 8, 128, 4096, 4, 8192
    x = synthetic.draw(B, W * L, H, D, seed=5, sharpen_k=True)
    o, lse, dq, dk, dv = _emulate(x, G, 0, W, L)
    o1, lse1, dq1, dk1, dv1 = _single(x, G, 0, W * L)
    assert torch.equal(o, o1) and torch.equal(lse, lse1) and torch.equal(dq, dq1)
    inner = torch.from_numpy(~_boundary_rows(W * L, L, G // 2, W, 0)).cuda()
    assert torch.equal(dk[:, inner], dk1[:, inner]) and torch.equal(dv[:, inner], dv1[:, inner])
    # boundary rows: two partial sums, each rounded, then summed and rounded once more
    for a, b in ((dk, dk1), (dv, dv1)):
        d = (a.float() - b.float()).abs().max().item() / b.float().abs().max().item()
        assert d < 1e-2, d


def test_halo_kernels_match_indexing():
    B, H, D, G, L = 2, 6, 128, 512, 1024
    s = G // 2
    g = torch.Generator().manual_seed(3)
    a = torch.randn(B, s + L, H, D, generator=g).bfloat16().cuda()
    b = torch.randn(B, s + L, H, D, generator=g).bfloat16().cuda()
    msg = torch.empty((2, B, s, H // 2, D), dtype=torch.bfloat16, device="cuda")
    assert s2.s2attn_sp_halo_bytes(B, H, D, G) == msg.numel() * 2
    ops = sp.HaloOps()
    ops.pack(a, b, msg, B, L, H, D, G, s2.S2_SP_KV)
    torch.cuda.synchronize()
    assert torch.equal(msg[0], a[:, L:L + s, H // 2:]) and torch.equal(msg[1], b[:, L:L + s, H // 2:])
    a2, b2 = a.clone(), b.clone()
    ops.unpack(msg, a2, b2, B, L, H, D, G, s2.S2_SP_KV)
    ea, eb = a.clone(), b.clone()
    ea[:, :s, H // 2:] = a[:, L:L + s, H // 2:]
    eb[:, :s, H // 2:] = b[:, L:L + s, H // 2:]
    torch.cuda.synchronize()
    assert torch.equal(a2, ea) and torch.equal(b2, eb)
    ops.pack(a, b, msg, B, L, H, D, G, s2.S2_SP_GRAD)
    a3, b3 = a.clone(), b.clone()
    ops.unpack(msg, a3, b3, B, L, H, D, G, s2.S2_SP_GRAD)
    ea, eb = a.clone(), b.clone()
    ea[:, L:L + s, H // 2:] = (a[:, L:L + s, H // 2:].float() + a[:, :s, H // 2:].float()).bfloat16()
    eb[:, L:L + s, H // 2:] = (b[:, L:L + s, H // 2:].float() + b[:, :s, H // 2:].float()).bfloat16()
    torch.cuda.synchronize()
    assert torch.equal(a3, ea) and torch.equal(b3, eb)
