"""Sequence-parallel halo exchange on gloo ranks (CPU only).

"4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §1.1 ("Sequence Parallel通信"):
the shifted heads need the s = G/2 rows in front of each shard from the
previous rank, and the backward returns those rows' gradients.  These tests
run shifted_sparse_attention_b200.sp's exchange logic (peers, message shapes,
send/receive pairing, the ring of ROLLED) over real torch.distributed gloo
point-to-point with host stand-ins for the two halo kernels (plain tensor
indexing, defined here), and check which rows arrive where.  The kernels
themselves are checked against the same indexing on the GPU.
"""
from __future__ import annotations

import json
import os
import socket
import sys
from pathlib import Path

import pytest
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parent.parent


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class HostHaloOps:
    """Host stand-in for the halo kernels: the shifted heads [H/2, H) of rows
    [L, L + s) (KV) or [0, s) (GRAD) to and from a [2, B, s, H/2, D] message."""

    def __init__(self):
        self.messages = []

    def pack(self, a, b, msg, B, L, H, D, G, part):
        s = G // 2
        r0 = L if part == 0 else 0
        msg[0] = a[:, r0:r0 + s, H // 2:]
        msg[1] = b[:, r0:r0 + s, H // 2:]
        self.messages.append(msg.numel() * msg.element_size())

    def unpack(self, msg, a, b, B, L, H, D, G, part):
        s = G // 2
        if part == 0:
            a[:, :s, H // 2:] = msg[0]
            b[:, :s, H // 2:] = msg[1]
        else:
            a[:, L:L + s, H // 2:] = (a[:, L:L + s, H // 2:].float() + msg[0].float()).bfloat16()
            b[:, L:L + s, H // 2:] = (b[:, L:L + s, H // 2:].float() + msg[1].float()).bfloat16()


def _rank_main(rank, world, port, variant, out_dir):
    import datetime

    import torch
    import torch.distributed as dist

    sys.path.insert(0, str(ROOT))
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from shifted_sparse_attention_b200 import sp

    B, H, D, G = 2, 4, 8, 8
    s, L = G // 2, 2 * G
    N = world * L
    g = torch.Generator().manual_seed(1)
    K = torch.randn(B, N, H, D, generator=g).bfloat16()
    V = torch.randn(B, N, H, D, generator=g).bfloat16()
    sentinel = -77.0
    k_ext = torch.full((B, s + L, H, D), sentinel).bfloat16()
    v_ext = torch.full((B, s + L, H, D), sentinel).bfloat16()
    sp.shard(k_ext, G).copy_(K[:, rank * L:(rank + 1) * L])
    sp.shard(v_ext, G).copy_(V[:, rank * L:(rank + 1) * L])
    ops = HostHaloOps()
    par = sp.SequenceParallelS2Attn(G, variant, ops=ops)
    par.exchange_kv(k_ext, v_ext)
    ok = {}
    prev = (rank - 1) % world
    has_halo = variant == 1 or rank > 0
    want_k = K[:, prev * L + L - s: prev * L + L, H // 2:] if has_halo else torch.full((B, s, H // 2, D), sentinel).bfloat16()
    want_v = V[:, prev * L + L - s: prev * L + L, H // 2:] if has_halo else torch.full((B, s, H // 2, D), sentinel).bfloat16()
    ok["halo_k"] = torch.equal(k_ext[:, :s, H // 2:], want_k)
    ok["halo_v"] = torch.equal(v_ext[:, :s, H // 2:], want_v)
    ok["class0_untouched"] = bool((k_ext[:, :s, :H // 2].float() == sentinel).all())
    ok["shard_untouched"] = torch.equal(sp.shard(k_ext, G), K[:, rank * L:(rank + 1) * L])

    # gradients: shard rows hold A_r, halo rows hold partial gradients P_r
    A = torch.randn(world, B, s + L, H, D, generator=g).bfloat16()
    dk_ext = A[rank].clone()
    dv_ext = (2 * A[rank]).clone()
    par.exchange_grad(dk_ext, dv_ext)
    nxt = (rank + 1) % world
    gets = variant == 1 or rank + 1 < world
    exp_k = A[rank].clone()
    exp_v = (2 * A[rank]).clone()
    if gets:
        exp_k[:, L:L + s, H // 2:] = (A[rank][:, L:L + s, H // 2:].float() + A[nxt][:, :s, H // 2:].float()).bfloat16()
        exp_v[:, L:L + s, H // 2:] = ((2 * A[rank])[:, L:L + s, H // 2:].float()
                                      + (2 * A[nxt])[:, :s, H // 2:].float()).bfloat16()
    ok["grad_k"] = torch.equal(dk_ext, exp_k)
    ok["grad_v"] = torch.equal(dv_ext, exp_v)
    ok["message_bytes"] = all(m == 2 * B * (H // 2) * s * D * 2 for m in ops.messages)  # V_KV
    ok["n_messages"] = len(ops.messages)
    dist.barrier()
    dist.destroy_process_group()
    Path(out_dir, "r%d.json" % rank).write_text(json.dumps(ok))


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("variant", [0, 1])
def test_halo_exchange_over_gloo(tmp_path, world, variant):
    mp.start_processes(_rank_main, args=(world, _free_port(), variant, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        ok = json.loads((tmp_path / ("r%d.json" % r)).read_text())
        n = ok.pop("n_messages")
        assert all(ok.values()), (r, ok)
        # packs: one K/V message unless this rank sends nothing (STRICT last rank),
        # one gradient message unless it received no halo (STRICT rank 0)
        expect = 2 if variant == 1 else (r + 1 < world) + (r > 0)
        assert n == expect, (r, n)


def test_peers():
    from shifted_sparse_attention_b200 import sp

    assert sp.peers(0, 1, 0) == (None, None)
    assert sp.peers(0, 1, 1) == (0, 0)
    assert sp.peers(0, 3, 0) == (1, None)
    assert sp.peers(2, 3, 0) == (None, 1)
    assert sp.peers(0, 3, 1) == (1, 2)
    assert sp.peers(2, 3, 1) == (0, 1)
