"""Sequence-parallel S²-Attn: one process per GPU, each holding a G-aligned shard.

"4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §1.1 ("Sequence Parallel通信"):
when the sequence is cut into shards whose boundaries are group boundaries,
only the shifted heads' group that straddles a boundary needs data from the
neighbouring rank: the s = G/2 K/V rows in front of the shard (the halo).
Exchanging exactly that halo, instead of rolling inside each shard, keeps the
multi-rank graph identical to the single-GPU graph; the backward returns the
halo rows' partial gradients to their owner.  Per direction the message is
V_KV = 2·B·(H/2)·s·D·2 bytes, the pages' volume.

Every tensor of a rank lives in an extended buffer [B, s + L, H, D] whose rows
[0, s) are the halo (``extended`` allocates one, ``shard`` views the shard
rows).  The halo rows are filled in place by the exchange, so the kernels read
one contiguous tensor.  Movement between buffers and messages runs in
libs2attn.so (``s2attn_sp_halo_pack`` / ``_unpack``); the point-to-point
transfer is torch.distributed (NCCL over NVLink on GPUs), one send and one
receive per rank and direction, issued together so no rank waits on another's
order.  The attention itself is ``s2attn_sp_fwd`` / ``s2attn_sp_bwd``.

Topology: STRICT sends the last shard rows to the next rank (the last rank
sends nothing, rank 0 receives nothing); ROLLED closes the ring (the last
rank's tail is rank 0's halo), which is its wrap-around group.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import binding as s2


class HaloOps:
    """Movement of the shifted heads' halo rows between extended buffers and a
    packed message [2, B, s, H/2, D] (part S2_SP_KV or S2_SP_GRAD; see
    include/s2attn.h).  Runs in libs2attn.so."""

    def pack(self, a, b, msg, B, L, H, D, G, part):
        s2._check(s2.s2attn_sp_halo_pack(a, b, msg, B, L, H, D, G, part))

    def unpack(self, msg, a, b, B, L, H, D, G, part):
        s2._check(s2.s2attn_sp_halo_unpack(msg, a, b, B, L, H, D, G, part))


def extended(B: int, L: int, H: int, D: int, G: int, device=None, dtype=torch.bfloat16) -> torch.Tensor:
    """An extended buffer [B, G/2 + L, H, D] (halo rows first)."""
    return torch.empty((B, G // 2 + L, H, D), dtype=dtype, device=device)


def shard(x_ext: torch.Tensor, G: int) -> torch.Tensor:
    """The shard rows [G/2, G/2 + L) of an extended buffer (a view)."""
    return x_ext[:, G // 2:]


def peers(rank: int, world: int, variant: int):
    """(rank the shard's last rows go to, rank the halo comes from); None where there is none."""
    if variant == s2.ROLLED:
        return (rank + 1) % world, (rank - 1) % world
    return (rank + 1 if rank + 1 < world else None), (rank - 1 if rank > 0 else None)


class SequenceParallelS2Attn:
    """S²-Attn over a sequence sharded across the ranks of ``group``.

    Rank r holds original positions [rL, rL + L) in extended buffers.  ``n_valid``
    is the number of valid rows of this rank's shard (L except on a padded last
    rank)."""

    def __init__(self, G: int, variant: int = s2.STRICT, group=None, ops: HaloOps | None = None):
        if variant not in (s2.STRICT, s2.ROLLED):
            raise ValueError("sequence parallelism supports the STRICT and ROLLED variants")
        self.G, self.s, self.variant, self.group = G, G // 2, variant, group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.ops = ops if ops is not None else HaloOps()

    # -------------------------------------------------------------- halo exchange
    def _dims(self, x_ext):
        B, Ne, H, D = (int(d) for d in x_ext.shape)
        L = Ne - self.s
        if L < self.G or L % self.G:
            raise ValueError("extended buffer of %d rows: the shard must be a multiple of G=%d" % (Ne, self.G))
        return B, L, H, D

    def _message(self, x_ext):
        B, L, H, D = self._dims(x_ext)
        return torch.empty((2, B, self.s, H // 2, D), dtype=x_ext.dtype, device=x_ext.device)

    def _sendrecv(self, send, to, recv, frm):
        if to is not None and to == self.rank and frm == self.rank:  # a ring of one rank
            recv.copy_(send)
            return
        ops = []
        if to is not None:
            ops.append(dist.P2POp(dist.isend, send, dist.get_global_rank(self.group, to) if self.group else to,
                                  self.group))
        if frm is not None:
            ops.append(dist.P2POp(dist.irecv, recv, dist.get_global_rank(self.group, frm) if self.group else frm,
                                  self.group))
        if ops:
            for w in dist.batch_isend_irecv(ops):
                w.wait()

    def exchange_kv(self, k_ext, v_ext):
        """Fill the halo rows of k_ext, v_ext with the previous rank's last s shard rows."""
        B, L, H, D = self._dims(k_ext)
        to, frm = peers(self.rank, self.world, self.variant)
        send = self._message(k_ext) if to is not None else None
        recv = self._message(k_ext) if frm is not None else None
        if send is not None:
            self.ops.pack(k_ext, v_ext, send, B, L, H, D, self.G, s2.S2_SP_KV)
        self._sendrecv(send, to, recv, frm)
        if recv is not None:
            self.ops.unpack(recv, k_ext, v_ext, B, L, H, D, self.G, s2.S2_SP_KV)

    def exchange_grad(self, dk_ext, dv_ext):
        """Return the halo rows' partial dK/dV to the rank they came from, which
        adds them onto its last s shard rows (the reverse of exchange_kv)."""
        B, L, H, D = self._dims(dk_ext)
        to_kv, frm_kv = peers(self.rank, self.world, self.variant)
        send = self._message(dk_ext) if frm_kv is not None else None
        recv = self._message(dk_ext) if to_kv is not None else None
        if send is not None:
            self.ops.pack(dk_ext, dv_ext, send, B, L, H, D, self.G, s2.S2_SP_GRAD)
        self._sendrecv(send, frm_kv, recv, to_kv)
        if recv is not None:
            self.ops.unpack(recv, dk_ext, dv_ext, B, L, H, D, self.G, s2.S2_SP_GRAD)

    # -------------------------------------------------------------- attention
    def forward(self, q_ext, k_ext, v_ext, n_valid: int | None = None, out=None, lse=None, exchange: bool = True):
        """Halo exchange of K/V, then the rank's forward; returns (o_ext, lse_ext [B, H, s + L])."""
        B, L, H, D = self._dims(q_ext)
        nv = L if n_valid is None else int(n_valid)
        if exchange:
            self.exchange_kv(k_ext, v_ext)
        o = torch.empty_like(q_ext) if out is None else out
        l = torch.empty((B, H, self.s + L), dtype=torch.float32, device=q_ext.device) if lse is None else lse
        s2._check(s2.s2attn_sp_fwd(q_ext, k_ext, v_ext, o, l, B, L, H, D, self.G, nv, self.variant, self.rank,
                                   self.world))
        return o, l

    def backward(self, q_ext, k_ext, v_ext, o_ext, dout_ext, lse_ext, n_valid: int | None = None, grads=None,
                 workspace=None, exchange: bool = True, stored_ds: bool = False):
        """The rank's backward (k_ext, v_ext still hold the forward's halo), then the
        halo gradient exchange; returns (dq_ext, dk_ext, dv_ext).  stored_ds: the
        dK/dV stage keeps dS for the dQ stage (see include/s2attn.h)."""
        B, L, H, D = self._dims(q_ext)
        nv = L if n_valid is None else int(n_valid)
        if grads is None:
            grads = (torch.empty_like(q_ext), torch.empty_like(k_ext), torch.empty_like(v_ext))
        dq, dk, dv = grads
        if stored_ds:
            ws_bytes = s2.s2attn_sp_ds_workspace_size(B, L, H, D, self.G, self.variant, self.rank, self.world)
        else:
            ws_bytes = s2.s2attn_bwd_workspace_size(B, self.s + L, H, D)
        if workspace is None:
            workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q_ext.device)
        stages = s2.S2_BWD_ALL_DS if stored_ds else s2.S2_BWD_ALL
        s2._check(s2.s2attn_sp_bwd_stages(q_ext, k_ext, v_ext, o_ext, dout_ext, lse_ext, dq, dk, dv, B, L, H, D,
                                          self.G, nv, self.variant, self.rank, self.world, workspace,
                                          workspace.numel() * workspace.element_size(), stages))
        if exchange:
            self.exchange_grad(dk, dv)
        return dq, dk, dv
