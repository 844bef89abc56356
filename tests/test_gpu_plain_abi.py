"""The plain entry points s2attn_fwd / s2attn_bwd (no valid length: n_valid = N)
on the small workload's own inputs (B=1, H=8, N=1024, D=64, G=256, strict,
seed 0), checked element by element against the float64 oracle (needs a B200).
Every other numeric test goes through the _v, staged or document forms."""
from __future__ import annotations

import pytest
import torch

import oracle
from shifted_sparse_attention_b200 import binding as s2
from shifted_sparse_attention_b200 import synthetic
from tests.tolerance import check_grad, check_lse, check_o, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("variant", [s2.STRICT, s2.ROLLED])
def test_plain_symbols_on_the_small_workload(variant):
    w = synthetic.WORKLOADS["small_n1024_g256"]
    B, N, H, D, G = w.B, w.N, w.H, w.D, w.G
    x = synthetic.workload_inputs(w.name)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "dout"))
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device="cuda")
    s2._check(s2.s2attn_fwd(q, k, v, o, lse, B, N, H, D, G, variant))
    ws_bytes = s2.s2attn_bwd_workspace_size(B, N, H, D)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
    s2._check(s2.s2attn_bwd(q, k, v, o, do, lse, dq, dk, dv, B, N, H, D, G, variant, ws, ws_bytes))
    torch.cuda.synchronize()
    s2.check_status()
    ref = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant)
    where = "small workload, plain symbols, variant %d" % variant
    check_o(o, ref["o"], where)
    check_lse(lse, ref["lse"], where)
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        check_grad(name, to_np(g), ref[name], where)
