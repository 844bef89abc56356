"""The allocation-free backward entry point (needs a B200).

s2attn_bwd_noalloc_v serves callers that cannot allocate device memory (a
plug-in inside a framework that owns the device heap, a runtime held to a
fixed footprint): it takes its scratch from a fixed array inside the library
instead of a caller-provided workspace.  Its results must match s2attn_bwd_v
(same tolerance as the other backward tests) on two calls in a row.  Before
the checked calls, one call on other inputs and a larger shape fills more of
the shared array with other statistics, so the checked calls show that what
an earlier call left behind is overwritten.  This file is collected last so
that a failure here does not hide the other tests' results.
"""
from __future__ import annotations

import pytest
import torch

from shifted_sparse_attention_b200 import binding as s2
from shifted_sparse_attention_b200 import synthetic
from tests.tolerance import check_grad

pytestmark = pytest.mark.gpu


def _noalloc(q, k, v, o, do, lse, B, N, H, D, G, n_valid, variant):
    L = s2.lib()
    dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
    rc = L.s2attn_bwd_noalloc_v(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                                lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                B, N, H, D, G, n_valid, variant, torch.cuda.current_stream().cuda_stream)
    assert rc == s2.S2_OK, s2.s2attn_last_error()
    return dq, dk, dv


def _fill_scratch_with_other_statistics():
    # B*H*N = 2*8*4096: twice the statistics of the largest checked case, other seed
    B, N, H, D, G = 2, 4096, 8, 128, 1024
    x = synthetic.draw(B, N, H, D, seed=4242)
    q, k, v, do = (t.cuda() for t in (x["q"], x["k"], x["v"], x["dout"]))
    do.mul_(7)  # statistics unlike the checked cases'
    o, lse = s2.forward(q, k, v, G, s2.ROLLED, N - 100)
    _noalloc(q, k, v, o, do, lse, B, N, H, D, G, N - 100, s2.ROLLED)
    torch.cuda.synchronize()


@pytest.mark.parametrize("B,N,H,D,G,variant,nv", [
    (2, 2048, 4, 128, 512, 0, 1900),
    (1, 2048, 4, 128, 512, 1, None),
    (1, 1024, 8, 64, 256, 0, None),
])
def test_noalloc_backward_matches_workspace_backward(B, N, H, D, G, variant, nv):
    n_valid = N if nv is None else nv
    x = synthetic.draw(B, N, H, D, seed=77 + N + variant)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "dout"))
    o, lse = s2.forward(q, k, v, G, variant, n_valid)
    ref = s2.backward(q, k, v, o, do, lse, G, variant, n_valid)
    _fill_scratch_with_other_statistics()
    for call in range(2):
        dq, dk, dv = _noalloc(q, k, v, o, do, lse, B, N, H, D, G, n_valid, variant)
        torch.cuda.synchronize()
        s2.check_status()
        for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
            check_grad(name, got.float().cpu().numpy(), want.float().cpu().numpy(), "call %d" % call)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    L = s2.lib()
    B, N, H, D = 4, 65536, 32, 128  # needs 64 MiB of scratch
    assert s2.s2attn_bwd_workspace_size(B, N, H, D) > (32 << 20)
    fake = 1 << 20  # never dereferenced: rejected before any launch
    rc = L.s2attn_bwd_noalloc_v(*([fake] * 9), B, N, H, D, 8192, N, 0, None)
    assert rc == s2.S2_ERR_UNSUPPORTED
    assert "scratch" in s2.s2attn_last_error()
