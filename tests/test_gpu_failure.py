"""Failure detection and full overwrite of outputs (needs a B200).

* Every wait inside the kernels is bounded; a wait that runs out records a
  timeout in the library's status word and the kernel exits normally.  The
  probe entry point runs that path with a barrier nothing completes (no fault,
  no trap): the next status check reports S2_ERR_TIMEOUT and the context keeps
  working.
* Outputs are overwritten in full, padded rows included: outputs poisoned
  with NaN before a call hold no NaN after it.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from shifted_sparse_attention_b200 import binding as s2
from shifted_sparse_attention_b200 import synthetic

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_a_timeout_and_the_context_survives():
    s2.check_status()
    assert s2.s2attn_debug_wait_probe(2_000_000) == s2.S2_OK
    with pytest.raises(s2.S2AttnError) as e:
        s2.check_status()
    assert e.value.code == s2.S2_ERR_TIMEOUT and "0x200" in str(e.value)
    s2.check_status()  # the flag was cleared by the report
    x = synthetic.draw(1, 1024, 4, 128, seed=3)
    o, lse = s2.forward(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), 256)
    s2.check_status()
    assert torch.isfinite(o).all()
    assert s2.s2attn_debug_wait_probe(10) == s2.S2_ERR_INVALID_ARG  # budget below the floor


@pytest.mark.parametrize("variant,nv,stored", [(0, None, False), (0, 1900, True), (1, 1283, False), (2, 1700, True)])
def test_outputs_are_overwritten_everywhere(variant, nv, stored):
    B, N, H, D, G = 2, 2048, 4, 128, 512 if variant != 2 else 2048
    x = synthetic.draw(B, N, H, D, seed=17 + variant)
    dev = {n: t.cuda() for n, t in x.items()}
    nan = float("nan")
    o = torch.full_like(dev["q"], nan)
    lse = torch.full((B, H, N), nan, dtype=torch.float32, device="cuda")
    grads = tuple(torch.full_like(dev["q"], nan) for _ in range(3))
    s2.forward(dev["q"], dev["k"], dev["v"], G, variant, nv, out=o, lse=lse)
    s2.backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, G, variant, nv, grads=grads, stored_ds=stored)
    torch.cuda.synchronize()
    s2.check_status()
    assert not torch.isnan(o).any() and not torch.isnan(lse).any()
    for g in grads:
        assert not torch.isnan(g).any()
    if nv is not None:
        assert (o[:, nv:] == 0).all() and torch.isneginf(lse[:, :, nv:]).all()
        for g in grads:
            assert (g[:, nv:] == 0).all()


def test_outputs_are_overwritten_under_document_masks():
    B, N, H, D, G = 1, 2048, 4, 128, 512
    ids = np.zeros((B, N), dtype=np.int32)
    ids[0, 700:] = 1
    ids[0, 1500:] = 2
    x = synthetic.draw(B, N, H, D, seed=29)
    dev = {n: t.cuda() for n, t in x.items()}
    docs = s2.doc_bounds(torch.from_numpy(ids).cuda())
    nan = float("nan")
    o = torch.full_like(dev["q"], nan)
    lse = torch.full((B, H, N), nan, dtype=torch.float32, device="cuda")
    grads = tuple(torch.full_like(dev["q"], nan) for _ in range(3))
    s2.forward(dev["q"], dev["k"], dev["v"], G, 0, out=o, lse=lse, docs=docs)
    s2.backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, G, 0, grads=grads, docs=docs, stored_ds=True)
    torch.cuda.synchronize()
    s2.check_status()
    assert not torch.isnan(o).any() and not torch.isnan(lse).any()
    for g in grads:
        assert not torch.isnan(g).any()
