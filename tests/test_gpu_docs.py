"""Packed sequences with a document mask on the GPU (needs a B200).

"4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §1.1: documents packed into one
sequence get a document mask applied identically to the original and the
shifted grouping.  Checked here: the document-bounds kernel, parity of the
forward and both backward passes with the float64 oracle under document
masks, and the section's leak test (changing one document leaves the
others' outputs and gradients bit-identical).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from shifted_sparse_attention_b200 import binding as s2
from shifted_sparse_attention_b200 import synthetic
from tests.tolerance import check_grad, check_lse, check_o, to_np

pytestmark = pytest.mark.gpu

STRICT, ROLLED, DENSE = 0, 1, 2


def _ids(N, cuts, B=1):
    ids = np.zeros((B, N), dtype=np.int32)
    c = sorted(set(x for x in cuts if 0 < x < N)) + [N]
    for d, (a, b) in enumerate(zip([0] + c[:-1], c)):
        ids[:, a:b] = d
    return ids


def _bounds_ref(ids):
    B, N = ids.shape
    out = np.zeros((B, N, 2), dtype=np.int32)
    for b in range(B):
        start = 0
        for x in range(1, N + 1):
            if x == N or ids[b, x] != ids[b, x - 1]:
                out[b, start:x] = (start, x)
                start = x
    return out


@pytest.mark.parametrize("B,N", [(1, 7), (2, 1000), (1, 1024), (3, 5000), (1, 106496)])
def test_doc_bounds_kernel(B, N):
    rng = np.random.default_rng(N + B)
    ids = np.cumsum(rng.random((B, N)) < 0.01, axis=1).astype(np.int32)
    ids[:, N // 2:] += 5  # a run boundary that the cumulative sum might not place
    got = s2.doc_bounds(torch.from_numpy(ids).cuda()).cpu().numpy()
    np.testing.assert_array_equal(got, _bounds_ref(ids))


def _run(x, G, variant, nv, ids):
    dev = {n: t.cuda() for n, t in x.items()}
    docs = s2.doc_bounds(torch.from_numpy(ids).cuda())
    o, lse = s2.forward(dev["q"], dev["k"], dev["v"], G, variant, nv, docs=docs)
    dq, dk, dv = s2.backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, G, variant, nv, docs=docs)
    s2.check_status()
    return o.cpu(), lse.cpu(), dq.cpu(), dk.cpu(), dv.cpu()


CASES = [
    # (B, N, H, D, G, variant, n_valid, cuts)
    (1, 2048, 4, 128, 512, STRICT, None, [5, 512, 768, 1030, 1031, 1800]),
    (1, 2048, 4, 128, 512, ROLLED, None, [256, 300, 1792, 1900]),
    (2, 2048, 4, 128, 512, STRICT, 1900, list(range(97, 2048, 97))),
    (1, 2048, 2, 128, 2048, DENSE, None, [100, 129, 1000]),
    (1, 1024, 8, 64, 256, STRICT, None, [128, 200, 640]),
    (1, 4096, 2, 128, 1024, ROLLED, 3000, [700, 2600, 2999, 3500]),
]


@pytest.mark.parametrize("B,N,H,D,G,variant,nv,cuts", CASES)
def test_document_mask_matches_oracle(B, N, H, D, G, variant, nv, cuts):
    x = synthetic.draw(B, N, H, D, seed=600 + N + variant)
    ids = _ids(N, cuts, B)
    o, lse, dq, dk, dv = _run(x, G, variant, nv, ids)
    ref = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant, n_valid=nv, doc=ids)
    where = str((B, N, H, D, G, variant, nv))
    check_o(o, ref["o"], where)
    n = N if nv is None else nv
    check_lse(lse, ref["lse"], where)
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        check_grad(name, to_np(g)[:, :n], ref[name][:, :n], where)


@pytest.mark.parametrize("variant", [STRICT, ROLLED])
def test_leak_test_on_the_gpu(variant):
    # boundaries inside a group (300), on an original group boundary (1024) and on a
    # shifted one (1280): changing a document leaves the others bit-identical
    B, N, H, D, G = 1, 2048, 4, 128, 512
    cuts = [300, 1024, 1280]
    ids = _ids(N, cuts)
    x = synthetic.draw(B, N, H, D, seed=77)
    ref = _run(x, G, variant, None, ids)
    for a, b in ((0, 300), (300, 1024), (1024, 1280)):
        y = {n: t.clone() for n, t in x.items()}
        for n in ("q", "k", "v", "dout"):
            y[n][:, a:b] = (torch.randn_like(y[n][:, a:b].float()) * 3).to(torch.bfloat16)
        got = _run(y, G, variant, None, ids)
        keep = np.ones(N, dtype=bool)  # every other document, including the rolled wrap group's partner
        keep[a:b] = False
        for t_ref, t_got in zip(ref, got):
            if t_ref.dim() == 3:  # lse [B, H, N]
                assert torch.equal(t_ref[:, :, keep], t_got[:, :, keep])
            else:
                assert torch.equal(t_ref[:, keep], t_got[:, keep])
