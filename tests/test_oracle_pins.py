"""Pins for the float64 oracle against what the pages and mathematics fix.

No test here touches the CUDA library.  Each pin is chosen so that a
plausible slip in the oracle (a wrong shift direction, the wrong half of the
heads, an off-by-one group boundary, a dropped term in a gradient, a transposed
operand) fails at least one of them; ``test_planted_mistakes_are_caught``
demonstrates that on mutated copies of the visibility predicate.
"""
from __future__ import annotations

import math
from pathlib import Path

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from oracle import segment_path
from shifted_sparse_attention_b200 import synthetic

GOLDEN = Path(__file__).resolve().parent / "golden"
STRICT, ROLLED, DENSE = oracle.STRICT, oracle.ROLLED, oracle.DENSE_CAUSAL


def _read_sets(name):
    out = {}
    for line in (GOLDEN / name).read_text().splitlines():
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        head, keys = line.split(":")
        case, q = head.split()
        out[(case, int(q))] = sorted(int(x) for x in keys.split())
    return out


CASES = {"c0": (STRICT, 0), "strict": (STRICT, 1), "rolled": (ROLLED, 1)}


def _visible_set(N, G, case, i, n_valid=None):
    variant, cls = CASES[case]
    A = oracle.adjacency(N, G, N if n_valid is None else n_valid, variant, cls)
    return sorted(np.nonzero(A[i])[0].tolist())


# --------------------------------------------------------------------------
# worked examples printed on the pages


def test_n8_g4_sets_match_worked_example():
    sets = _read_sets("n8_g4_visible_sets.txt")
    assert len(sets) == 24
    for (case, q), keys in sets.items():
        assert _visible_set(8, 4, case, q) == keys, (case, q)


def test_n8_g4_statements_verbatim():
    # the four statements the page makes directly
    assert _visible_set(8, 4, "c0", 4) == [4]
    assert _visible_set(8, 4, "strict", 4) == [2, 3, 4]
    # shifted middle group = [2,3,4,5]: row 5 sees exactly that group
    assert _visible_set(8, 4, "strict", 5) == [2, 3, 4, 5]
    # rolled last group [6,7,0,1]: original position 0 reads 6 and 7
    assert {6, 7} <= set(_visible_set(8, 4, "rolled", 0))
    assert _visible_set(8, 4, "rolled", 1) == [0, 1, 6, 7]
    # strict keeps short head / tail groups: no wrapped edge
    assert _visible_set(8, 4, "strict", 0) == [0]


def test_n16_g4_queries():
    for (case, q), keys in _read_sets("n16_g4_queries.txt").items():
        assert _visible_set(16, 4, case, q) == keys, (case, q)


def test_n8192_g2048_first_groups():
    lines = [l.split() for l in (GOLDEN / "n8192_g2048_first_groups.txt").read_text().splitlines()
             if l.strip() and not l.startswith("#")]
    N, G = 8192, 2048
    for case, b, e in lines:
        b, e = int(b), int(e)
        variant, cls = CASES[case]
        # the last row of the group sees the whole group and nothing before it
        last = e - 1
        assert oracle.visible(N, G, N, variant, cls, last, b)
        assert not oracle.visible(N, G, N, variant, cls, last, b - 1) if b > 0 else True
        # the first row of the group sees only itself
        assert oracle.visible(N, G, N, variant, cls, b, b)
        if b > 0:
            assert not oracle.visible(N, G, N, variant, cls, b, b - 1)
        # the next row starts a new group
        assert not oracle.visible(N, G, N, variant, cls, e, e - 1)


# --------------------------------------------------------------------------
# closed forms and invariants


def _closed_form_pairs(N, G, variant, cls):
    s, M = G // 2, N // G
    tri = lambda L: L * (L + 1) // 2
    if variant == DENSE:
        return tri(N)
    if cls == 0 or variant == ROLLED:
        return M * tri(G)
    return 2 * tri(s) + (M - 1) * tri(G)


@pytest.mark.parametrize("N,G", [(8, 4), (16, 4), (24, 8), (32, 32), (48, 12), (64, 16), (96, 8)])
def test_pair_counts_closed_form(N, G):
    for variant, cls in [(STRICT, 0), (STRICT, 1), (ROLLED, 0), (ROLLED, 1), (DENSE, 0), (DENSE, 1)]:
        assert oracle.pair_count(N, G, N, variant, cls) == _closed_form_pairs(N, G, variant, cls)


def test_pair_count_ratio_tends_to_g_over_n():
    # per head, group attention visits about N·G/2 pairs against N^2/2 for full causal
    G = 8
    for N in (64, 128, 256):
        full = oracle.pair_count(N, G, N, DENSE, 0)
        c0 = oracle.pair_count(N, G, N, STRICT, 0)
        assert abs(c0 / full - G / N) < 2.0 / N + 1e-12


def test_strict_is_causal_and_rolled_breaks_causality_by_s_squared():
    for N, G in [(8, 4), (16, 4), (32, 8), (64, 16)]:
        s = G // 2
        A_strict = oracle.adjacency(N, G, N, STRICT, 1)
        A_rolled = oracle.adjacency(N, G, N, ROLLED, 1)
        upper = np.triu(np.ones((N, N), dtype=bool), 1)
        assert not (A_strict & upper).any()
        viol = A_rolled & upper
        assert viol.sum() == s * s
        rows, cols = np.nonzero(viol)
        assert rows.max() < s and cols.min() >= N - s
        # apart from the wrap group the two variants agree
        assert (A_strict[s:N - s] == A_rolled[s:N - s]).all()


def test_union_graph_has_no_permanent_cut():
    # R_{l+1}(i) = union over j in N_0(i) ∪ N_1(i) of R_l(j)  (page §2.2 recursion), N=16, G=4
    N, G = 16, 4
    A0 = oracle.adjacency(N, G, N, STRICT, 0)
    A1 = oracle.adjacency(N, G, N, STRICT, 1)
    U = A0 | A1

    def reach(adj, layers):
        R = np.eye(N, dtype=bool)
        for _ in range(layers):
            R = (adj.astype(np.int64) @ R.astype(np.int64)) > 0
        return R

    # plain grouping never leaves the group; S² reaches the whole prefix
    assert reach(A0, 10)[N - 1].nonzero()[0].tolist() == [12, 13, 14, 15]
    R = reach(U, 10)
    assert R[N - 1].nonzero()[0].tolist() == list(range(N))
    # causality: no position ever receives information from the future
    assert not (R & np.triu(np.ones((N, N), dtype=bool), 1)).any()
    # one layer already crosses the original boundary at 12 through the shifted group [10, 14)
    assert reach(U, 1)[13].nonzero()[0].tolist() == [10, 11, 12, 13]
    assert reach(A0, 1)[13].nonzero()[0].tolist() == [12, 13]


def test_padding_semantics_in_predicate():
    N, G, nv = 16, 4, 11
    for variant in (STRICT, ROLLED, DENSE):
        for cls in (0, 1):
            A = oracle.adjacency(N, G, nv, variant, cls)
            assert not A[nv:].any() and not A[:, nv:].any()
            Afull = oracle.adjacency(N, G, N, variant, cls)
            assert (A[:nv, :nv] == Afull[:nv, :nv]).all()


# --------------------------------------------------------------------------
# numerics: library routines and the second route


def _f64(x):
    return x.to(torch.float64)


def _sdpa_causal(q, k, v):
    """torch's library causal attention on [B, L, h, D] float64."""
    o = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(1, 2), k.transpose(1, 2), v.transpose(1, 2), is_causal=True)
    return o.transpose(1, 2)


def test_class0_heads_equal_library_causal_attention_per_group():
    B, N, H, D, G = 2, 64, 4, 16, 16
    x = synthetic.draw(B, N, H, D, seed=3)
    res = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=STRICT)
    q, k, v, g = (_f64(x[n]).requires_grad_(True) for n in ("q", "k", "v", "dout"))
    outs = []
    for a in range(0, N, G):
        outs.append(_sdpa_causal(q[:, a:a + G, : H // 2], k[:, a:a + G, : H // 2], v[:, a:a + G, : H // 2]))
    o_ref = torch.cat(outs, dim=1)
    (o_ref * g[:, :, : H // 2]).sum().backward()
    np.testing.assert_allclose(res["o"][:, :, : H // 2], o_ref.detach().numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(res["dq"][:, :, : H // 2], q.grad[:, :, : H // 2].numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(res["dk"][:, :, : H // 2], k.grad[:, :, : H // 2].numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(res["dv"][:, :, : H // 2], v.grad[:, :, : H // 2].numpy(), rtol=0, atol=1e-12)


def test_dense_causal_equals_library_causal_attention_and_lse():
    B, N, H, D = 1, 40, 2, 8
    x = synthetic.draw(B, N, H, D, seed=5)
    res = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=N, variant=DENSE)
    q, k, v, g = (_f64(x[n]).requires_grad_(True) for n in ("q", "k", "v", "dout"))
    o_ref = _sdpa_causal(q, k, v)
    (o_ref * g).sum().backward()
    np.testing.assert_allclose(res["o"], o_ref.detach().numpy(), rtol=0, atol=1e-12)
    for name, t in (("dq", q), ("dk", k), ("dv", v)):
        np.testing.assert_allclose(res[name], t.grad.numpy(), rtol=0, atol=1e-12)
    # lse: natural log of the softmax denominator, scale 1/sqrt(D).  The library
    # side is scipy's logsumexp: torch's CPU float64 logsumexp was seen to return
    # values up to 1e-9 away from a direct evaluation, on some runs only.
    s = np.einsum("bihd,bjhd->bhij", _f64(x["q"]).numpy(), _f64(x["k"]).numpy()) / math.sqrt(D)
    s[:, :, ~np.tril(np.ones((N, N), dtype=bool))] = -np.inf
    np.testing.assert_allclose(res["lse"], scipy.special.logsumexp(s, axis=-1), rtol=0, atol=1e-12)


@pytest.mark.parametrize("variant", [STRICT, ROLLED])
@pytest.mark.parametrize("n_valid", [None, 1, 3, 4, 5, 7])
def test_mask_route_equals_segment_route(variant, n_valid):
    # lengths 1,3,4,5,7,8 with G=4 cover partial groups and boundaries (page §1.1)
    B, N, H, D, G = 1, 8, 4, 8, 4
    x = synthetic.draw(B, N, H, D, seed=11)
    res = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant, n_valid=n_valid)
    o, lse, dq, dk, dv = segment_path.forward_backward(
        _f64(x["q"]), _f64(x["k"]), _f64(x["v"]), _f64(x["dout"]), G=G, variant=variant, n_valid=n_valid)
    np.testing.assert_allclose(res["o"], o.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_array_equal(np.isinf(res["lse"]), np.isinf(lse.numpy()))
    fin = np.isfinite(res["lse"])
    np.testing.assert_allclose(res["lse"][fin], lse.numpy()[fin], rtol=0, atol=1e-12)
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        np.testing.assert_allclose(res[name], t.numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("variant", [STRICT, ROLLED, DENSE])
def test_mask_route_equals_segment_route_larger(variant):
    B, N, H, D, G = 2, 48, 4, 16, 12
    x = synthetic.draw(B, N, H, D, seed=12)
    res = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant, n_valid=41)
    o, lse, dq, dk, dv = segment_path.forward_backward(
        _f64(x["q"]), _f64(x["k"]), _f64(x["v"]), _f64(x["dout"]), G=G, variant=variant, n_valid=41)
    np.testing.assert_allclose(res["o"], o.numpy(), rtol=0, atol=1e-12)
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        np.testing.assert_allclose(res[name], t.numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("variant", [STRICT, ROLLED])
def test_gradients_match_central_finite_differences(variant):
    B, N, H, D, G = 1, 8, 2, 4, 4
    x = synthetic.draw(B, N, H, D, seed=21)
    res = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant)
    g = _f64(x["dout"]).numpy()
    base = {n: _f64(x[n]).numpy() for n in ("q", "k", "v")}

    # the oracle reads bf16 inputs; finite differences go through the second
    # route in float64 (already shown equal to the oracle's forward)
    def loss(arrs):
        o, _ = segment_path.forward(*(torch.from_numpy(arrs[n]) for n in ("q", "k", "v")), G=G, variant=variant)
        return float((o.numpy() * g).sum())

    eps = 1e-6
    rng = np.random.default_rng(0)
    for name in ("q", "k", "v"):
        for _ in range(12):
            idx = tuple(int(rng.integers(0, s)) for s in base[name].shape)
            plus = {n: a.copy() for n, a in base.items()}
            minus = {n: a.copy() for n, a in base.items()}
            plus[name][idx] += eps
            minus[name][idx] -= eps
            fd = (loss(plus) - loss(minus)) / (2 * eps)
            assert abs(fd - res["d" + name][idx]) < 1e-7, (name, idx, fd, res["d" + name][idx])


def test_softmax_invariants():
    B, N, H, D, G = 1, 32, 4, 8, 8
    x = synthetic.draw(B, N, H, D, seed=2)
    ones = torch.ones_like(x["v"])
    for variant in (STRICT, ROLLED, DENSE):
        res = oracle.attention(x["q"], x["k"], ones, G=G, variant=variant, n_valid=29)
        assert np.allclose(res["o"][:, :29], 1.0, atol=1e-13, rtol=0)
        assert (res["o"][:, 29:] == 0).all() and np.isneginf(res["lse"][:, :, 29:]).all()
        # Q = 0: every visible key has weight 1/|S_i|, lse = ln |S_i|
        zero = torch.zeros_like(x["q"])
        res0 = oracle.attention(zero, x["k"], x["v"], G=G, variant=variant)
        for h in range(H):
            cls = 1 if h >= H // 2 else 0
            A = oracle.adjacency(N, G, N, variant, cls)
            np.testing.assert_allclose(res0["lse"][0, h], np.log(A.sum(1)), atol=1e-13, rtol=0)
            vbar = (A.astype(np.float64) @ _f64(x["v"])[0, :, h].numpy()) / A.sum(1)[:, None]
            np.testing.assert_allclose(res0["o"][0, :, h], vbar, atol=1e-12, rtol=0)


def test_padding_values_have_no_effect():
    B, N, H, D, G, nv = 1, 32, 4, 8, 8, 27
    x = synthetic.draw(B, N, H, D, seed=4)
    y = {n: t.clone() for n, t in x.items()}
    noise = synthetic.draw(B, N, H, D, seed=99)
    for n in y:
        y[n][:, nv:] = noise[n][:, nv:] * 7
    for variant in (STRICT, ROLLED, DENSE):
        a = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant, n_valid=nv)
        b = oracle.attention(y["q"], y["k"], y["v"], y["dout"], G=G, variant=variant, n_valid=nv)
        for name in ("o", "lse", "dq", "dk", "dv"):
            np.testing.assert_array_equal(a[name], b[name])
        assert (a["dk"][:, nv:] == 0).all() and (a["dv"][:, nv:] == 0).all() and (a["dq"][:, nv:] == 0).all()


def test_row_window_and_head_subset_compose_to_full_result():
    B, N, H, D, G = 2, 32, 4, 8, 8
    x = synthetic.draw(B, N, H, D, seed=6)
    full = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=ROLLED)
    heads = [1, 6]
    parts = [oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=ROLLED, rows=r, heads=heads)
             for r in ((0, 13), (13, N))]
    for bh in heads:
        b, h = divmod(bh, H)
        for name in ("o", "dq"):
            got = np.where(np.isnan(parts[0][name]), parts[1][name], parts[0][name])
            np.testing.assert_allclose(got[b, :, h], full[name][b, :, h], atol=1e-13, rtol=0)
        for name in ("dk", "dv"):
            np.testing.assert_allclose(parts[0][name][b, :, h] + parts[1][name][b, :, h],
                                       full[name][b, :, h], atol=1e-13, rtol=0)


@pytest.mark.parametrize("variant", [STRICT, ROLLED, DENSE])
def test_window_entry_equals_full_oracle(variant):
    # the windowed entry (used for full-size samples) against the pinned full routine
    B, N, H, D, G, nv = 2, 48, 4, 8, 12, 43
    x = synthetic.draw(B, N, H, D, seed=31)
    full = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant, n_valid=nv)
    heads = [0, 3, 5, 6]
    for r0, r1 in ((0, 48), (18, 24), (36, 48)):
        w = oracle.attention_window(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant, rows=(r0, r1),
                                    heads=heads, n_valid=nv)
        part = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant, n_valid=nv,
                                rows=(r0, r1), heads=heads)
        for t, bh in enumerate(heads):
            b, h = divmod(bh, H)
            np.testing.assert_array_equal(w["o"][t], full["o"][b, r0:r1, h])
            np.testing.assert_array_equal(w["lse"][t], full["lse"][b, h, r0:r1])
            np.testing.assert_array_equal(w["dq"][t], full["dq"][b, r0:r1, h])
            # dk, dv: the window's rows' contributions to the window's keys
            np.testing.assert_allclose(w["dk"][t], part["dk"][b, r0:r1, h], rtol=0, atol=1e-15)
            np.testing.assert_allclose(w["dv"][t], part["dv"][b, r0:r1, h], rtol=0, atol=1e-15)


# --------------------------------------------------------------------------
# power of the pins: plausible mistakes in the predicate must be rejected


def _mutants():
    def floor_div(a, b):
        return a // b

    # (a right shift by G/2 is not a mistake: it yields the same partition as a left one)
    def quarter_shift(N, G, i, j):  # shift by G/4 instead of G/2
        s = G // 4
        return j <= i and floor_div(i - s, G) == floor_div(j - s, G)

    def off_by_one(N, G, i, j):  # boundary one position late
        s = G // 2 + 1
        return j <= i and floor_div(i - s, G) == floor_div(j - s, G)

    def wrap_teaching(N, G, i, j):  # floor(((i+s) mod N)/G) equality with original causality
        s = G // 2
        return j <= i and ((i + s) % N) // G == ((j + s) % N) // G

    def no_causal(N, G, i, j):
        s = G // 2
        return floor_div(i - s, G) == floor_div(j - s, G)

    return {"quarter_shift": quarter_shift, "off_by_one": off_by_one,
            "wrap_teaching": wrap_teaching, "no_causal": no_causal}


def _pins_pass(pred):
    """Re-run the worked-example pins for the shifted heads on a predicate."""
    ok = True
    for (case, q), keys in _read_sets("n8_g4_visible_sets.txt").items():
        if case == "strict":
            ok &= sorted(j for j in range(8) if pred(8, 4, q, j)) == keys
    for (case, q), keys in _read_sets("n16_g4_queries.txt").items():
        if case == "strict":
            ok &= sorted(j for j in range(16) if pred(16, 4, q, j)) == keys
    return ok


def test_planted_mistakes_are_caught():
    for name, pred in _mutants().items():
        assert not _pins_pass(pred), name
    # and the real predicate passes the same check
    assert _pins_pass(lambda N, G, i, j: oracle.visible(N, G, N, STRICT, 1, i, j))


# --------------------------------------------------------------------------
# segment identities of the gradients (used by the full-size GPU checks)


@pytest.mark.parametrize("variant,n_valid", [(STRICT, None), (ROLLED, None), (DENSE, None), (STRICT, 45),
                                             (ROLLED, 51), (DENSE, 37)])
def test_gradient_segment_identities(variant, n_valid):
    """Each softmax row sums to one, so dV summed over a segment's keys equals dO
    summed over its valid queries; sum_j dS_ij = g_i·o_i - Delta_i = 0, so dK sums to
    zero over a segment ([PT] §3's gradient).  A dropped Delta term or a
    mis-normalised softmax breaks one of them.  The segment layout the GPU tests use
    (tests/seg_layout.py) is checked here against the oracle's own matrices: every
    row of a segment sees only keys of that segment, and its last row sees all of
    them."""
    from tests.seg_layout import segments

    B, N, H, D, G = 1, 64, 4, 8, 16
    nv = N if n_valid is None else n_valid
    x = synthetic.draw(B, N, H, D, seed=12)
    res = oracle.attention(x["q"], x["k"], x["v"], x["dout"], G=G, variant=variant, n_valid=nv)
    g = _f64(x["dout"])[0].numpy().copy()
    g[nv:] = 0
    for h in range(H):
        cls = 0 if variant == DENSE else int(h >= H // 2)
        A = oracle.adjacency(N, G, nv, variant, cls)
        segs = segments(N, G, variant, cls)
        covered = np.zeros(N, dtype=int)
        for seg in segs:
            rows = np.concatenate([np.arange(a, b) for a, b in seg])
            covered[rows] += 1
            outside = np.ones(N, dtype=bool)
            outside[rows] = False
            assert not A[np.ix_(rows, np.nonzero(outside)[0])].any(), (h, seg)
            last = rows[rows < nv][-1] if (rows < nv).any() else None
            if last is not None:
                assert A[last, rows[rows < nv]].all(), (h, seg)
            np.testing.assert_allclose(res["dv"][0, rows, h].sum(0), g[rows, h].sum(0), atol=1e-11, rtol=0)
            np.testing.assert_allclose(res["dk"][0, rows, h].sum(0), 0.0, atol=1e-11, rtol=0)
        assert (covered == 1).all()
