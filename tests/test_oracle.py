"""Pins of the fp64 oracle against facts fixed outside itself.

* a hand-computed worked example (tests/golden/worked_example.json);
* textbook special case: with no branches the method is per-document causal
  attention, checked against torch's scaled_dot_product_attention in fp64;
* brute force over the explicit mask versus the row-set form, the decomposed
  form (main part + branch part + Eq. 2 merge) and the ring form (zigzag
  chunks over R CPU ranks) on tiny random packings;
* closed forms (K = 0 gives LSE = log of the visible-key count, V = c gives
  O = c, a document's first row sees only itself);
* merge algebra (associativity, commutativity, empty partial);
* backward: autograd in fp64 and central finite differences against the closed
  form, and the invariants sum_j dV_j = sum_i dO_i and sum_j dK_j = 0 per KV group.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as orc
import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _val(x):
    if isinstance(x, (int, float)):
        return float(x)
    x = x.strip()
    if x.startswith("ln "):
        return math.log(float(x[3:]))
    if x == "-(2/3) ln 2 + 2 ln 3":
        return -(2.0 / 3.0) * math.log(2.0) + 2.0 * math.log(3.0)
    if "/" in x:
        a, b = x.split("/")
        return float(a) / float(b)
    return float(x)


def _golden_inputs():
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    inp = g["inputs"]
    f = lambda key, shape: np.array([_val(t) for t in inp[key]], dtype=np.float64).reshape(shape)
    q = f("q", (3, 1, 1))
    k = f("k", (3, 1, 1))
    v = f("v", (3, 1, 1))
    qb = f("qb", (1, 2, 1, 1))
    kb = f("kb", (1, 2, 1, 1))
    vb = f("vb", (1, 2, 1, 1))
    cu = np.array(inp["cu_seqlens"])
    anc = np.array(inp["anchors"])
    return g, (q, k, v, qb, kb, vb, cu, anc)


@pytest.mark.parametrize("mode,key", [(orc.CHAIN, "expected_chain"), (orc.BLOCK, "expected_block")])
@pytest.mark.parametrize("form", ["brute", "rows", "decomposed", "ring1", "ring2"])
def test_golden_worked_example_forward(mode, key, form):
    g, (q, k, v, qb, kb, vb, cu, anc) = _golden_inputs()
    exp = g[key]
    if form == "brute":
        om, ob, lse = orc.forward_brute(q, k, v, qb, kb, vb, cu, anc, 2, mode, scale=1.0)
    elif form == "decomposed":
        om, ob, lse = orc.forward_decomposed(q, k, v, qb, kb, vb, cu, anc, 2, mode, scale=1.0)
    elif form.startswith("ring"):
        om, ob, lse = orc.forward_ring(q, k, v, qb, kb, vb, cu, anc, 2, mode, R=int(form[-1]), scale=1.0)
    else:
        rows, O, lse = orc.forward_rows(q, k, v, qb, kb, vb, cu, anc, 2, mode, scale=1.0)
        om, ob = O[:3], O[3:].reshape(1, 2, 1, 1)
    np.testing.assert_allclose(om.reshape(-1), [_val(x) for x in exp["o_main"]], rtol=0, atol=1e-12)
    np.testing.assert_allclose(ob.reshape(-1), [_val(x) for x in exp["o_branch"]], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse.reshape(-1), [_val(x) for x in exp["lse"]], rtol=0, atol=1e-12)


@pytest.mark.parametrize("form", ["brute", "rows"])
def test_golden_worked_example_backward(form):
    g, (q, k, v, qb, kb, vb, cu, anc) = _golden_inputs()
    exp = g["expected_backward_chain_do_main2"]
    do = np.zeros((3, 1, 1))
    do[2] = 1.0
    dob = np.zeros((1, 2, 1, 1))
    if form == "brute":
        dq, dk, dv, dqb, dkb, dvb = orc.backward_brute(q, k, v, qb, kb, vb, do, dob, cu, anc, 2, orc.CHAIN, scale=1.0)
    else:
        rows, dQ, dk, dv, dkb, dvb = orc.backward_rows(q, k, v, qb, kb, vb, do, dob, cu, anc, 2, orc.CHAIN, scale=1.0)
        dq, dqb = dQ[:3], dQ[3:]
    chk = lambda a, key: np.testing.assert_allclose(np.asarray(a).reshape(-1), [_val(x) for x in exp[key]], rtol=0, atol=1e-12)
    chk(dv, "dv_main")
    chk(dk, "dk_main")
    chk(dq, "dq_main")
    chk(dqb, "dq_branch")
    chk(dkb, "dk_branch")
    chk(dvb, "dv_branch")


# ---------------------------------------------------------------------------
# random tiny problems
# ---------------------------------------------------------------------------

def _tiny(seed, S, ndoc, nanc, B, mode, Hq, Hkv, d, dtype=np.float64):
    g = torch.Generator()
    g.manual_seed(seed)
    lengths, anchors = wl.random_packing(S, ndoc, nanc, g)
    rs = np.random.default_rng(seed)
    Nb = len(anchors)
    q = rs.standard_normal((S, Hq, d))
    k = rs.standard_normal((S, Hkv, d))
    v = rs.standard_normal((S, Hkv, d))
    qb = rs.standard_normal((Nb, B, Hq, d))
    kb = rs.standard_normal((Nb, B, Hkv, d))
    vb = rs.standard_normal((Nb, B, Hkv, d))
    cu = np.concatenate([[0], np.cumsum(lengths)])
    return q, k, v, qb, kb, vb, cu, np.array(anchors, dtype=np.int64)


TINY_CASES = [
    # seed, S, ndoc, nanc, B, mode, Hq, Hkv, d
    (1, 17, 1, 5, 4, orc.CHAIN, 2, 1, 8),
    (2, 33, 3, 7, 3, orc.CHAIN, 4, 2, 8),
    (3, 40, 4, 6, 4, orc.BLOCK, 2, 2, 8),
    (4, 64, 5, 12, 2, orc.BLOCK, 4, 1, 8),
    (5, 29, 2, 0, 3, orc.CHAIN, 2, 1, 8),
    (6, 48, 6, 48, 3, orc.CHAIN, 2, 1, 8),   # anchor at every position
    (7, 24, 1, 4, 1, orc.CHAIN, 1, 1, 64),
    (8, 50, 2, 9, 5, orc.BLOCK, 3, 3, 64),
]


@pytest.mark.parametrize("case", TINY_CASES)
def test_forms_agree_tiny(case):
    seed, S, ndoc, nanc, B, mode, Hq, Hkv, d = case
    q, k, v, qb, kb, vb, cu, anc = _tiny(seed, S, ndoc, nanc, B, mode, Hq, Hkv, d)
    om, ob, L = orc.forward_brute(q, k, v, qb, kb, vb, cu, anc, B, mode)
    rows, O2, L2 = orc.forward_rows(q, k, v, qb, kb, vb, cu, anc, B, mode, block=7)
    np.testing.assert_allclose(O2[:S], om, atol=1e-12, rtol=0)
    np.testing.assert_allclose(O2[S:], ob.reshape(-1, Hq, d), atol=1e-12, rtol=0)
    np.testing.assert_allclose(L2, L, atol=1e-12, rtol=0)
    om3, ob3, L3 = orc.forward_decomposed(q, k, v, qb, kb, vb, cu, anc, B, mode)
    np.testing.assert_allclose(om3, om, atol=1e-12, rtol=0)
    np.testing.assert_allclose(ob3, ob, atol=1e-12, rtol=0)
    np.testing.assert_allclose(L3, L, atol=1e-12, rtol=0)
    for R in (1, 2, 3, 4):
        om4, ob4, L4 = orc.forward_ring(q, k, v, qb, kb, vb, cu, anc, B, mode, R=R)
        np.testing.assert_allclose(om4, om, atol=1e-12, rtol=0)
        np.testing.assert_allclose(ob4, ob, atol=1e-12, rtol=0)
        np.testing.assert_allclose(L4, L, atol=1e-12, rtol=0)


@pytest.mark.parametrize("R", [1, 2, 4, 8])
def test_ring_step_order_invariance(R):
    q, k, v, qb, kb, vb, cu, anc = _tiny(11, 64, 3, 10, 3, orc.CHAIN, 2, 1, 8)
    ref = orc.forward_brute(q, k, v, qb, kb, vb, cu, anc, 3, orc.CHAIN)
    rs = np.random.default_rng(R)
    for _ in range(3):
        order = rs.permutation(R)
        out = orc.forward_ring(q, k, v, qb, kb, vb, cu, anc, 3, orc.CHAIN, R=R, step_order=order)
        for a, b in zip(out, ref):
            np.testing.assert_allclose(a, b, atol=1e-12, rtol=0)


def test_zigzag_chunks_partition_and_balance():
    cu = np.array([0, 5, 5 + 37, 5 + 37 + 64])
    for R in (1, 2, 3, 4, 8):
        ch = orc.zigzag_chunks(cu, R)
        assert len(ch) == 3 * 2 * R
        for di in range(3):
            cs = [c for c in ch if c[0] == di]
            # contiguous, ordered, covering [s, e)
            assert cs[0][2] == cu[di] and cs[-1][3] == cu[di + 1]
            for a, b in zip(cs, cs[1:]):
                assert a[3] == b[2]
            owners = [c[4] for c in cs]
            for r in range(R):
                assert owners.count(r) == 2
                # rank r owns chunk r and 2R-1-r
                assert owners[r] == r and owners[2 * R - 1 - r] == r


# ---------------------------------------------------------------------------
# textbook special case: no branches -> per-document causal attention (SDPA)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("Hq,Hkv,d", [(2, 2, 8), (4, 2, 16), (4, 1, 64)])
def test_no_branches_is_per_document_causal_sdpa(Hq, Hkv, d):
    g = torch.Generator()
    g.manual_seed(Hq * 100 + d)
    lengths, _ = wl.random_packing(70, 4, 0, g)
    cu = np.concatenate([[0], np.cumsum(lengths)])
    rs = np.random.default_rng(d)
    S = int(cu[-1])
    q = rs.standard_normal((S, Hq, d))
    k = rs.standard_normal((S, Hkv, d))
    v = rs.standard_normal((S, Hkv, d))
    empty = np.zeros((0, 2, Hq, d)), np.zeros((0, 2, Hkv, d)), np.zeros((0, 2, Hkv, d))
    rows, O, L = orc.forward_rows(q, k, v, *empty, cu, np.zeros(0, dtype=np.int64), 2, orc.CHAIN)
    G = Hq // Hkv
    for di in range(len(lengths)):
        s, e = int(cu[di]), int(cu[di + 1])
        tq = torch.from_numpy(q[s:e]).permute(1, 0, 2)  # [H, L, d]
        tk = torch.from_numpy(k[s:e]).permute(1, 0, 2).repeat_interleave(G, dim=0)
        tv = torch.from_numpy(v[s:e]).permute(1, 0, 2).repeat_interleave(G, dim=0)
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
        np.testing.assert_allclose(O[s:e], ref.permute(1, 0, 2).numpy(), atol=1e-12, rtol=0)
        # LSE from the library's own logsumexp over the causal scores
        sc = torch.einsum("hid,hjd->hij", tq, tk) / math.sqrt(d)
        causal = torch.ones(e - s, e - s, dtype=torch.bool).tril()
        lse_ref = torch.logsumexp(sc.masked_fill(~causal, float("-inf")), dim=-1)
        np.testing.assert_allclose(L[:, s:e], lse_ref.numpy(), atol=1e-12, rtol=0)


def test_branch_row_equals_sdpa_with_explicit_key_list():
    """A branch row is ordinary attention over (prefix keys ++ own branch keys):
    compare with SDPA applied to that explicitly assembled key list."""
    q, k, v, qb, kb, vb, cu, anc = _tiny(21, 40, 2, 6, 4, orc.CHAIN, 2, 2, 16)
    rows, O, L = orc.forward_rows(q, k, v, qb, kb, vb, cu, anc, 4, orc.CHAIN)
    S = 40
    for b, a in enumerate(anc):
        di = np.searchsorted(cu, a, side="right") - 1
        s = int(cu[di])
        for t in range(4):
            for h in range(2):
                keys = np.concatenate([k[s:a + 1, h], kb[b, :t + 1, h]])
                vals = np.concatenate([v[s:a + 1, h], vb[b, :t + 1, h]])
                ref = torch.nn.functional.scaled_dot_product_attention(
                    torch.from_numpy(qb[b, t, h])[None, None], torch.from_numpy(keys)[None],
                    torch.from_numpy(vals)[None])
                np.testing.assert_allclose(O[S + b * 4 + t, h], ref[0, 0].numpy(), atol=1e-12, rtol=0)


# ---------------------------------------------------------------------------
# closed forms
# ---------------------------------------------------------------------------

def _visible_count(cu, anc, B, mode, S):
    """Number of visible keys per concatenated row, from the counting rule:
    main row i: i - s(i) + 1; branch row (b,t): a_b - s(a_b) + 1 plus t+1
    (chain) or B (block)."""
    out = []
    starts = {}
    for di in range(len(cu) - 1):
        for p in range(cu[di], cu[di + 1]):
            starts[p] = cu[di]
    for i in range(S):
        out.append(i - starts[i] + 1)
    for a in anc:
        for t in range(B):
            out.append(a - starts[a] + 1 + (t + 1 if mode == orc.CHAIN else B))
    return np.array(out, dtype=np.float64)


@pytest.mark.parametrize("mode", [orc.CHAIN, orc.BLOCK])
@pytest.mark.parametrize("form", ["brute", "rows", "decomposed", "ring"])
def test_closed_form_zero_keys(mode, form):
    q, k, v, qb, kb, vb, cu, anc = _tiny(31, 45, 3, 8, 3, mode, 2, 1, 8)
    k = np.zeros_like(k)
    kb = np.zeros_like(kb)
    S = 45
    if form == "brute":
        om, ob, L = orc.forward_brute(q, k, v, qb, kb, vb, cu, anc, 3, mode)
    elif form == "decomposed":
        om, ob, L = orc.forward_decomposed(q, k, v, qb, kb, vb, cu, anc, 3, mode)
    elif form == "ring":
        om, ob, L = orc.forward_ring(q, k, v, qb, kb, vb, cu, anc, 3, mode, R=3)
    else:
        _, O, L = orc.forward_rows(q, k, v, qb, kb, vb, cu, anc, 3, mode)
        om, ob = O[:S], O[S:].reshape(-1, 3, 2, 8)
    cnt = _visible_count(list(cu), list(anc), 3, mode, S)
    for h in range(2):
        np.testing.assert_allclose(L[h], np.log(cnt), atol=1e-12, rtol=0)
    # with K = 0 every visible key weighs the same: O = mean of visible values
    om0 = np.zeros_like(om)
    starts = np.repeat(cu[:-1], np.diff(cu))
    for i in range(S):
        om0[i] = v[starts[i]:i + 1, 0].mean(axis=0)  # Hkv = 1: both q heads read KV head 0
    np.testing.assert_allclose(om, om0, atol=1e-12, rtol=0)
    for b, a in enumerate(anc):
        s = starts[a]
        for t in range(3):
            nb = t + 1 if mode == orc.CHAIN else 3
            tot = v[s:a + 1, 0].sum(axis=0) + vb[b, :nb, 0].sum(axis=0)
            for h in range(2):
                np.testing.assert_allclose(ob[b, t, h], tot / (a - s + 1 + nb), atol=1e-12, rtol=0)


def test_closed_form_constant_values_and_first_row():
    q, k, v, qb, kb, vb, cu, anc = _tiny(41, 30, 1, 5, 4, orc.CHAIN, 2, 2, 8)
    c = np.linspace(-1, 1, 8)
    v[:] = c
    vb[:] = c
    om, ob, L = orc.forward_brute(q, k, v, qb, kb, vb, cu, anc, 4, orc.CHAIN)
    np.testing.assert_allclose(om, np.broadcast_to(c, om.shape), atol=1e-12)
    np.testing.assert_allclose(ob, np.broadcast_to(c, ob.shape), atol=1e-12)
    sc = 1.0 / math.sqrt(8)
    for h in range(2):
        np.testing.assert_allclose(L[h, 0], sc * q[0, h] @ k[0, h], atol=1e-12)


def test_visible_pair_count_matches_mask():
    for case in TINY_CASES:
        seed, S, ndoc, nanc, B, mode, Hq, Hkv, d = case
        _, _, _, _, _, _, cu, anc = _tiny(seed, S, ndoc, nanc, B, mode, 1, 1, 1)
        M = orc.visible_mask(cu, anc, B, mode)
        assert orc.visible_pair_count(cu, anc, B, mode) == int(M.sum())
        assert int(M.sum()) == int(_visible_count(list(cu), list(anc), B, mode, S).sum())


# ---------------------------------------------------------------------------
# merge algebra (Eq. 2)
# ---------------------------------------------------------------------------

def test_merge_partition_any_order_any_tree():
    rs = np.random.default_rng(5)
    n, d, m = 6, 8, 40
    Q = rs.standard_normal((n, d))
    K = rs.standard_normal((m, d))
    V = rs.standard_normal((m, d))
    full_O, full_L = orc.attend(Q, K, V, np.ones((n, m), dtype=bool), 0.3)
    for parts in range(2, 9):
        lab = rs.integers(0, parts, size=m)
        P = []
        for p in range(parts):
            sel = lab == p
            P.append(orc.attend(Q, K[sel], V[sel], np.ones((n, sel.sum()), dtype=bool), 0.3))
        order = list(rs.permutation(parts))
        # random binary tree: repeatedly merge two random live partials
        live = [P[i] for i in order]
        while len(live) > 1:
            i, j = sorted(rs.choice(len(live), 2, replace=False))
            a, b = live[i], live[j]
            mo, ml = orc.lse_merge([a[0], b[0]], [a[1], b[1]])
            live = [x for t, x in enumerate(live) if t not in (i, j)] + [(mo, ml)]
        np.testing.assert_allclose(live[0][0], full_O, atol=1e-12)
        np.testing.assert_allclose(live[0][1], full_L, atol=1e-12)
        # flat k-way merge
        mo, ml = orc.lse_merge([x[0] for x in P], [x[1] for x in P])
        np.testing.assert_allclose(mo, full_O, atol=1e-12)
        np.testing.assert_allclose(ml, full_L, atol=1e-12)


def test_merge_empty_partial_is_identity():
    rs = np.random.default_rng(6)
    O = rs.standard_normal((5, 4))
    L = rs.standard_normal(5)
    eO, eL = np.zeros((5, 4)), np.full(5, -np.inf)
    for parts in ([O, eO], [eO, O]):
        ls = [L, eL] if parts[0] is O else [eL, L]
        mo, ml = orc.lse_merge(parts, ls)
        np.testing.assert_allclose(mo, O, atol=0)
        np.testing.assert_allclose(ml, L, atol=0)
    mo, ml = orc.lse_merge([eO, eO], [eL, eL])
    assert np.all(mo == 0) and np.all(np.isneginf(ml))


# ---------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------

def _torch_branch_attention(Q, K, V, M, G, sc):
    """Independent autograd formulation: masked softmax via torch ops."""
    outs = []
    for h in range(Q.shape[1]):
        s = sc * Q[:, h] @ K[:, h // G].T
        s = s.masked_fill(~M, float("-inf"))
        outs.append(torch.softmax(s, dim=-1) @ V[:, h // G])
    return torch.stack(outs, dim=1)


@pytest.mark.parametrize("case", TINY_CASES[:6])
def test_backward_closed_form_matches_autograd(case):
    seed, S, ndoc, nanc, B, mode, Hq, Hkv, d = case
    q, k, v, qb, kb, vb, cu, anc = _tiny(seed, S, ndoc, nanc, B, mode, Hq, Hkv, d)
    rs = np.random.default_rng(seed + 99)
    do = rs.standard_normal(q.shape)
    dob = rs.standard_normal(qb.shape)
    ref = orc.backward_brute(q, k, v, qb, kb, vb, do, dob, cu, anc, B, mode)
    rows_out = orc.backward_rows(q, k, v, qb, kb, vb, do, dob, cu, anc, B, mode, block=5)
    Nb = len(anc)
    cat = lambda a, b, H: torch.from_numpy(np.concatenate([a, b.reshape(-1, H, d)])).requires_grad_(True)
    Q, K, V = cat(q, qb, Hq), cat(k, kb, Hkv), cat(v, vb, Hkv)
    M = torch.from_numpy(orc.visible_mask(cu, anc, B, mode))
    O = _torch_branch_attention(Q, K, V, M, Hq // Hkv, 1.0 / math.sqrt(d))
    dO = torch.from_numpy(np.concatenate([do, dob.reshape(-1, Hq, d)]))
    (O * dO).sum().backward()
    gq, gk, gv = Q.grad.numpy(), K.grad.numpy(), V.grad.numpy()
    np.testing.assert_allclose(ref[0], gq[:S], atol=1e-10)
    np.testing.assert_allclose(ref[3].reshape(-1, Hq, d), gq[S:], atol=1e-10)
    np.testing.assert_allclose(ref[1], gk[:S], atol=1e-10)
    np.testing.assert_allclose(ref[4].reshape(-1, Hkv, d), gk[S:], atol=1e-10)
    np.testing.assert_allclose(ref[2], gv[:S], atol=1e-10)
    np.testing.assert_allclose(ref[5].reshape(-1, Hkv, d), gv[S:], atol=1e-10)
    # row-set form, full rows, equals the brute form
    _, dQ, dk, dv, dkb, dvb = rows_out
    np.testing.assert_allclose(dQ[:S], ref[0], atol=1e-12)
    np.testing.assert_allclose(dQ[S:], ref[3].reshape(-1, Hq, d), atol=1e-12)
    np.testing.assert_allclose(dk, ref[1], atol=1e-12)
    np.testing.assert_allclose(dv, ref[2], atol=1e-12)
    np.testing.assert_allclose(dkb, ref[4], atol=1e-12)
    np.testing.assert_allclose(dvb, ref[5], atol=1e-12)


def test_backward_finite_differences():
    q, k, v, qb, kb, vb, cu, anc = _tiny(51, 20, 2, 4, 3, orc.CHAIN, 2, 1, 4)
    rs = np.random.default_rng(52)
    do = rs.standard_normal(q.shape)
    dob = rs.standard_normal(qb.shape)
    grads = orc.backward_brute(q, k, v, qb, kb, vb, do, dob, cu, anc, 3, orc.CHAIN)

    def f(q_, k_, v_, qb_, kb_, vb_):
        om, ob, _ = orc.forward_brute(q_, k_, v_, qb_, kb_, vb_, cu, anc, 3, orc.CHAIN)
        return float((om * do).sum() + (ob * dob).sum())

    arrs = [q, k, v, qb, kb, vb]
    gmap = {0: grads[0], 1: grads[1], 2: grads[2], 3: grads[3], 4: grads[4], 5: grads[5]}
    eps = 1e-6
    for which in range(6):
        a = arrs[which]
        for _ in range(6):
            idx = tuple(rs.integers(0, s) for s in a.shape)
            plus = [x.copy() for x in arrs]
            minus = [x.copy() for x in arrs]
            plus[which][idx] += eps
            minus[which][idx] -= eps
            fd = (f(*plus) - f(*minus)) / (2 * eps)
            an = gmap[which][idx]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (which, idx, fd, an)


@pytest.mark.parametrize("case", TINY_CASES)
def test_gradient_invariants(case):
    seed, S, ndoc, nanc, B, mode, Hq, Hkv, d = case
    q, k, v, qb, kb, vb, cu, anc = _tiny(seed, S, ndoc, nanc, B, mode, Hq, Hkv, d)
    rs = np.random.default_rng(seed + 7)
    do = rs.standard_normal(q.shape)
    dob = rs.standard_normal(qb.shape)
    _, dQ, dk, dv, dkb, dvb = orc.backward_rows(q, k, v, qb, kb, vb, do, dob, cu, anc, B, mode)
    G = Hq // Hkv
    dO = np.concatenate([do, dob.reshape(-1, Hq, d)])
    for g in range(Hkv):
        sdv = dv[:, g].sum(axis=0) + dvb[..., g, :].sum(axis=(0, 1))
        np.testing.assert_allclose(sdv, dO[:, g * G:(g + 1) * G].sum(axis=(0, 1)), atol=1e-9)
        sdk = dk[:, g].sum(axis=0) + dkb[..., g, :].sum(axis=(0, 1))
        np.testing.assert_allclose(sdk, 0.0, atol=1e-9)


def test_sparse_do_rows_give_exact_key_gradients():
    """With dO zero outside a row subset, backward_rows restricted to that
    subset equals the full closed-form gradient."""
    q, k, v, qb, kb, vb, cu, anc = _tiny(61, 56, 3, 10, 3, orc.BLOCK, 4, 2, 8)
    rs = np.random.default_rng(62)
    R = 56 + 30
    rows = np.sort(rs.choice(R, 17, replace=False))
    dO = np.zeros((R, 4, 8))
    dO[rows] = rs.standard_normal((17, 4, 8))
    do, dob = dO[:56], dO[56:].reshape(10, 3, 4, 8)
    full = orc.backward_brute(q, k, v, qb, kb, vb, do, dob, cu, anc, 3, orc.BLOCK)
    _, dQ, dk, dv, dkb, dvb = orc.backward_rows(q, k, v, qb, kb, vb, do, dob, cu, anc, 3, orc.BLOCK, rows=rows)
    np.testing.assert_allclose(dk, full[1], atol=1e-12)
    np.testing.assert_allclose(dv, full[2], atol=1e-12)
    np.testing.assert_allclose(dkb, full[4], atol=1e-12)
    np.testing.assert_allclose(dvb, full[5], atol=1e-12)
    dq_full = np.concatenate([full[0], full[3].reshape(-1, 4, 8)])
    np.testing.assert_allclose(dQ, dq_full[rows], atol=1e-12)


def test_sampled_rows_match_full_rows():
    q, k, v, qb, kb, vb, cu, anc = _tiny(71, 60, 4, 15, 3, orc.CHAIN, 4, 2, 8)
    _, O, L = orc.forward_rows(q, k, v, qb, kb, vb, cu, anc, 3, orc.CHAIN)
    rows = np.array([0, 5, 17, 59, 60, 61, 70, 104])
    r2, O2, L2 = orc.forward_rows(q, k, v, qb, kb, vb, cu, anc, 3, orc.CHAIN, rows=rows, block=3)
    np.testing.assert_allclose(O2, O[rows], atol=1e-13)
    np.testing.assert_allclose(L2, L[:, rows], atol=1e-13)


def test_pins_catch_planted_mistakes(monkeypatch):
    """A mistake planted in the oracle (anchor dropped from its own prefix)
    must be caught by the closed-form count pin."""
    q, k, v, qb, kb, vb, cu, anc = _tiny(31, 45, 3, 8, 3, orc.CHAIN, 2, 1, 8)
    k = np.zeros_like(k)
    kb = np.zeros_like(kb)
    real = orc.branch_attention.row_limits

    def wrong_limits(cu_, anchors_, B_):
        s, lim = real(cu_, anchors_, B_)
        S = int(np.asarray(cu_)[-1])
        lim = lim.copy()
        lim[S:] -= 1  # anchor excluded
        return s, lim

    monkeypatch.setattr(orc.branch_attention, "row_limits", wrong_limits)
    _, O, L = orc.branch_attention.forward_rows(q, k, v, qb, kb, vb, cu, anc, 3, orc.CHAIN)
    cnt = _visible_count(list(cu), list(anc), 3, orc.CHAIN, 45)
    assert not np.allclose(L[0], np.log(cnt), atol=1e-12)
