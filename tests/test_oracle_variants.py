"""Pins of the oracle's mask variants and of its per-rank ring partials.

* main-prefix window W: a window covering every document changes nothing; with
  K = 0 the LSE is the log of the visible-key count, counted here by distance
  (a key j is kept when 0 <= l - j < W) rather than by the oracle's interval
  rule; W = 1 leaves every main row its own key alone (O = v, LSE = own
  score); all forms agree; the backward matches torch autograd in fp64 on the
  explicit mask; an off-by-one planted in the window is caught;
* per-branch bitmask: lower-triangular words reproduce the chain mask and
  all-ones words the block mask exactly; K = 0 counts are the prefix plus the
  set bits; all forms and autograd agree;
* ring partials: partial k covers exactly the visible keys of virtual rank k's
  zigzag chunks (K = 0 counts), and the R partials merged by Eq. 2 give the
  main-sequence component.
"""
import math

import numpy as np
import pytest
import torch

import oracle as orc
import workloads as wl


def _tiny(seed, S, ndoc, nanc, B, Hq, Hkv, d):
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


def _random_masks(seed, Nb, B, p=0.5):
    rs = np.random.default_rng(seed)
    bits = rs.random((Nb, B, B)) < p
    words = np.zeros((Nb, B), dtype=np.uint64)
    for u in range(B):
        words |= bits[:, :, u].astype(np.uint64) << np.uint64(u)
    if Nb:
        words[0, 0] = 0  # a row that sees no branch key at all
    return words


def _doc_start(cu, p):
    for di in range(len(cu) - 1):
        if cu[di] <= p < cu[di + 1]:
            return int(cu[di])
    raise ValueError(p)


def _count_by_distance(cu, anc, B, W, S, branch_count):
    """Visible keys per row: main keys j of the row's document with
    0 <= l - j < W (all of them if W <= 0), plus branch_count(b, t)."""
    out = []
    for i in range(S):
        s = _doc_start(cu, i)
        out.append(sum(1 for j in range(s, i + 1) if W <= 0 or i - j < W))
    for b, a in enumerate(anc):
        s = _doc_start(cu, a)
        n = sum(1 for j in range(s, a + 1) if W <= 0 or a - j < W)
        for t in range(B):
            out.append(n + branch_count(b, t))
    return np.array(out, dtype=np.float64)


FORMS = ["brute", "rows", "decomposed", "ring"]


def _forward(form, args, B, mode, **kw):
    q, k, v, qb, kb, vb, cu, anc = args
    S, Hq, d = q.shape
    if form == "brute":
        return orc.forward_brute(q, k, v, qb, kb, vb, cu, anc, B, mode, **kw)
    if form == "decomposed":
        return orc.forward_decomposed(q, k, v, qb, kb, vb, cu, anc, B, mode, **kw)
    if form == "ring":
        return orc.forward_ring(q, k, v, qb, kb, vb, cu, anc, B, mode, R=3, **kw)
    _, O, L = orc.forward_rows(q, k, v, qb, kb, vb, cu, anc, B, mode, block=5, **kw)
    return O[:S], O[S:].reshape(-1, B, Hq, d), L


# --------------------------------------------------------------------------- window

@pytest.mark.parametrize("form", FORMS)
def test_window_covering_every_document_changes_nothing(form):
    args = _tiny(3, 40, 3, 9, 3, 2, 1, 8)
    cu = args[6]
    W = int(np.diff(cu).max())
    ref = _forward(form, args, 3, orc.CHAIN)
    got = _forward(form, args, 3, orc.CHAIN, window=W)
    for a, b in zip(got, ref):
        np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("W", [1, 2, 5, 9])
@pytest.mark.parametrize("form", FORMS)
def test_window_closed_form_zero_keys(form, W):
    q, k, v, qb, kb, vb, cu, anc = _tiny(31, 45, 3, 8, 3, 2, 1, 8)
    k = np.zeros_like(k)
    kb = np.zeros_like(kb)
    S = 45
    om, ob, L = _forward(form, (q, k, v, qb, kb, vb, cu, anc), 3, orc.CHAIN, window=W)
    cnt = _count_by_distance(list(cu), list(anc), 3, W, S, lambda b, t: t + 1)
    for h in range(2):
        np.testing.assert_allclose(L[h], np.log(cnt), atol=1e-12, rtol=0)
    for i in range(S):  # O = mean of the visible values
        s = _doc_start(cu, i)
        keep = [j for j in range(s, i + 1) if i - j < W]
        np.testing.assert_allclose(om[i, 0], v[keep, 0].mean(axis=0), atol=1e-12, rtol=0)
    for b, a in enumerate(anc):
        s = _doc_start(cu, a)
        keep = [j for j in range(s, a + 1) if a - j < W]
        for t in range(3):
            tot = v[keep, 0].sum(axis=0) + vb[b, :t + 1, 0].sum(axis=0)
            np.testing.assert_allclose(ob[b, t, 1], tot / (len(keep) + t + 1), atol=1e-12, rtol=0)


def test_window_one_leaves_each_main_row_its_own_key():
    q, k, v, qb, kb, vb, cu, anc = _tiny(5, 30, 2, 0, 3, 2, 2, 8)
    om, _, L = orc.forward_brute(q, k, v, qb, kb, vb, cu, anc, 3, orc.CHAIN, window=1)
    np.testing.assert_array_equal(om, v)  # softmax over one key: weight exactly 1
    sc = 1.0 / math.sqrt(8)
    for h in range(2):
        np.testing.assert_allclose(L[h], sc * (q[:, h] * k[:, h]).sum(-1), atol=1e-13, rtol=0)


@pytest.mark.parametrize("W", [1, 3, 7, 16])
def test_window_forms_agree(W):
    args = _tiny(8, 50, 2, 9, 5, 3, 3, 16)
    ref = _forward("brute", args, 5, orc.BLOCK, window=W)
    for form in ("rows", "decomposed"):
        for a, b in zip(_forward(form, args, 5, orc.BLOCK, window=W), ref):
            np.testing.assert_allclose(a, b, atol=1e-12, rtol=0)
    q, k, v, qb, kb, vb, cu, anc = args
    for R in (1, 2, 4):
        out = orc.forward_ring(q, k, v, qb, kb, vb, cu, anc, 5, orc.BLOCK, R=R, window=W)
        for a, b in zip(out, ref):
            np.testing.assert_allclose(a, b, atol=1e-12, rtol=0)


def test_window_pair_count_matches_mask():
    for seed in range(4):
        _, _, _, _, _, _, cu, anc = _tiny(seed, 37, 3, 11, 4, 1, 1, 4)
        for W in (1, 2, 6, 40):
            for mode in (orc.CHAIN, orc.BLOCK):
                M = orc.visible_mask(cu, anc, 4, mode, window=W)
                assert orc.visible_pair_count(cu, anc, 4, mode, window=W) == int(M.sum())


def _autograd(q, k, v, qb, kb, vb, do, dob, M, G, sc):
    """Gradients of sum(O * dO) for attention under the boolean mask M over
    the concatenated rows and keys, by torch autograd in fp64."""
    cat = lambda a, b: torch.cat([torch.from_numpy(a), torch.from_numpy(b).reshape(-1, *a.shape[1:])])
    Q, K, V = (cat(a, b).requires_grad_() for a, b in ((q, qb), (k, kb), (v, vb)))
    dO = cat(do, dob)
    Mt = torch.from_numpy(M)
    out = []
    for h in range(Q.shape[1]):
        s = sc * Q[:, h] @ K[:, h // G].T
        s = s.masked_fill(~Mt, -math.inf)
        out.append(torch.softmax(s, dim=-1) @ V[:, h // G])
    (torch.stack(out, 1) * dO).sum().backward()
    return Q.grad.numpy(), K.grad.numpy(), V.grad.numpy()


@pytest.mark.parametrize("variant", ["window", "bitmask", "window+bitmask"])
def test_variant_backward_matches_autograd(variant):
    B = 4
    q, k, v, qb, kb, vb, cu, anc = _tiny(12, 33, 3, 7, B, 4, 2, 8)
    rs = np.random.default_rng(3)
    do = rs.standard_normal(q.shape)
    dob = rs.standard_normal(qb.shape)
    W = 5 if "window" in variant else 0
    mode = orc.BITMASK if "bitmask" in variant else orc.CHAIN
    bm = _random_masks(4, len(anc), B) if mode == orc.BITMASK else None
    M = orc.visible_mask(cu, anc, B, mode, window=W, branch_mask=bm)
    dQ, dK, dV = _autograd(q, k, v, qb, kb, vb, do, dob, M, 2, 1 / math.sqrt(8))
    S = q.shape[0]
    for form in ("brute", "rows"):
        if form == "brute":
            g = orc.backward_brute(q, k, v, qb, kb, vb, do, dob, cu, anc, B, mode, window=W, branch_mask=bm)
            dq, dk, dv, dqb, dkb, dvb = g
        else:
            _, dQr, dk, dv, dkb, dvb = orc.backward_rows(q, k, v, qb, kb, vb, do, dob, cu, anc, B, mode,
                                                        window=W, branch_mask=bm, block=6)
            dq, dqb = dQr[:S], dQr[S:]
        np.testing.assert_allclose(np.concatenate([dq, np.reshape(dqb, (-1,) + q.shape[1:])]), dQ, atol=1e-10)
        np.testing.assert_allclose(np.concatenate([dk, np.reshape(dkb, (-1,) + k.shape[1:])]), dK, atol=1e-10)
        np.testing.assert_allclose(np.concatenate([dv, np.reshape(dvb, (-1,) + v.shape[1:])]), dV, atol=1e-10)


def test_window_pins_catch_an_off_by_one(monkeypatch):
    """A window that keeps one key too many (l - W instead of l - W + 1) is
    caught by the distance count."""
    q, k, v, qb, kb, vb, cu, anc = _tiny(31, 45, 3, 8, 3, 2, 1, 8)
    k = np.zeros_like(k)
    kb = np.zeros_like(kb)
    real = orc.branch_attention.row_first_keys
    monkeypatch.setattr(orc.branch_attention, "row_first_keys",
                        lambda s, lim, window=0: real(s, lim, window + 1 if window else window))
    _, O, L = orc.branch_attention.forward_rows(q, k, v, qb, kb, vb, cu, anc, 3, orc.CHAIN, window=4)
    cnt = _count_by_distance(list(cu), list(anc), 3, 4, 45, lambda b, t: t + 1)
    assert not np.allclose(L[0], np.log(cnt), atol=1e-12)


# --------------------------------------------------------------------------- bitmask

@pytest.mark.parametrize("form", FORMS)
def test_bitmask_reproduces_chain_and_block(form):
    B = 4
    args = _tiny(2, 33, 3, 7, B, 4, 2, 8)
    Nb = len(args[7])
    lower = np.array([(1 << (t + 1)) - 1 for t in range(B)], dtype=np.uint64)
    chain_words = np.tile(lower, (Nb, 1))
    block_words = np.full((Nb, B), (1 << B) - 1, dtype=np.uint64)
    for words, mode in ((chain_words, orc.CHAIN), (block_words, orc.BLOCK)):
        ref = _forward(form, args, B, mode)
        got = _forward(form, args, B, orc.BITMASK, branch_mask=words)
        for a, b in zip(got, ref):
            np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("form", FORMS)
def test_bitmask_closed_form_zero_keys(form):
    B = 5
    q, k, v, qb, kb, vb, cu, anc = _tiny(17, 41, 2, 9, B, 2, 1, 8)
    k = np.zeros_like(k)
    kb = np.zeros_like(kb)
    words = _random_masks(9, len(anc), B)
    om, ob, L = _forward(form, (q, k, v, qb, kb, vb, cu, anc), B, orc.BITMASK, branch_mask=words)
    popcount = lambda b, t: bin(int(words[b, t])).count("1")
    cnt = _count_by_distance(list(cu), list(anc), B, 0, 41, popcount)
    np.testing.assert_allclose(L[0], np.log(cnt), atol=1e-12, rtol=0)
    for b, a in enumerate(anc):
        s = _doc_start(cu, a)
        for t in range(B):
            seen = [u for u in range(B) if (int(words[b, t]) >> u) & 1]
            tot = v[s:a + 1, 0].sum(axis=0) + vb[b, seen, 0].sum(axis=0)
            np.testing.assert_allclose(ob[b, t, 0], tot / (a - s + 1 + len(seen)), atol=1e-12, rtol=0)


def test_bitmask_forms_agree_and_count():
    B = 6
    args = _tiny(21, 60, 4, 13, B, 3, 1, 16)
    q, k, v, qb, kb, vb, cu, anc = args
    words = _random_masks(5, len(anc), B, p=0.3)
    ref = _forward("brute", args, B, orc.BITMASK, branch_mask=words)
    for form in ("rows", "decomposed", "ring"):
        for a, b in zip(_forward(form, args, B, orc.BITMASK, branch_mask=words), ref):
            np.testing.assert_allclose(a, b, atol=1e-12, rtol=0)
    M = orc.visible_mask(cu, anc, B, orc.BITMASK, branch_mask=words)
    assert orc.visible_pair_count(cu, anc, B, orc.BITMASK, branch_mask=words) == int(M.sum())


# --------------------------------------------------------------------------- ring partials

def _owner_of(cu, R):
    """Virtual rank owning each main position: its document is cut into 2R
    chunks [s + floor(kL/2R), s + floor((k+1)L/2R)); chunk k belongs to rank
    k for k < R and to 2R-1-k otherwise.  Enumerated position by position."""
    own = {}
    for di in range(len(cu) - 1):
        s, e = int(cu[di]), int(cu[di + 1])
        L = e - s
        for p in range(s, e):
            kk = max(c for c in range(2 * R) if s + (c * L) // (2 * R) <= p)
            own[p] = kk if kk < R else 2 * R - 1 - kk
    return own


@pytest.mark.parametrize("R,W", [(1, 0), (2, 0), (3, 0), (4, 6), (8, 0)])
def test_ring_partials_cover_each_ranks_keys(R, W):
    B = 3
    q, k, v, qb, kb, vb, cu, anc = _tiny(41, 70, 3, 12, B, 2, 1, 8)
    k0, kb0 = np.zeros_like(k), np.zeros_like(kb)
    PO, PL = orc.forward_ring(q, k0, v, qb, kb0, vb, cu, anc, B, orc.CHAIN, R=R, window=W, partials=True)
    own = _owner_of(list(cu), R)
    S = 70
    rows_lim = list(range(S)) + [int(a) for a in anc for _ in range(B)]
    for r, lim in enumerate(rows_lim):
        s = _doc_start(cu, lim)
        for kk in range(R):
            keys = [j for j in range(s, lim + 1) if own[j] == kk and (W <= 0 or lim - j < W)]
            if keys:
                assert PL[kk, 0, r] == pytest.approx(math.log(len(keys)), abs=1e-12)
                np.testing.assert_allclose(PO[kk, r, 0], v[keys, 0].mean(axis=0), atol=1e-12)
            else:
                assert PL[kk, 0, r] == -np.inf and not PO[kk, r].any()


@pytest.mark.parametrize("R", [2, 4, 5])
def test_ring_partials_merge_to_main_component(R):
    B = 3
    q, k, v, qb, kb, vb, cu, anc = _tiny(43, 64, 2, 10, B, 4, 2, 8)
    PO, PL = orc.forward_ring(q, k, v, qb, kb, vb, cu, anc, B, orc.CHAIN, R=R, partials=True)
    O, L = orc.lse_merge(list(PO), [pl.T for pl in PL])
    Om, Lm = orc.main_part(q, k, v, qb, cu, anc, B)
    np.testing.assert_allclose(O, Om, atol=1e-12)
    np.testing.assert_allclose(L.T, Lm, atol=1e-12)
