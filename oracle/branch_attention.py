"""fp64 CPU oracle for branch attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline / reference leg of ``bench.py`` use it.  It shares no code with the
CUDA library (no kernels, headers, tables or helpers); both sides take their
inputs from the seeded generators in ``workloads``.

What it computes
----------------
Source: "Online Draft Co-Training for Speculative Decoding in Large-Scale,
Long-Context RL Post-Training" (arXiv 2609.07108), §3.2 and Eq. 2, as described
on the rcap.io post (paragraph "The first hard part is branch attention under
context parallelism"), the evolve.pub review (Summary; FAQ "How does the paper
run draft branch attention under context parallelism?") and the cere-bro wiki
page ("Obstacle one, context parallelism").

The pages say a branch query sees the causal prefix of the main sequence up to
its anchor plus a few branch-local keys, that the two pieces are computed
separately and merged with the log-sum-exp rule ring attention uses between
ring steps, and that the decomposition leaves the numerics unchanged.  So the method reaches,
up to rounding order, plain masked softmax attention over the concatenated
[main; branch] rows and keys.  The oracle writes that definition out:

* packed main sequence of S tokens, documents given by ``cu_seqlens``;
  s(i) = start of the document holding position i;
* main row i sees main keys j in [s(i), i];
* branch b hangs off anchor a_b (a packed main position) and has B rows
  t = 0..B-1.  Row (b, t) sees main keys j in [s(a_b), a_b] and branch keys
  (b, u) with u <= t (CHAIN, EAGLE-3 training-time test) or all u < B (BLOCK,
  DFlash-style block draft);
* BITMASK (a generic per-branch mask, the form DSpark's Markov head needs;
  the pages do not spell that mask out): row (b, t) sees branch key (b, u)
  iff bit u of branch_mask[b, t] is set (branch_mask uint64 [Nb, B]);
* optional main-prefix window W > 0 (the pages call the recipe independent of
  the draft architecture; windowed drafts are one such variant): a row whose
  last visible main key is l sees only main keys [max(s(l), l - W + 1), l];
  branch keys are unaffected; W <= 0 means no window;
* main rows never see branch keys; no branch sees another branch's keys;
* s_ij = scale * <q_i, k_j>, scale = 1/sqrt(d) unless given;
  L_i = log sum_j exp(s_ij) (natural log), O_i = sum_j exp(s_ij - L_i) v_j;
* GQA: q head h uses KV head floor(h / (Hq / Hkv)).

Backward (the pages are silent; this is the textbook softmax-attention
gradient of the definition above): D_i = <dO_i, O_i>, P_ij = exp(s_ij - L_i),
dS_ij = P_ij (<dO_i, v_j> - D_i), dQ_i = scale sum_j dS_ij k_j,
dK_j = scale sum_{h in group} sum_i dS_ij q_i, dV_j = sum_{h in group} sum_i P_ij dO_i.

Forms
-----
1. ``forward_brute`` / ``backward_brute``: explicit [R, R] mask over the
   concatenated rows (R = S + Nb*B) and a naive softmax.  Tiny sizes only.
2. ``forward_rows`` / ``backward_rows``: per row, the visible key set gathered
   from the definition, one softmax over it; row blocks for speed.  Works on
   any subset of rows (sampled rows at large S).
3. ``forward_decomposed`` / ``forward_ring``: the method's own steps, written to
   be checked against 1-2: main-sequence part with per-row causal limits,
   branch-local part, Eq. 2 merge; and the ring form with R CPU ranks holding
   zigzag chunks, K/V chunks "sent" around the ring and per-step partials merged
   in ring order.

Readings where the pages are silent (all forms agree on them):
anchor included in its own prefix; causal-within-branch includes self (u <= t);
the prefix never crosses a document boundary; scale 1/sqrt(d); natural-log LSE;
an empty partial is (O, LSE) = (0, -inf) and merging with it is the identity;
zigzag chunk k of a document [s, s+L) is [s + floor(kL/2R), s + floor((k+1)L/2R)),
rank r owns chunks r and 2R-1-r, a branch belongs to the rank owning its anchor.

Inputs may be numpy arrays or torch tensors (bf16 converts exactly to fp64).
Layouts: q [S,Hq,d], k/v [S,Hkv,d], qb [Nb,B,Hq,d], kb/vb [Nb,B,Hkv,d],
LSE [Hq, S+Nb*B] with main rows first, then branch rows b-major, depth minor.
"""
from __future__ import annotations

import math

import numpy as np

CHAIN = 0
BLOCK = 1
BITMASK = 2


# --------------------------------------------------------------------------
# helpers: conversion and the visible-key definition
# --------------------------------------------------------------------------

def f64(x) -> np.ndarray:
    """Exact conversion of a numpy array or (bf16/fp32) torch tensor to fp64."""
    if hasattr(x, "detach"):
        x = x.detach().cpu()
        import torch  # local: only needed for tensors
        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def i64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.asarray(x, dtype=np.int64)


def default_scale(d: int, scale=None) -> float:
    return 1.0 / math.sqrt(d) if (scale is None or scale <= 0) else float(scale)


def doc_start_of(cu: np.ndarray, pos) -> np.ndarray:
    """Start of the document holding each packed main position."""
    idx = np.searchsorted(cu, np.asarray(pos), side="right") - 1
    return cu[idx]


def row_limits(cu, anchors, B):
    """Per concatenated row: (doc start, last visible main key).  Main row i:
    (s(i), i).  Branch row (b, t): (s(a_b), a_b)."""
    cu = i64(cu)
    anchors = i64(anchors)
    S = int(cu[-1])
    main = np.arange(S)
    lim = np.concatenate([main, np.repeat(anchors, B)])
    return doc_start_of(cu, lim), lim


def row_first_keys(starts, lim, window=0):
    """First visible main key of each row: its document start, or with a
    window W > 0 the later of that and lim - W + 1."""
    starts = np.asarray(starts)
    if window is None or window <= 0:
        return starts
    return np.maximum(starts, np.asarray(lim) - int(window) + 1)


def branch_sees(mode, t, u, mask_bits=None):
    """Does depth t of a branch see that branch's key u?  CHAIN: u <= t;
    BLOCK: always; BITMASK: bit u of the row's mask word.  Works elementwise
    on arrays (mask_bits: the row's uint64 word, broadcast like t)."""
    t = np.asarray(t)
    u = np.asarray(u)
    if mode == CHAIN:
        return u <= t
    if mode == BLOCK:
        return np.ones(np.broadcast(t, u).shape, dtype=bool)
    if mode == BITMASK:
        bits = np.asarray(mask_bits, dtype=np.uint64)
        return ((bits >> u.astype(np.uint64)) & np.uint64(1)) == np.uint64(1)
    raise ValueError(f"unknown mask mode {mode}")


def visible_mask(cu, anchors, B: int, mode: int, window: int = 0, branch_mask=None) -> np.ndarray:
    """Explicit [R, R] boolean mask over concatenated rows x keys, written
    entry by entry from the definition (tiny sizes only)."""
    cu = i64(cu)
    anchors = i64(anchors)
    S = int(cu[-1])
    Nb = len(anchors)
    R = S + Nb * B
    M = np.zeros((R, R), dtype=bool)
    for i in range(S):
        s = int(doc_start_of(cu, i))
        if window and window > 0:
            s = max(s, i - window + 1)
        for j in range(s, i + 1):
            M[i, j] = True
    for b in range(Nb):
        a = int(anchors[b])
        s = int(doc_start_of(cu, a))
        if window and window > 0:
            s = max(s, a - window + 1)
        for t in range(B):
            r = S + b * B + t
            for j in range(s, a + 1):
                M[r, j] = True
            for u in range(B):
                if mode == BLOCK:
                    seen = True
                elif mode == CHAIN:
                    seen = u <= t
                else:
                    seen = (int(branch_mask[b][t]) >> u) & 1 == 1
                if seen:
                    M[r, S + b * B + u] = True
    return M


class _Lazy:
    """fp64 view of rows of a [N, H, d] array/tensor, or of the row-wise
    concatenation of a main [S, H, d] and a branch [Nb, B, H, d] input,
    converted only where read (keeps sampled-row checks at large S cheap)."""

    def __init__(self, main, br=None):
        self.main = main
        self.S = main.shape[0]
        self.br = None
        if br is not None and br.shape[0] * br.shape[1] > 0:
            self.br = br.reshape(br.shape[0] * br.shape[1], *br.shape[2:])

    @staticmethod
    def _take(x, idx, h):
        if hasattr(x, "detach"):
            import torch
            t = x[torch.as_tensor(idx, dtype=torch.long), h]
            return t.detach().cpu().to(torch.float64).numpy()
        return np.asarray(x[idx, h], dtype=np.float64)

    def rows(self, idx, h):
        idx = np.asarray(idx, dtype=np.int64)
        if self.br is None or (idx < self.S).all():
            return self._take(self.main, idx, h)
        out = np.empty((len(idx), self.main.shape[2]))
        m = idx < self.S
        if m.any():
            out[m] = self._take(self.main, idx[m], h)
        if (~m).any():
            out[~m] = self._take(self.br, idx[~m] - self.S, h)
        return out


def _concat(main, br):
    """[S,H,d] and [Nb,B,H,d] -> [S+Nb*B, H, d]."""
    main = f64(main)
    br = f64(br)
    return np.concatenate([main, br.reshape(-1, main.shape[1], main.shape[2])], axis=0)


def _split_rows(x, S, Nb, B):
    return x[:S], x[S:].reshape(Nb, B, *x.shape[1:])


# --------------------------------------------------------------------------
# form 1: brute force over the full mask
# --------------------------------------------------------------------------

def forward_brute(q, k, v, qb, kb, vb, cu, anchors, B, mode, scale=None, window=0,
                  branch_mask=None):
    """Returns (O_main [S,Hq,d], O_branch [Nb,B,Hq,d], LSE [Hq,R])."""
    Q, K, V = _concat(q, qb), _concat(k, kb), _concat(v, vb)
    S = int(i64(cu)[-1])
    Nb = len(i64(anchors))
    Hq, Hkv, d = Q.shape[1], K.shape[1], Q.shape[2]
    G = Hq // Hkv
    sc = default_scale(d, scale)
    M = visible_mask(cu, anchors, B, mode, window, branch_mask)
    O = np.zeros_like(Q)
    lse = np.zeros((Hq, Q.shape[0]))
    for h in range(Hq):
        g = h // G
        s = sc * (Q[:, h] @ K[:, g].T)
        s = np.where(M, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        l = e.sum(axis=1, keepdims=True)
        lse[h] = (m + np.log(l))[:, 0]
        O[:, h] = (e / l) @ V[:, g]
    om, ob = _split_rows(O, S, Nb, B)
    return om, ob, lse


def backward_brute(q, k, v, qb, kb, vb, do, dob, cu, anchors, B, mode, scale=None, window=0,
                   branch_mask=None):
    """Closed-form gradients over the full mask.
    Returns (dq, dk, dv, dqb, dkb, dvb) in the input layouts (fp64)."""
    Q, K, V = _concat(q, qb), _concat(k, kb), _concat(v, vb)
    dO = _concat(do, dob)
    S = int(i64(cu)[-1])
    Nb = len(i64(anchors))
    Hq, Hkv, d = Q.shape[1], K.shape[1], Q.shape[2]
    G = Hq // Hkv
    sc = default_scale(d, scale)
    M = visible_mask(cu, anchors, B, mode, window, branch_mask)
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    for h in range(Hq):
        g = h // G
        s = np.where(M, sc * (Q[:, h] @ K[:, g].T), -np.inf)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        P = e / e.sum(axis=1, keepdims=True)
        O = P @ V[:, g]
        Dv = (dO[:, h] * O).sum(axis=1, keepdims=True)
        dP = dO[:, h] @ V[:, g].T
        dS = P * (dP - Dv)
        dQ[:, h] = sc * (dS @ K[:, g])
        dK[:, g] += sc * (dS.T @ Q[:, h])
        dV[:, g] += P.T @ dO[:, h]
    dq, dqb = _split_rows(dQ, S, Nb, B)
    dk, dkb = _split_rows(dK, S, Nb, B)
    dv, dvb = _split_rows(dV, S, Nb, B)
    return dq, dk, dv, dqb, dkb, dvb


# --------------------------------------------------------------------------
# form 2: per-row visible key sets (row blocks), any subset of rows
# --------------------------------------------------------------------------

def _row_blocks(rows, cu, anchors, B, block, window=0):
    """Group requested concatenated row indices into blocks whose rows share a
    document; yields (rows, first main key of the block, per-row first main
    keys, limits, branch_id, depth)."""
    cu = i64(cu)
    anchors = i64(anchors)
    S = int(cu[-1])
    rows = np.asarray(rows, dtype=np.int64)
    starts, lim = row_limits(cu, anchors, B)
    first = row_first_keys(starts, lim, window)
    doc = np.searchsorted(cu, lim[rows], side="right") - 1
    order = np.lexsort((lim[rows], doc))
    rows = rows[order]
    doc = doc[order]
    i = 0
    n = len(rows)
    while i < n:
        j = i
        while j < n and doc[j] == doc[i] and j - i < block:
            j += 1
        r = rows[i:j]
        isb = r >= S
        bid = np.where(isb, (r - S) // max(B, 1), -1)
        dep = np.where(isb, (r - S) % max(B, 1), -1)
        yield r, int(first[r].min()), first[r], lim[r], bid, dep
        i = j


class _Window:
    """Key rows gathered for one row block: main keys [s0, s0 + n) (``s0`` set)
    or the listed branch key rows (``ids`` set)."""

    def __init__(self, data, s0, ids=None):
        self.data, self.s0, self.ids = data, s0, ids


def _block_scores(Qh, Kmain, Kbr, s0, first, lim, bid, dep, B, mode, sc, branch_mask=None):
    """Scores of a row block against its visible keys: main keys [s0, max lim]
    (masked to each row's own [first, limit]) and the branch keys of the
    block's branches (masked to each row's own branch and mask rule).  Returns
    (scores [nr, nk], main key index array, branch key index array)."""
    hi = int(lim.max())
    mk = np.arange(s0, hi + 1)
    s_main = sc * (Qh @ Kmain.data.T)
    s_main = np.where((mk[None, :] <= lim[:, None]) & (mk[None, :] >= first[:, None]), s_main, -np.inf)
    if Kbr is None:
        return s_main, mk, np.zeros(0, dtype=np.int64)
    bk = Kbr.ids
    kb_b = bk // B
    kb_u = bk % B
    s_br = sc * (Qh @ Kbr.data.T)
    bits = None
    if mode == BITMASK:
        bm = np.asarray(branch_mask, dtype=np.uint64)
        bits = np.where(bid >= 0, bm[np.maximum(bid, 0), np.maximum(dep, 0)], 0)[:, None]
    vis = (kb_b[None, :] == bid[:, None]) & branch_sees(mode, dep[:, None], kb_u[None, :], bits)
    s_br = np.where(vis, s_br, -np.inf)
    return np.concatenate([s_main, s_br], axis=1), mk, bk


def forward_rows(q, k, v, qb, kb, vb, cu, anchors, B, mode, scale=None, rows=None,
                 heads=None, block=512, window=0, branch_mask=None):
    """O and LSE of the requested concatenated rows (default: all rows).
    Returns (rows [n], O [n, Hq, d], LSE [Hq, n]); heads outside ``heads`` are 0."""
    S, Hq, d = q.shape
    Hkv = k.shape[1]
    Nb = qb.shape[0]
    G = Hq // Hkv
    sc = default_scale(d, scale)
    if rows is None:
        rows = np.arange(S + Nb * B)
    rows = np.asarray(rows, dtype=np.int64)
    heads = list(range(Hq)) if heads is None else list(heads)
    Qc = _Lazy(q, qb)
    Km, Vm = _Lazy(k), _Lazy(v)
    Kb, Vb = _Lazy(kb.reshape(-1, 1, Hkv, d)[:, 0] if Nb else k[:0]), _Lazy(vb.reshape(-1, 1, Hkv, d)[:, 0] if Nb else v[:0])
    pos = {int(r): n for n, r in enumerate(rows)}
    O = np.zeros((len(rows), Hq, d))
    L = np.full((Hq, len(rows)), np.nan)
    for r, s0, first, lim, bid, dep in _row_blocks(rows, cu, anchors, B, block, window):
        idx = np.array([pos[int(x)] for x in r])
        hi = int(lim.max())
        mk = np.arange(s0, hi + 1)
        ub = np.unique(bid[bid >= 0])
        bk = (ub[:, None] * B + np.arange(B)[None, :]).reshape(-1) if len(ub) else np.zeros(0, np.int64)
        for h in heads:
            g = h // G
            Kmain = _Window(Km.rows(mk, g), s0)
            Kbr = _Window(Kb.rows(bk, g), None, bk) if len(bk) else None
            s, _, _ = _block_scores(Qc.rows(r, h), Kmain, Kbr, s0, first, lim, bid, dep, B, mode, sc,
                                    branch_mask)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            l = e.sum(axis=1, keepdims=True)
            Vv = np.concatenate([Vm.rows(mk, g), Vb.rows(bk, g) if len(bk) else np.zeros((0, d))], axis=0)
            O[idx, h] = (e / l) @ Vv
            L[h, idx] = (m + np.log(l))[:, 0]
    return rows, O, L


def backward_rows(q, k, v, qb, kb, vb, do, dob, cu, anchors, B, mode, scale=None, rows=None,
                  heads=None, block=512, window=0, branch_mask=None):
    """Closed-form backward restricted to the contributions of the requested
    rows (default: all rows).  With dO zero outside ``rows`` this is the exact
    full gradient.  Returns (rows, dQ [n, Hq, d] of those rows,
    dk, dv [S,Hkv,d], dkb, dvb [Nb,B,Hkv,d]); only ``heads`` contribute."""
    S, Hq, d = q.shape
    Hkv = k.shape[1]
    Nb = qb.shape[0]
    G = Hq // Hkv
    sc = default_scale(d, scale)
    if rows is None:
        rows = np.arange(S + Nb * B)
    rows = np.asarray(rows, dtype=np.int64)
    heads = list(range(Hq)) if heads is None else list(heads)
    Qc = _Lazy(q, qb)
    dOc = _Lazy(do, dob)
    Km, Vm = _Lazy(k), _Lazy(v)
    Kb = _Lazy(kb.reshape(-1, 1, Hkv, d)[:, 0] if Nb else k[:0])
    Vb = _Lazy(vb.reshape(-1, 1, Hkv, d)[:, 0] if Nb else v[:0])
    dk = np.zeros((S, Hkv, d))
    dv = np.zeros((S, Hkv, d))
    dkbf = np.zeros((Nb * B, Hkv, d))
    dvbf = np.zeros((Nb * B, Hkv, d))
    pos = {int(r): n for n, r in enumerate(rows)}
    dQ = np.zeros((len(rows), Hq, d))
    for r, s0, first, lim, bid, dep in _row_blocks(rows, cu, anchors, B, block, window):
        idx = np.array([pos[int(x)] for x in r])
        hi = int(lim.max())
        mk = np.arange(s0, hi + 1)
        ub = np.unique(bid[bid >= 0])
        bk = (ub[:, None] * B + np.arange(B)[None, :]).reshape(-1) if len(ub) else np.zeros(0, np.int64)
        for h in heads:
            g = h // G
            Km_g = Km.rows(mk, g)
            Kb_g = Kb.rows(bk, g) if len(bk) else np.zeros((0, d))
            Qh = Qc.rows(r, h)
            s, _, _ = _block_scores(Qh, _Window(Km_g, s0), _Window(Kb_g, None, bk) if len(bk) else None,
                                    s0, first, lim, bid, dep, B, mode, sc, branch_mask)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            P = e / e.sum(axis=1, keepdims=True)
            Kk = np.concatenate([Km_g, Kb_g], axis=0)
            Vv = np.concatenate([Vm.rows(mk, g), Vb.rows(bk, g) if len(bk) else np.zeros((0, d))], axis=0)
            O = P @ Vv
            dOh = dOc.rows(r, h)
            Dv = (dOh * O).sum(axis=1, keepdims=True)
            dP = dOh @ Vv.T
            dS = P * (dP - Dv)
            dQ[idx, h] = sc * (dS @ Kk)
            gk = sc * (dS.T @ Qh)
            gv = P.T @ dOh
            nm = len(mk)
            dk[mk, g] += gk[:nm]
            dv[mk, g] += gv[:nm]
            if len(bk):
                dkbf[bk, g] += gk[nm:]
                dvbf[bk, g] += gv[nm:]
    return rows, dQ, dk, dv, dkbf.reshape(Nb, B, Hkv, d), dvbf.reshape(Nb, B, Hkv, d)


# --------------------------------------------------------------------------
# form 3: the method's own decomposition (main part, branch part, Eq. 2 merge)
# --------------------------------------------------------------------------

def attend(Qh, Kg, Vg, mask, sc):
    """Partial softmax attention of rows Qh [n,d] over keys Kg/Vg [m,d] under a
    boolean mask [n,m].  Rows with no visible key give the empty partial
    (O = 0, LSE = -inf)."""
    n = Qh.shape[0]
    O = np.zeros((n, Vg.shape[1]))
    L = np.full(n, -np.inf)
    if Kg.shape[0] == 0:
        return O, L
    s = np.where(mask, sc * (Qh @ Kg.T), -np.inf)
    any_ = mask.any(axis=1)
    if not any_.any():
        return O, L
    m = np.where(any_, s.max(axis=1), 0.0)
    e = np.where(mask, np.exp(s - m[:, None]), 0.0)
    l = e.sum(axis=1)
    ok = l > 0
    O[ok] = (e[ok] / l[ok, None]) @ Vg
    L[ok] = m[ok] + np.log(l[ok])
    return O, L


def lse_merge(o_parts, lse_parts):
    """Eq. 2, k-way: L = log sum_p exp(L_p), O = sum_p exp(L_p - L) O_p.
    o_parts: list of [n, ..., d]; lse_parts: list of matching [n, ...] arrays.
    Empty partials (LSE = -inf) contribute nothing; all-empty gives (0, -inf)."""
    lse = np.stack([np.asarray(x, dtype=np.float64) for x in lse_parts])
    mx = lse.max(axis=0)
    finite = np.isfinite(mx)
    mxs = np.where(finite, mx, 0.0)
    w = np.where(np.isfinite(lse), np.exp(lse - mxs), 0.0)
    tot = w.sum(axis=0)
    L = np.where(finite, mxs + np.log(np.where(finite, tot, 1.0)), -np.inf)
    O = np.zeros_like(np.asarray(o_parts[0], dtype=np.float64))
    for p, op in enumerate(o_parts):
        coef = np.where(finite, np.where(np.isfinite(lse[p]), np.exp(lse[p] - np.where(finite, L, 0.0)), 0.0), 0.0)
        O = O + coef[..., None] * np.asarray(op, dtype=np.float64)
    return O, L


def main_part(q, k, v, qb, cu, anchors, B, scale=None, window=0):
    """Main-sequence component for every row (main rows then branch rows):
    each row against main keys [s(limit), limit] (with a window W > 0:
    [max(s(limit), limit - W + 1), limit]).  Returns O [R,Hq,d], LSE [Hq,R]."""
    q, k, v, qb = (f64(x) for x in (q, k, v, qb))
    S, Hq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    sc = default_scale(d, scale)
    Qc = np.concatenate([q, qb.reshape(-1, Hq, d)], axis=0)
    starts, lim = row_limits(cu, anchors, B)
    R = Qc.shape[0]
    O = np.zeros((R, Hq, d))
    L = np.zeros((Hq, R))
    cu_ = i64(cu)
    for di in range(len(cu_) - 1):
        s, e = int(cu_[di]), int(cu_[di + 1])
        r = np.nonzero((lim >= s) & (lim < e))[0]
        if len(r) == 0:
            continue
        keys = np.arange(s, e)
        first = row_first_keys(starts[r], lim[r], window)
        mask = (keys[None, :] <= lim[r][:, None]) & (keys[None, :] >= first[:, None])
        for h in range(Hq):
            g = h // G
            O[r, h], L[h, r] = attend(Qc[r, h], k[s:e, g], v[s:e, g], mask, sc)
    return O, L


def branch_part(qb, kb, vb, B, mode, scale=None, branch_mask=None):
    """Branch-local component: each branch row against its own branch's keys
    (u <= t for CHAIN, all u for BLOCK, the row's bits for BITMASK).  Returns
    O [Nb*B,Hq,d], LSE [Hq,Nb*B]."""
    qb, kb, vb = (f64(x) for x in (qb, kb, vb))
    Nb, _, Hq, d = qb.shape
    Hkv = kb.shape[2]
    G = Hq // Hkv
    sc = default_scale(d, scale)
    O = np.zeros((Nb * B, Hq, d))
    L = np.zeros((Hq, Nb * B))
    t = np.arange(B)
    for b in range(Nb):
        bits = np.asarray(branch_mask, dtype=np.uint64)[b][:, None] if mode == BITMASK else None
        mask = branch_sees(mode, t[:, None], t[None, :], bits)
        for h in range(Hq):
            g = h // G
            O[b * B:(b + 1) * B, h], L[h, b * B:(b + 1) * B] = attend(qb[b, :, h], kb[b, :, g], vb[b, :, g], mask, sc)
    return O, L


def forward_decomposed(q, k, v, qb, kb, vb, cu, anchors, B, mode, scale=None, window=0,
                       branch_mask=None):
    """Main part + branch part merged by Eq. 2.  Same outputs as forward_brute."""
    S = q.shape[0]
    Nb = qb.shape[0]
    Om, Lm = main_part(q, k, v, qb, cu, anchors, B, scale, window)
    O = Om.copy()
    L = Lm.copy()
    if Nb:
        Ob, Lb = branch_part(qb, kb, vb, B, mode, scale, branch_mask)
        ob, lb = lse_merge([Om[S:], Ob], [Lm[:, S:].T, Lb.T])
        O[S:] = ob
        L[:, S:] = lb.T
    om, obr = _split_rows(O, S, Nb, B)
    return om, obr, L


def zigzag_chunks(cu, R: int):
    """Per document of length L at start s: 2R chunks, chunk k =
    [s + floor(kL/2R), s + floor((k+1)L/2R)), owned by rank k if k < R else
    2R-1-k.  Returns a list of (doc, k, start, end, rank)."""
    cu = i64(cu)
    out = []
    for di in range(len(cu) - 1):
        s, e = int(cu[di]), int(cu[di + 1])
        L = e - s
        for kk in range(2 * R):
            a = s + (kk * L) // (2 * R)
            b = s + ((kk + 1) * L) // (2 * R)
            out.append((di, kk, a, b, kk if kk < R else 2 * R - 1 - kk))
    return out


def forward_ring(q, k, v, qb, kb, vb, cu, anchors, B, mode, R, scale=None, step_order=None,
                 window=0, branch_mask=None, partials=False):
    """Ring form with R CPU ranks.  Rank r holds the main Q/K/V rows of its
    zigzag chunks and the branches anchored in them.  For ring step st (in
    ``step_order``, default 0..R-1) rank r holds the K/V chunks sent from rank
    (r - st) mod R, attends its rows to the visible ones and merges the step's
    partial into its running (O, LSE) with Eq. 2.  Finally each rank merges its
    branch rows' branch-local part.  Branch K/V never leave their rank.

    With ``partials`` it returns instead, for every rank k, the partial
    (O, LSE) of every row over the visible main keys of rank k's chunks, i.e.
    what the row's rank computes at the ring step where k's K/V visit it:
    (O [R, rows, Hq, d], LSE [R, Hq, rows]); empty partials are (0, -inf)."""
    q, k, v, qb, kb, vb = (f64(x) for x in (q, k, v, qb, kb, vb))
    S, Hq, d = q.shape
    Hkv = k.shape[1]
    Nb = qb.shape[0]
    G = Hq // Hkv
    sc = default_scale(d, scale)
    anc = i64(anchors)
    chunks = zigzag_chunks(cu, R)
    starts, lim = row_limits(cu, anchors, B)
    first = row_first_keys(starts, lim, window)
    Qc = np.concatenate([q, qb.reshape(-1, Hq, d)], axis=0)
    owner_rows = {r: [] for r in range(R)}
    owner_keys = {r: [] for r in range(R)}
    for (_, _, a, b, rk) in chunks:
        owner_rows[rk].extend(range(a, b))
        owner_keys[rk].extend(range(a, b))
        for bi in np.nonzero((anc >= a) & (anc < b))[0]:
            owner_rows[rk].extend(range(S + bi * B, S + (bi + 1) * B))
    # each rank's resident K/V "shard" (what it would send around the ring)
    shard = {r: (np.array(owner_keys[r], dtype=np.int64),
                 k[owner_keys[r]], v[owner_keys[r]]) for r in range(R)}
    O = np.zeros((S + Nb * B, Hq, d))
    L = np.full((Hq, S + Nb * B), -np.inf)
    steps = list(range(R)) if step_order is None else list(step_order)
    assert sorted(steps) == list(range(R))
    if partials:
        PO = np.zeros((R, S + Nb * B, Hq, d))
        PL = np.full((R, Hq, S + Nb * B), -np.inf)
    for r in range(R):
        rows = np.array(sorted(owner_rows[r]), dtype=np.int64)
        if len(rows) == 0:
            continue
        run_O = np.zeros((len(rows), Hq, d))
        run_L = np.full((Hq, len(rows)), -np.inf)
        for st in steps:
            kidx, Ks, Vs = shard[(r - st) % R]  # the chunk pair received at this step
            mask = (kidx[None, :] >= first[rows][:, None]) & (kidx[None, :] <= lim[rows][:, None])
            pO = np.zeros_like(run_O)
            pL = np.full_like(run_L, -np.inf)
            for h in range(Hq):
                g = h // G
                pO[:, h], pL[h] = attend(Qc[rows, h], Ks[:, g], Vs[:, g], mask, sc)
            if partials:
                PO[(r - st) % R, rows] = pO
                PL[(r - st) % R][:, rows] = pL
            mo, ml = lse_merge([run_O, pO], [run_L.T, pL.T])
            run_O, run_L = mo, ml.T
        isb = rows >= S
        if isb.any() and not partials:
            br_rows = rows[isb]
            bid = (br_rows - S) // B
            dep = (br_rows - S) % B
            bO = np.zeros((len(br_rows), Hq, d))
            bL = np.full((Hq, len(br_rows)), -np.inf)
            for n, (bi, t) in enumerate(zip(bid, dep)):
                u = np.arange(B)
                bits = np.asarray(branch_mask, dtype=np.uint64)[bi, t] if mode == BITMASK else None
                m = branch_sees(mode, t, u, bits)[None, :]
                for h in range(Hq):
                    g = h // G
                    o1, l1 = attend(qb[bi, t, h][None, :], kb[bi, :, g], vb[bi, :, g], m, sc)
                    bO[n, h], bL[h, n] = o1[0], l1[0]
            mo, ml = lse_merge([run_O[isb], bO], [run_L[:, isb].T, bL.T])
            run_O[isb] = mo
            run_L[:, isb] = ml.T
        O[rows] = run_O
        L[:, rows] = run_L
    if partials:
        return PO, PL
    om, obr = _split_rows(O, S, Nb, B)
    return om, obr, L


# --------------------------------------------------------------------------
# counting
# --------------------------------------------------------------------------

def visible_pair_count(cu, anchors, B, mode, window=0, branch_mask=None) -> int:
    """Exact number of visible (row, key) pairs per q head, from the
    definition: sum over main rows of (i - s(i) + 1) plus, per branch,
    B * (a_b - s(a_b) + 1) main pairs and B(B+1)/2 (CHAIN), B*B (BLOCK) or the
    set bits of its mask rows (BITMASK) branch pairs.  With a window W > 0 a
    prefix of n keys counts min(n, W)."""
    cu = i64(cu)
    anc = i64(anchors)
    S = int(cu[-1])
    pos = np.arange(S)
    n_main = pos - doc_start_of(cu, pos) + 1
    if window and window > 0:
        n_main = np.minimum(n_main, window)
    main = int(n_main.sum())
    if len(anc) == 0:
        return main
    n_pre = anc - doc_start_of(cu, anc) + 1
    if window and window > 0:
        n_pre = np.minimum(n_pre, window)
    pre = int(n_pre.sum()) * B
    if mode == CHAIN:
        loc = len(anc) * (B * (B + 1) // 2)
    elif mode == BLOCK:
        loc = len(anc) * B * B
    else:
        words = np.asarray(branch_mask, dtype=np.uint64).reshape(-1)
        loc = sum(bin(int(x) & ((1 << B) - 1)).count("1") for x in words)
    return main + pre + loc
