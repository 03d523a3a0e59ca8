"""Shared helpers of the GPU parity tests (imported by tests/test_gpu_*.py).

Inputs come from the seeded generators in ``workloads``; expected values from
the fp64 oracle only.  Tolerances are the ones the target states for bf16
inputs with fp32 accumulation against the fp64 oracle: max-abs 2e-2 on O,
1e-3 on LSE, 5e-2 on dQ/dK/dV.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as orc
import workloads as wl

TOL_O = 2e-2
TOL_LSE = 1e-3
TOL_GRAD = 5e-2

# small cases: (name, lengths, anchors (list or "every"), Hq, Hkv, d, B, mode, R)
SMALL_CASES = [
    ("tiny_cfg_like", [256], [23, 43, 60, 72, 179, 200, 201, 255], 4, 4, 64, 4, wl.CHAIN, 2),
    ("packed_chain_gqa", [97, 40, 163], "rand40", 4, 2, 128, 3, wl.CHAIN, 3),
    ("packed_block16", [211, 300, 189], "rand30", 8, 2, 128, 16, wl.BLOCK, 4),
    ("single_token", [1], [0], 2, 1, 64, 2, wl.CHAIN, 1),
    ("short_docs_R8", [1, 2, 3, 1, 50, 130], "ends", 4, 4, 128, 3, wl.CHAIN, 8),
    ("no_branches", [513, 255], [], 4, 1, 128, 3, wl.CHAIN, 2),
    ("duplicate_anchors", [300], [0, 0, 17, 17, 17, 299, 299], 2, 2, 128, 5, wl.BLOCK, 2),
    ("every_position_d64", [200, 57], "every", 8, 2, 64, 3, wl.CHAIN, 2),
    ("every_position_d128", [333], "every", 4, 1, 128, 3, wl.CHAIN, 4),
    ("long_doc_multi_tile", [1500], "rand50", 2, 1, 128, 4, wl.CHAIN, 2),
]


def make_case(case, seed=7, device="cpu"):
    name, lengths, anchors, Hq, Hkv, d, B, mode, R = case
    S = sum(lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)])
    g = torch.Generator()
    g.manual_seed(seed)
    if anchors == "every":
        anchors = list(range(S))
    elif anchors == "ends":
        anchors = sorted(set([int(c) - 1 for c in cu[1:]] + [int(c) for c in cu[:-1]]))
    elif isinstance(anchors, str) and anchors.startswith("rand"):
        n = int(anchors[4:])
        anchors = sorted(torch.randperm(S, generator=g)[:n].tolist())
    return wl.make_custom(lengths, anchors, Hq=Hq, Hkv=Hkv, d=d, B=B, mode=mode, seed=seed,
                          device=device, R=R, cfg_name=name)


def attn_for(problem, ba, R=None, **kw):
    """The library's handle for a problem; ``kw``: window, branch_mask."""
    c = problem.cfg
    return ba.BranchAttention(problem.cu_seqlens, problem.anchors, Hq=c.Hq, Hkv=c.Hkv, d=c.d,
                              B=c.B, mode=c.mode, R=c.R if R is None else R, **kw)


def to_device(problem, device="cuda"):
    for f in ("q", "k", "v", "qb", "kb", "vb", "do", "dob"):
        t = getattr(problem, f)
        if t is not None:
            setattr(problem, f, t.to(device))
    return problem


def oracle_fwd(problem, rows=None, heads=None, **kw):
    """(rows, O [n,Hq,d], LSE [Hq,n]) from the fp64 row-set oracle; ``kw``:
    window, branch_mask."""
    c = problem.cfg
    return orc.forward_rows(problem.q, problem.k, problem.v, problem.qb, problem.kb, problem.vb,
                            problem.cu_seqlens.numpy(), problem.anchors.numpy(), c.B, c.mode,
                            rows=rows, heads=heads, **kw)


def gather_rows(o, ob, rows, S):
    """Rows (concatenated order) of the device outputs o [S,H,d], ob [Nb,B,H,d] as fp64 numpy."""
    rows = np.asarray(rows)
    H, d = o.shape[1], o.shape[2]
    obf = ob.reshape(-1, H, d)
    out = np.empty((len(rows), H, d))
    m = rows < S
    if m.any():
        out[m] = o[torch.as_tensor(rows[m], device=o.device)].double().cpu().numpy()
    if (~m).any():
        out[~m] = obf[torch.as_tensor(rows[~m] - S, device=o.device)].double().cpu().numpy()
    return out


def max_abs(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    if a.size == 0:
        return 0.0
    assert np.isfinite(a).all(), "non-finite values in device output"
    return float(np.abs(a - b).max())


def sub_heads(problem, groups):
    """A view of the problem restricted to the listed KV groups (and their G
    query heads), keeping the GQA mapping; tensors stay where they are."""
    c = problem.cfg
    G = c.Hq // c.Hkv
    heads = [g * G + i for g in groups for i in range(G)]
    hq = torch.as_tensor(heads, device=problem.q.device)
    hk = torch.as_tensor(list(groups), device=problem.k.device)
    p = wl.Problem(c, problem.seed, problem.cu_seqlens, problem.anchors,
                   problem.q.index_select(1, hq), problem.k.index_select(1, hk),
                   problem.v.index_select(1, hk), problem.qb.index_select(2, hq),
                   problem.kb.index_select(2, hk), problem.vb.index_select(2, hk),
                   None if problem.do is None else problem.do.index_select(1, hq),
                   None if problem.dob is None else problem.dob.index_select(2, hq))
    return p, heads


def oracle_rows_by_group(problem, rows=None, groups=None, backward=False, **kw):
    """The row-set oracle over the given concatenated rows (default: all) for
    the query heads of every listed KV group (default: all), one thread per
    group.

    Each thread runs the oracle, unchanged, on a view of the problem restricted
    to one KV group (``sub_heads``); numpy's BLAS calls and ufunc loops release
    the GIL, so the groups run side by side (BLAS itself is limited to one
    thread per caller meanwhile).  Inputs may stay on the device: the oracle
    converts only the rows it reads.

    Returns a dict with ``heads`` (query heads, group-major), ``rows``,
    ``O`` [n, len(heads), d] and ``L`` [len(heads), n]; with ``backward`` (dO
    in the problem) also ``dQ`` [n, len(heads), d] and, per listed group in
    that order, the key gradients those rows' dO produce: ``dk``/``dv``
    [S, len(groups), d] and ``dkb``/``dvb`` [Nb, B, len(groups), d]."""
    import os
    from concurrent.futures import ThreadPoolExecutor

    from threadpoolctl import threadpool_limits

    c = problem.cfg
    G = c.Hq // c.Hkv
    groups = list(range(c.Hkv)) if groups is None else list(groups)
    if rows is None:
        rows = np.arange(problem.S + problem.Nb * c.B)
    rows = np.asarray(rows, dtype=np.int64)
    cu, anc = problem.cu_seqlens.numpy(), problem.anchors.numpy()

    def one(g):
        sub, _ = sub_heads(problem, [g])
        args = (sub.q, sub.k, sub.v, sub.qb, sub.kb, sub.vb)
        _, O, L = orc.forward_rows(*args, cu, anc, c.B, c.mode, rows=rows, **kw)
        if not backward:
            return O, L
        _, dQ, dk, dv, dkb, dvb = orc.backward_rows(*args, sub.do, sub.dob, cu, anc, c.B, c.mode,
                                                    rows=rows, **kw)
        return O, L, dQ, dk, dv, dkb, dvb

    workers = max(1, min(len(groups), os.cpu_count() or 1))
    with threadpool_limits(limits=max(1, (os.cpu_count() or 1) // workers)):
        with ThreadPoolExecutor(max_workers=workers) as ex:
            res = list(ex.map(one, groups))
    out = {"heads": [g * G + i for g in groups for i in range(G)], "rows": rows,
           "O": np.concatenate([r[0] for r in res], axis=1),
           "L": np.concatenate([r[1] for r in res], axis=0)}
    if backward:
        out["dQ"] = np.concatenate([r[2] for r in res], axis=1)
        out["dk"] = np.concatenate([r[3] for r in res], axis=1)
        out["dv"] = np.concatenate([r[4] for r in res], axis=1)
        out["dkb"] = np.concatenate([r[5] for r in res], axis=2)
        out["dvb"] = np.concatenate([r[6] for r in res], axis=2)
    return out


def config_rows(problem, n_rows, seed):
    """Seeded, stratified query rows of a large configuration: about half main
    and half branch rows, plus the first and last row of every document, every
    zigzag chunk edge and the branch rows of anchors at document ends."""
    edges = [e[2] for e in orc.zigzag_chunks(problem.cu_seqlens.numpy(), problem.cfg.R)]
    return wl.sample_rows(problem.cu_seqlens, problem.anchors, problem.cfg.B, n_rows, seed=seed,
                          extra=edges).numpy()
