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


def attn_for(problem, ba, R=None):
    c = problem.cfg
    return ba.BranchAttention(problem.cu_seqlens, problem.anchors, Hq=c.Hq, Hkv=c.Hkv, d=c.d,
                              B=c.B, mode=c.mode, R=c.R if R is None else R)


def to_device(problem, device="cuda"):
    for f in ("q", "k", "v", "qb", "kb", "vb", "do", "dob"):
        t = getattr(problem, f)
        if t is not None:
            setattr(problem, f, t.to(device))
    return problem


def oracle_fwd(problem, rows=None, heads=None):
    """(rows, O [n,Hq,d], LSE [Hq,n]) from the fp64 row-set oracle."""
    c = problem.cfg
    return orc.forward_rows(problem.q, problem.k, problem.v, problem.qb, problem.kb, problem.vb,
                            problem.cu_seqlens.numpy(), problem.anchors.numpy(), c.B, c.mode,
                            rows=rows, heads=heads)


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
