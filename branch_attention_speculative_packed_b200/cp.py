"""Context parallelism over several GPUs: one process per GPU, torch.distributed.

Paper: §3.2 as described on the rcap.io post and the evolve.pub review (FAQ on
branch attention under context parallelism).  The packed main sequence is
split zigzag-wise over the CP ranks (document [s, s+L) cut into 2R chunks at
s + floor(kL/2R); rank r owns chunks r and 2R-1-r); every rank computes its own
rows -- the main rows of its chunks and the branch rows anchored there --
against their whole causal main prefix, and a branch's K/V never leave the
rank that owns its anchor.

On NVSwitch every GPU reaches every peer at full bandwidth, so the ring's R-1
K/V steps become one all-gather of the main K/V (the exchange volume is the
same, and it does not depend on the number or depth of branches).  Each rank
then runs the library on its rows only (``cp_rank``); the Eq. 2 merge of the
ring steps is the kernels' own online softmax.  In the backward the ranks'
partial main-key gradients are summed with one all-reduce in fp32; query and
branch-key gradients stay on their rank.

Local layout: a rank holds its main rows in position order (``main_pos``)
and its branches in index order (``branch_ids``): q, do [n_main, Hq, d],
k, v [n_main, Hkv, d], qb, dob [n_br, B, Hq, d], kb, vb [n_br, B, Hkv, d].
The library works in the packed (global) row order, so each rank places its
rows into full-size buffers; rows of other ranks are never read there.

``local`` is the per-rank compute: by default the CUDA library
(``BranchAttention(..., R=world, cp_rank=rank)``); anything with the same
``fused_fwd`` / ``bwd`` contract can stand in (the CPU tests use one).
"""
from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist

from .api import BranchAttention


def zigzag_rows(cu_seqlens, anchors, R: int, r: int):
    """(main positions, branch ids) owned by virtual rank r, ascending."""
    cu = np.asarray(torch.as_tensor(cu_seqlens).cpu(), dtype=np.int64)
    anc = np.asarray(torch.as_tensor(anchors).cpu(), dtype=np.int64)
    pos = []
    for di in range(len(cu) - 1):
        s, e = int(cu[di]), int(cu[di + 1])
        L = e - s
        for k in (r, 2 * R - 1 - r):
            pos.append(np.arange(s + (k * L) // (2 * R), s + ((k + 1) * L) // (2 * R), dtype=np.int64))
    main_pos = np.unique(np.concatenate(pos)) if pos else np.zeros(0, np.int64)
    owned = np.zeros(int(cu[-1]), dtype=bool)
    owned[main_pos] = True
    branch_ids = np.nonzero(owned[anc])[0] if len(anc) else np.zeros(0, np.int64)
    return torch.from_numpy(main_pos), torch.from_numpy(branch_ids.astype(np.int64))


class ContextParallelBranchAttention:
    """Branch attention with the packed sequence split over the ranks of
    ``group`` (zigzag, one share per rank)."""

    def __init__(self, cu_seqlens, anchors, *, Hq, Hkv, d, B, mode, group=None, window=0,
                 branch_mask=None, scale=None, device="cuda", local=None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.cu = torch.as_tensor(cu_seqlens, dtype=torch.int32).cpu()
        self.anc = torch.as_tensor(anchors, dtype=torch.int32).cpu()
        self.S = int(self.cu[-1])
        self.Nb = int(self.anc.numel())
        self.Hq, self.Hkv, self.d, self.B = Hq, Hkv, d, B
        self.device = torch.device(device)
        self.local = local if local is not None else BranchAttention(
            self.cu, self.anc, Hq=Hq, Hkv=Hkv, d=d, B=B, mode=mode, R=self.world, scale=scale,
            device=device, window=window, branch_mask=branch_mask, cp_rank=self.rank)
        shares = [zigzag_rows(self.cu, self.anc, self.world, j) for j in range(self.world)]
        self.shares = [(m.to(self.device), b.to(self.device)) for m, b in shares]
        self.main_pos, self.branch_ids = self.shares[self.rank]
        self.n_max = max(int(m.numel()) for m, _ in shares)
        # this rank's rows in the packed row order: main rows, then b-major branch rows
        br_rows = (self.S + self.branch_ids[:, None] * B + torch.arange(B, device=self.device)).reshape(-1)
        self.rows = torch.cat([self.main_pos, br_rows])

    # ------------------------------------------------------------------ exchange
    def gather_main(self, x_local):
        """All-gather of a main-row tensor [n_main, ...] of every rank into the
        full packed tensor [S, ...] (one collective; 16-bit floats move as their
        bytes, which every backend carries)."""
        n = x_local.shape[0]
        raw = x_local.element_size() == 2
        wire = x_local.contiguous().view(torch.uint8) if raw else x_local
        tail = wire.shape[1:]
        buf = wire.new_zeros((self.n_max,) + tuple(tail))
        buf[:n] = wire
        parts = [torch.empty_like(buf) for _ in range(self.world)]
        dist.all_gather(parts, buf, group=self.group)
        full = wire.new_empty((self.S,) + tuple(tail))
        for j, (m, _) in enumerate(self.shares):
            full[m] = parts[j][: m.numel()]
        return full.view(x_local.dtype) if raw else full

    def _full(self, x_local, n_rows, is_branch):
        """Place this rank's rows into a zero-filled full-size buffer."""
        shape = (n_rows,) + tuple(x_local.shape[1:])
        out = x_local.new_zeros(shape)
        out[self.branch_ids if is_branch else self.main_pos] = x_local
        return out

    # ------------------------------------------------------------------ forward / backward
    def forward(self, q, k, v, qb, kb, vb):
        """This rank's rows: (o [n_main,Hq,d], ob [n_br,B,Hq,d], lse fp32
        [Hq, n_main + n_br*B] in the order main rows, then branch rows)."""
        kf, vf = self.gather_main(k), self.gather_main(v)
        qf = self._full(q, self.S, False)
        qbf, kbf, vbf = (self._full(x, self.Nb, True) for x in (qb, kb, vb))
        o, ob, lse = self.local.fused_fwd(qf, kf, vf, qbf, kbf, vbf)
        self._saved = (qf, kf, vf, qbf, kbf, vbf, o, ob, lse)
        return o[self.main_pos], ob[self.branch_ids], lse[:, self.rows]

    def backward(self, do, dob):
        """Gradients of this rank's share: (dq, dk, dv of its main rows; dqb,
        dkb, dvb of its branches), after summing the main-key gradients of all
        ranks."""
        qf, kf, vf, qbf, kbf, vbf, o, ob, lse = self._saved
        dof = self._full(do, self.S, False)
        dobf = self._full(dob, self.Nb, True)
        dq, dk, dv, dqb, dkb, dvb = self.local.bwd(qf, kf, vf, qbf, kbf, vbf, o, ob, lse, dof, dobf)
        dkv = torch.stack([dk.float(), dv.float()])
        dist.all_reduce(dkv, op=dist.ReduceOp.SUM, group=self.group)
        m, b = self.main_pos, self.branch_ids
        return (dq[m], dkv[0][m].to(dk.dtype), dkv[1][m].to(dv.dtype), dqb[b], dkb[b], dvb[b])
