"""Context parallelism across processes, on CPU: gloo ranks run the library's
context-parallel orchestration (zigzag shares, one all-gather of the main K/V,
one all-reduce of the main-key gradients) with the fp64 oracle standing in
for each rank's kernels, and every rank's share of O, LSE, dQ, dK, dV and the
branch-key gradients must equal the single-process oracle's.

The stand-in has the library's cp_rank contract: it computes only its rank's
rows against the full K/V it is given, writes a partial dK/dV for every main
key (its own rows' contributions) and the gradients of its own branches."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleRank:
    """Per-rank compute with the library's cp_rank contract, from the oracle."""

    def __init__(self, cu, anc, B, mode, R, r, window=0, branch_mask=None):
        import oracle as orc
        from branch_attention_speculative_packed_b200.cp import zigzag_rows
        self.orc = orc
        self.cu, self.anc, self.B, self.mode = np.asarray(cu), np.asarray(anc), B, mode
        self.kw = dict(window=window, branch_mask=branch_mask)
        m, b = zigzag_rows(cu, anc, R, r)
        self.S = int(self.cu[-1])
        self.rows = np.concatenate([m.numpy(), (self.S + b.numpy()[:, None] * B + np.arange(B)).reshape(-1)])

    def fused_fwd(self, q, k, v, qb, kb, vb):
        S, Hq, d = q.shape
        Nb = qb.shape[0]
        rows, O, L = self.orc.forward_rows(q, k, v, qb, kb, vb, self.cu, self.anc, self.B, self.mode,
                                           rows=self.rows, **self.kw)
        Ofull = torch.zeros(S + Nb * self.B, Hq, d, dtype=torch.float64)
        Ofull[torch.as_tensor(rows)] = torch.from_numpy(O)
        lse = torch.full((Hq, S + Nb * self.B), float("nan"), dtype=torch.float64)
        lse[:, torch.as_tensor(rows)] = torch.from_numpy(L)
        return Ofull[:S], Ofull[S:].reshape(Nb, self.B, Hq, d), lse

    def bwd(self, q, k, v, qb, kb, vb, o, ob, lse, do, dob):
        S, Hq, d = q.shape
        Nb = qb.shape[0]
        rows, dQ, dk, dv, dkb, dvb = self.orc.backward_rows(q, k, v, qb, kb, vb, do, dob, self.cu, self.anc,
                                                            self.B, self.mode, rows=self.rows, **self.kw)
        dq = torch.zeros(S + Nb * self.B, Hq, d, dtype=torch.float64)
        dq[torch.as_tensor(rows)] = torch.from_numpy(dQ)
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x))
        return dq[:S], t(dk), t(dv), dq[S:].reshape(Nb, self.B, Hq, d), t(dkb), t(dvb)


CASES = {
    # name: (lengths, anchors, Hq, Hkv, d, B, mode, window, bitmask)
    "chain": ([40, 9, 75], "every", 4, 2, 8, 3, 0, 0, False),
    "block_window": ([120, 33], [0, 5, 32, 60, 61, 119, 120, 152], 2, 1, 8, 4, 1, 17, False),
    "bitmask": ([64, 3, 50], [1, 2, 30, 63, 64, 66, 100, 116], 2, 2, 8, 5, 2, 0, True),
}


def _problem(name):
    lengths, anchors, Hq, Hkv, d, B, mode, W, bits = CASES[name]
    S = sum(lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    anc = np.arange(S) if anchors == "every" else np.array(anchors, dtype=np.int64)
    rs = np.random.default_rng(len(name))
    t = lambda *shape: torch.from_numpy(rs.standard_normal(shape))
    Nb = len(anc)
    x = dict(q=t(S, Hq, d), k=t(S, Hkv, d), v=t(S, Hkv, d), qb=t(Nb, B, Hq, d), kb=t(Nb, B, Hkv, d),
             vb=t(Nb, B, Hkv, d), do=t(S, Hq, d), dob=t(Nb, B, Hq, d))
    bm = rs.integers(0, 2 ** B, size=(Nb, B), dtype=np.uint64) if bits else None
    return cu, anc, Hq, Hkv, d, B, mode, W, bm, x


def _worker(rank, world, port, name, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=120))
    try:
        import oracle as orc
        from branch_attention_speculative_packed_b200.cp import ContextParallelBranchAttention
        cu, anc, Hq, Hkv, d, B, mode, W, bm, x = _problem(name)
        local = OracleRank(cu, anc, B, mode, world, rank, W, bm)
        cp = ContextParallelBranchAttention(cu, anc, Hq=Hq, Hkv=Hkv, d=d, B=B, mode=mode, window=W,
                                            branch_mask=bm, device="cpu", local=local)
        m, b = cp.main_pos, cp.branch_ids
        o, ob, lse = cp.forward(x["q"][m], x["k"][m], x["v"][m], x["qb"][b], x["kb"][b], x["vb"][b])
        grads = cp.backward(x["do"][m], x["dob"][b])
        # the single-process oracle over every row
        rows, O, L = orc.forward_rows(x["q"], x["k"], x["v"], x["qb"], x["kb"], x["vb"], cu, anc, B, mode,
                                      window=W, branch_mask=bm)
        _, dQ, dk, dv, dkb, dvb = orc.backward_rows(x["q"], x["k"], x["v"], x["qb"], x["kb"], x["vb"],
                                                    x["do"], x["dob"], cu, anc, B, mode, window=W,
                                                    branch_mask=bm)
        S = int(cu[-1])
        mine = cp.rows.numpy()
        err = 0.0
        err = max(err, np.abs(np.concatenate([o.numpy(), ob.numpy().reshape(-1, Hq, d)]) - O[mine]).max())
        err = max(err, np.abs(lse.numpy() - L[:, mine]).max())
        dq, dkr, dvr, dqb, dkbr, dvbr = (g.numpy() for g in grads)
        err = max(err, np.abs(np.concatenate([dq, dqb.reshape(-1, Hq, d)]) - dQ[mine]).max())
        err = max(err, np.abs(dkr - dk[m.numpy()]).max(), np.abs(dvr - dv[m.numpy()]).max())
        if len(b):
            err = max(err, np.abs(dkbr - dkb[b.numpy()]).max(), np.abs(dvbr - dvb[b.numpy()]).max())
        out.put((rank, float(err), len(mine), int(m.numel())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("name", sorted(CASES))
def test_context_parallel_ranks_match_single_process_oracle(name, world):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, name, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cu, anc, *_ = _problem(name)
    S = int(cu[-1])
    assert sum(r[3] for r in res) == S            # the shares partition the main rows
    for rank, err, n_rows, _ in res:
        assert err < 1e-6, (rank, err)            # fp32 reduction of the key gradients


def test_zigzag_shares_partition_rows_and_branches():
    sys.path.insert(0, ROOT)
    from branch_attention_speculative_packed_b200.cp import zigzag_rows
    cu = np.array([0, 5, 5 + 37, 5 + 37 + 64, 5 + 37 + 64 + 1])
    rs = np.random.default_rng(0)
    anc = np.sort(rs.integers(0, cu[-1], 40))
    for R in (1, 2, 3, 4, 8):
        mains, brs = [], []
        for r in range(R):
            m, b = zigzag_rows(cu, anc, R, r)
            mains.append(m.numpy())
            brs.append(b.numpy())
            owned = set(m.tolist())
            assert all(int(anc[i]) in owned for i in b)        # a branch lives with its anchor
        allm = np.sort(np.concatenate(mains))
        assert (allm == np.arange(cu[-1])).all()               # every main row exactly once
        allb = np.sort(np.concatenate(brs))
        assert (allb == np.arange(len(anc))).all()             # every branch exactly once
