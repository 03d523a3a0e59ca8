"""GPU parity, through the C ABI, of the mask variants (main-prefix window,
per-branch bitmask) and of the per-virtual-rank ring partials of the main
component, against the fp64 oracle.

The ring-partial tests are where the zigzag split shows on the GPU: partial k
of a row must hold exactly the visible keys of virtual rank k's chunks, so a
wrong chunk edge moves keys between partials and fails element by element;
merged with the library's own Eq. 2 kernel the partials must give the main
component."""
import numpy as np
import pytest
import torch

import oracle as orc
import workloads as wl
from gpu_cases import (SMALL_CASES, TOL_GRAD, TOL_LSE, TOL_O, attn_for, gather_rows, make_case,
                       max_abs, oracle_fwd, oracle_rows_by_group, to_device)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ba():
    from branch_attention_speculative_packed_b200 import build
    build.build()
    import branch_attention_speculative_packed_b200 as m
    return m


def _np(t):
    return t.double().cpu().numpy()


def _fwd_bwd(ba, prob, **kw):
    a = attn_for(prob, ba, **kw)
    c = prob.cfg
    nan = float("nan")
    o = torch.full_like(prob.q, nan)
    ob = torch.full((prob.Nb, c.B, c.Hq, c.d), nan, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((c.Hq, a.rows), nan, dtype=torch.float32, device="cuda")
    a.fused_fwd(prob.q, prob.k, prob.v, prob.qb, prob.kb, prob.vb, out=(o, ob, lse))
    out = tuple(torch.full_like(t, nan) for t in (prob.q, prob.k, prob.v, prob.qb, prob.kb, prob.vb))
    grads = a.bwd(prob.q, prob.k, prob.v, prob.qb, prob.kb, prob.vb, o, ob, lse, prob.do, prob.dob,
                  out=out)
    ba.sync_status()
    return (o, ob, lse), grads


def _check_against_oracle(cpu, prob, fwd, grads, **kw):
    c = cpu.cfg
    S = cpu.S
    rows, O, L = oracle_fwd(cpu, **kw)
    o, ob, lse = fwd
    assert max_abs(gather_rows(o, ob, rows, S), O) <= TOL_O
    assert max_abs(lse.cpu().numpy(), L) <= TOL_LSE
    _, dQ, dk, dv, dkb, dvb = orc.backward_rows(cpu.q, cpu.k, cpu.v, cpu.qb, cpu.kb, cpu.vb, cpu.do,
                                                cpu.dob, cpu.cu_seqlens.numpy(), cpu.anchors.numpy(),
                                                c.B, c.mode, **kw)
    dq, dkd, dvd, dqb, dkbd, dvbd = grads
    assert max_abs(_np(dq), dQ[:S]) <= TOL_GRAD
    assert max_abs(_np(dkd), dk) <= TOL_GRAD
    assert max_abs(_np(dvd), dv) <= TOL_GRAD
    if cpu.Nb:
        assert max_abs(_np(dqb).reshape(-1, c.Hq, c.d), dQ[S:]) <= TOL_GRAD
        assert max_abs(_np(dkbd), dkb) <= TOL_GRAD
        assert max_abs(_np(dvbd), dvb) <= TOL_GRAD


# --------------------------------------------------------------------------- window

WINDOW_CASES = [(1, 1), (1, 9), (1, 100), (1, 1000), (2, 37), (4, 3), (7, 16), (9, 130), (9, 400)]


@pytest.mark.parametrize("idx,W", WINDOW_CASES,
                         ids=[f"{SMALL_CASES[i][0]}-W{W}" for i, W in WINDOW_CASES])
def test_window_fwd_bwd_small(ba, idx, W):
    cpu = make_case(SMALL_CASES[idx])
    prob = to_device(make_case(SMALL_CASES[idx]))
    fwd, grads = _fwd_bwd(ba, prob, window=W)
    _check_against_oracle(cpu, prob, fwd, grads, window=W)


def test_window_8k_config_w1024(ba):
    """The 8K EAGLE-3 configuration with a 1024-key window: every row, key and
    head, forward and backward."""
    W = 1024
    prob = wl.make_problem(1, device="cuda")
    (o, ob, lse), grads = _fwd_bwd(ba, prob, window=W)
    ref = oracle_rows_by_group(prob, backward=True, window=W)
    c = prob.cfg
    S = prob.S
    assert max_abs(gather_rows(o, ob, ref["rows"], S), ref["O"]) <= TOL_O
    assert max_abs(lse.cpu().numpy(), ref["L"]) <= TOL_LSE
    dq, dkd, dvd, dqb, dkbd, dvbd = grads
    assert max_abs(_np(dq), ref["dQ"][:S]) <= TOL_GRAD
    assert max_abs(_np(dqb).reshape(-1, c.Hq, c.d), ref["dQ"][S:]) <= TOL_GRAD
    assert max_abs(_np(dkd), ref["dk"]) <= TOL_GRAD
    assert max_abs(_np(dvd), ref["dv"]) <= TOL_GRAD
    assert max_abs(_np(dkbd), ref["dkb"]) <= TOL_GRAD
    assert max_abs(_np(dvbd), ref["dvb"]) <= TOL_GRAD


# --------------------------------------------------------------------------- bitmask

def _mask_words(seed, Nb, B):
    """Seeded per-branch mask words (bit u of word [b, t]: row t sees key u),
    with a few rows that see no branch key and a few that see them all."""
    rs = np.random.default_rng(seed)
    bits = rs.random((Nb, B, B)) < 0.5
    w = np.zeros((Nb, B), dtype=np.uint64)
    for u in range(B):
        w |= bits[:, :, u].astype(np.uint64) << np.uint64(u)
    if Nb:
        w[0, :] = 0
        w[-1, :] = np.uint64((1 << B) - 1)
    return w


BITMASK_CASES = [
    ("bitmask_chainlike", [97, 40, 163], "rand40", 4, 2, 128, 3, 2, 3),
    ("bitmask_block16", [211, 300, 189], "rand30", 8, 2, 128, 16, 2, 4),
    ("bitmask_b33_d64", [400, 77], "rand12", 4, 1, 64, 33, 2, 2),
    ("bitmask_every_position", [333], "every", 4, 1, 128, 3, 2, 4),
]


@pytest.mark.parametrize("case", BITMASK_CASES, ids=[c[0] for c in BITMASK_CASES])
def test_bitmask_fwd_bwd_and_branch_part(ba, case):
    cpu = make_case(case)
    c = cpu.cfg
    words = _mask_words(len(case[0]), cpu.Nb, c.B)
    prob = to_device(make_case(case))
    fwd, grads = _fwd_bwd(ba, prob, branch_mask=words)
    _check_against_oracle(cpu, prob, fwd, grads, branch_mask=words)
    # the standalone branch-local component (step a3) under the same words
    Obr, Lbr = orc.branch_part(cpu.qb, cpu.kb, cpu.vb, c.B, c.mode, branch_mask=words)
    a = attn_for(prob, ba, branch_mask=words)
    obr, lbr = a.branch_fwd(prob.q, prob.k, prob.v, prob.qb, prob.kb, prob.vb)
    ba.sync_status()
    assert max_abs(obr.cpu().numpy(), Obr) <= TOL_O
    got, exp = lbr.cpu().numpy(), Lbr
    assert (np.isneginf(got) == np.isneginf(exp)).all()
    fin = np.isfinite(exp)
    assert np.abs(got[fin] - exp[fin]).max() <= TOL_LSE


def test_bitmask_with_window(ba):
    """Both variants at once: mask words on the branch keys, a window on the
    main prefix."""
    case = BITMASK_CASES[1]
    cpu = make_case(case)
    words = _mask_words(7, cpu.Nb, cpu.cfg.B)
    prob = to_device(make_case(case))
    fwd, grads = _fwd_bwd(ba, prob, branch_mask=words, window=45)
    _check_against_oracle(cpu, prob, fwd, grads, branch_mask=words, window=45)


# --------------------------------------------------------------------------- ring partials

RING_CASES = [(0, 1, 0), (0, 2, 0), (1, 3, 0), (2, 4, 0), (4, 8, 0), (9, 5, 0), (9, 2, 200),
              (8, 7, 0), (5, 3, 0)]


@pytest.mark.parametrize("idx,R,W", RING_CASES,
                         ids=[f"{SMALL_CASES[i][0]}-R{R}-W{W}" for i, R, W in RING_CASES])
def test_ring_partials_match_oracle_and_merge(ba, idx, R, W):
    cpu = make_case(SMALL_CASES[idx])
    c = cpu.cfg
    cu, anc = cpu.cu_seqlens.numpy(), cpu.anchors.numpy()
    PO, PL = orc.forward_ring(cpu.q, cpu.k, cpu.v, cpu.qb, cpu.kb, cpu.vb, cu, anc, c.B, c.mode, R=R,
                              window=W, partials=True)
    prob = to_device(make_case(SMALL_CASES[idx]))
    a = attn_for(prob, ba, R=R, window=W)
    o, l = a.main_fwd_ring(prob.q, prob.k, prob.v, prob.qb, prob.kb, prob.vb)
    ba.sync_status()
    assert max_abs(o.cpu().numpy(), PO) <= TOL_O
    got = l.cpu().numpy()
    assert (np.isneginf(got) == np.isneginf(PL)).all(), "empty partials differ"
    fin = np.isfinite(PL)
    assert np.abs(got[fin] - PL[fin]).max() <= TOL_LSE
    # Eq. 2 over the R partials on the device = the main component
    Om, Lm = orc.main_part(cpu.q, cpu.k, cpu.v, cpu.qb, cu, anc, c.B, window=W)
    mo, ml = ba.lse_merge([o[k] for k in range(R)], [l[k] for k in range(R)])
    ba.sync_status()
    assert max_abs(mo.double().cpu().numpy(), Om) <= TOL_O
    assert max_abs(ml.cpu().numpy(), Lm) <= TOL_LSE


# --------------------------------------------------------------------------- one rank's rows

CP_CASES = [(1, 3, 0), (2, 4, 0), (4, 8, 0), (9, 2, 0), (7, 5, 0), (9, 3, 150)]


@pytest.mark.parametrize("idx,R,W", CP_CASES, ids=[f"{SMALL_CASES[i][0]}-R{R}-W{W}" for i, R, W in CP_CASES])
def test_one_rank_rows_assemble_the_whole_problem(ba, idx, R, W):
    """Context parallelism emulated on one GPU: each virtual rank r computes
    only its zigzag rows (cp_rank = r) against the full K/V; the union of the
    ranks' rows and the sum of their partial main-key gradients must equal the
    oracle's forward and backward of the whole problem.  The ranks run one
    after another: no kernel waits on another."""
    from branch_attention_speculative_packed_b200.cp import zigzag_rows
    cpu = make_case(SMALL_CASES[idx])
    c = cpu.cfg
    cu, anc = cpu.cu_seqlens.numpy(), cpu.anchors.numpy()
    prob = to_device(make_case(SMALL_CASES[idx]))
    S, Nb, B = prob.S, prob.Nb, c.B
    nan = float("nan")
    o_all = torch.full_like(prob.q, nan)
    ob_all = torch.full((Nb, B, c.Hq, c.d), nan, dtype=torch.bfloat16, device="cuda")
    lse_all = torch.full((c.Hq, S + Nb * B), nan, dtype=torch.float32, device="cuda")
    dq_all, dqb_all = torch.full_like(prob.q, nan), torch.full_like(prob.qb, nan)
    dkb_all, dvb_all = torch.full_like(prob.kb, nan), torch.full_like(prob.vb, nan)
    dk_sum = torch.zeros(prob.k.shape, dtype=torch.float32, device="cuda")
    dv_sum = torch.zeros_like(dk_sum)
    for r in range(R):
        m, b = (t.cuda() for t in zigzag_rows(cu, anc, R, r))
        rows = torch.cat([m, (S + b[:, None] * B + torch.arange(B, device="cuda")).reshape(-1)])
        a = attn_for(prob, ba, R=R, cp_rank=r, window=W)
        o, ob, lse = a.fused_fwd(prob.q, prob.k, prob.v, prob.qb, prob.kb, prob.vb)
        g = a.bwd(prob.q, prob.k, prob.v, prob.qb, prob.kb, prob.vb, o, ob, lse, prob.do, prob.dob)
        ba.sync_status()
        o_all[m], ob_all[b], lse_all[:, rows] = o[m], ob[b], lse[:, rows]
        dq_all[m], dqb_all[b], dkb_all[b], dvb_all[b] = g[0][m], g[3][b], g[4][b], g[5][b]
        dk_sum += g[1].float()
        dv_sum += g[2].float()
    rows, O, L = oracle_fwd(cpu, window=W)
    assert max_abs(gather_rows(o_all, ob_all, rows, S), O) <= TOL_O
    assert max_abs(lse_all.cpu().numpy(), L) <= TOL_LSE
    _, dQ, dk, dv, dkb, dvb = orc.backward_rows(cpu.q, cpu.k, cpu.v, cpu.qb, cpu.kb, cpu.vb, cpu.do,
                                                cpu.dob, cu, anc, B, c.mode, window=W)
    assert max_abs(_np(dq_all), dQ[:S]) <= TOL_GRAD
    assert max_abs(dk_sum.double().cpu().numpy(), dk) <= TOL_GRAD
    assert max_abs(dv_sum.double().cpu().numpy(), dv) <= TOL_GRAD
    if Nb:
        assert max_abs(_np(dqb_all).reshape(-1, c.Hq, c.d), dQ[S:]) <= TOL_GRAD
        assert max_abs(_np(dkb_all), dkb) <= TOL_GRAD
        assert max_abs(_np(dvb_all), dvb) <= TOL_GRAD


# --------------------------------------------------------------------------- context parallelism over NCCL

def _cp_worker(port, out):
    import os
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    import torch.distributed as dist
    try:
        torch.cuda.set_device(0)
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                                timeout=__import__("datetime").timedelta(seconds=120))
        from branch_attention_speculative_packed_b200.cp import ContextParallelBranchAttention
        cpu = make_case(SMALL_CASES[1])
        c = cpu.cfg
        prob = to_device(make_case(SMALL_CASES[1]))
        cp = ContextParallelBranchAttention(prob.cu_seqlens, prob.anchors, Hq=c.Hq, Hkv=c.Hkv, d=c.d, B=c.B,
                                            mode=c.mode, device="cuda")
        m, b = cp.main_pos, cp.branch_ids
        o, ob, lse = cp.forward(prob.q[m], prob.k[m], prob.v[m], prob.qb[b], prob.kb[b], prob.vb[b])
        g = cp.backward(prob.do[m], prob.dob[b])
        torch.cuda.synchronize()
        rows, O, L = oracle_fwd(cpu)
        S = prob.S
        err_o = max_abs(gather_rows(o, ob, rows, S), O)
        err_l = max_abs(lse.cpu().numpy(), L)
        _, dQ, dk, dv, dkb, dvb = orc.backward_rows(cpu.q, cpu.k, cpu.v, cpu.qb, cpu.kb, cpu.vb, cpu.do,
                                                    cpu.dob, cpu.cu_seqlens.numpy(), cpu.anchors.numpy(),
                                                    c.B, c.mode)
        err_g = max(max_abs(_np(g[0]), dQ[:S]), max_abs(_np(g[1]), dk), max_abs(_np(g[2]), dv),
                    max_abs(_np(g[3]).reshape(-1, c.Hq, c.d), dQ[S:]), max_abs(_np(g[4]), dkb),
                    max_abs(_np(g[5]), dvb))
        dist.destroy_process_group()
        out.put((err_o, err_l, err_g))
    except Exception as e:
        out.put(repr(e))


def test_context_parallel_driver_over_nccl_one_rank():
    """The context-parallel driver end to end with NCCL and the CUDA kernels on
    a one-rank group (this pool gives one GPU per call): the all-gather and the
    all-reduce run through NCCL, the kernels through cp_rank = 0, and the
    result matches the oracle.  Multi-rank runs are covered by the gloo tests
    on CPU."""
    import socket
    import torch.multiprocessing as mp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    p = ctx.Process(target=_cp_worker, args=(port, out))
    p.start()
    res = out.get(timeout=300)
    p.join(timeout=60)
    assert not isinstance(res, str), res
    err_o, err_l, err_g = res
    assert err_o <= TOL_O and err_l <= TOL_LSE and err_g <= TOL_GRAD, res
