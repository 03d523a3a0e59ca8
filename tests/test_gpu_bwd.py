"""GPU parity of the backward (dQ, dK, dV through the main-sequence and the
branch-local components) against the fp64 oracle, through the C ABI.

The device backward consumes the device forward's O and LSE (that is the
product path); the oracle recomputes everything from q, k, v and dO alone."""
import numpy as np
import pytest
import torch

import oracle as orc
import workloads as wl
from gpu_cases import (SMALL_CASES, TOL_GRAD, attn_for, make_case, max_abs, sub_heads,
                       to_device)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ba():
    from branch_attention_speculative_packed_b200 import build
    build.build()
    import branch_attention_speculative_packed_b200 as m
    return m


def _fwd_bwd(ba, prob, do=None, dob=None):
    a = attn_for(prob, ba)
    o, ob, lse = a.fused_fwd(prob.q, prob.k, prob.v, prob.qb, prob.kb, prob.vb)
    nan = float("nan")
    out = (torch.full_like(prob.q, nan), torch.full_like(prob.k, nan), torch.full_like(prob.v, nan),
           torch.full_like(prob.qb, nan), torch.full_like(prob.kb, nan), torch.full_like(prob.vb, nan))
    grads = a.bwd(prob.q, prob.k, prob.v, prob.qb, prob.kb, prob.vb, o, ob, lse,
                  prob.do if do is None else do, prob.dob if dob is None else dob, out=out)
    ba.sync_status()
    return grads


def _np(t):
    return t.double().cpu().numpy()


@pytest.mark.parametrize("case", SMALL_CASES, ids=[c[0] for c in SMALL_CASES])
def test_bwd_small(ba, case):
    cpu = make_case(case)
    c = cpu.cfg
    _, dQ, dk, dv, dkb, dvb = orc.backward_rows(cpu.q, cpu.k, cpu.v, cpu.qb, cpu.kb, cpu.vb, cpu.do,
                                                cpu.dob, cpu.cu_seqlens.numpy(), cpu.anchors.numpy(),
                                                c.B, c.mode)
    prob = to_device(make_case(case))
    dq, dkd, dvd, dqb, dkbd, dvbd = _fwd_bwd(ba, prob)
    S = prob.S
    assert max_abs(_np(dq), dQ[:S]) <= TOL_GRAD
    assert max_abs(_np(dkd), dk) <= TOL_GRAD
    assert max_abs(_np(dvd), dv) <= TOL_GRAD
    if prob.Nb:
        assert max_abs(_np(dqb).reshape(-1, c.Hq, c.d), dQ[S:]) <= TOL_GRAD
        assert max_abs(_np(dkbd), dkb) <= TOL_GRAD
        assert max_abs(_np(dvbd), dvb) <= TOL_GRAD


@pytest.mark.parametrize("R", [1, 3, 8])
def test_bwd_independent_of_R(ba, R):
    case = ("R_sweep_bwd", [700, 301, 5], "rand60", 4, 2, 128, 3, wl.CHAIN, R)
    cpu = make_case(case)
    c = cpu.cfg
    _, dQ, dk, dv, dkb, dvb = orc.backward_rows(cpu.q, cpu.k, cpu.v, cpu.qb, cpu.kb, cpu.vb, cpu.do,
                                                cpu.dob, cpu.cu_seqlens.numpy(), cpu.anchors.numpy(),
                                                c.B, c.mode)
    prob = to_device(make_case(case))
    dq, dkd, dvd, dqb, dkbd, dvbd = _fwd_bwd(ba, prob)
    S = prob.S
    assert max_abs(_np(dq), dQ[:S]) <= TOL_GRAD
    assert max_abs(_np(dkd), dk) <= TOL_GRAD
    assert max_abs(_np(dvd), dv) <= TOL_GRAD
    assert max_abs(_np(dqb).reshape(-1, c.Hq, c.d), dQ[S:]) <= TOL_GRAD


def _check_invariants(prob, grads, rel=2e-2):
    """sum_j dV_j = sum over the group's heads and rows of dO; sum_j dK_j = 0."""
    c = prob.cfg
    G = c.Hq // c.Hkv
    dq, dk, dv, dqb, dkb, dvb = grads
    sdv = dv.double().sum(0) + dvb.double().sum((0, 1))           # [Hkv, d]
    do_all = prob.do.double().sum(0) + prob.dob.double().sum((0, 1))  # [Hq, d]
    ref = do_all.view(c.Hkv, G, c.d).sum(1)
    scale = ref.abs().max().item()
    assert (sdv - ref).abs().max().item() <= rel * scale + 1.0
    sdk = dk.double().sum(0) + dkb.double().sum((0, 1))
    mag = dk.double().abs().sum(0).max().item()
    assert sdk.abs().max().item() <= rel * mag + 1e-3


@pytest.mark.parametrize("idx,groups", [(1, [2]), (2, [5])])
def test_bwd_config_full(ba, idx, groups):
    """8K chain and 32K block configs, every row and key, query heads of the
    listed KV groups in the oracle (all heads on the GPU)."""
    prob = wl.make_problem(idx, device="cuda")
    grads = _fwd_bwd(ba, prob)
    for g_ in grads:
        assert bool(torch.isfinite(g_.float()).all())
    _check_invariants(prob, grads)
    sub, heads = sub_heads(prob, groups)
    host = [t.cpu() for t in (sub.q, sub.k, sub.v, sub.qb, sub.kb, sub.vb, sub.do, sub.dob)]
    c = prob.cfg
    _, dQ, dk, dv, dkb, dvb = orc.backward_rows(*host, prob.cu_seqlens.numpy(), prob.anchors.numpy(),
                                                c.B, c.mode)
    dq, dkd, dvd, dqb, dkbd, dvbd = grads
    S = prob.S
    gi = torch.as_tensor(groups, device="cuda")
    hi = torch.as_tensor(heads, device="cuda")
    assert max_abs(_np(dq.index_select(1, hi)), dQ[:S]) <= TOL_GRAD
    assert max_abs(_np(dqb.index_select(2, hi)).reshape(-1, len(heads), c.d), dQ[S:]) <= TOL_GRAD
    assert max_abs(_np(dkd.index_select(1, gi)), dk) <= TOL_GRAD
    assert max_abs(_np(dvd.index_select(1, gi)), dv) <= TOL_GRAD
    assert max_abs(_np(dkbd.index_select(2, gi)), dkb) <= TOL_GRAD
    assert max_abs(_np(dvbd.index_select(2, gi)), dvb) <= TOL_GRAD


@pytest.mark.parametrize("idx,n_rows,groups", [(3, 1024, [6]), (4, 256, [1])])
def test_bwd_config_sampled(ba, idx, n_rows, groups):
    """64K and 256K configs.  (1) Full random dO: dQ of sampled rows matches
    the oracle (a row's dQ depends only on that row), gradient invariants hold.
    (2) dO zero outside the sampled rows: then every dK, dV is exactly the
    oracle's sum over those rows, checked for every key of the listed group."""
    prob = wl.make_problem(idx, device="cuda")
    c = prob.cfg
    edges = [e[2] for e in orc.zigzag_chunks(prob.cu_seqlens.numpy(), c.R)]
    rows = wl.sample_rows(prob.cu_seqlens, prob.anchors, c.B, n_rows, seed=idx, extra=edges).numpy()
    S = prob.S
    grads = _fwd_bwd(ba, prob)
    _check_invariants(prob, grads)
    sub, heads = sub_heads(prob, groups)
    host = [t.cpu() for t in (sub.q, sub.k, sub.v, sub.qb, sub.kb, sub.vb, sub.do, sub.dob)]
    r2, dQ, _, _, _, _ = orc.backward_rows(*host, prob.cu_seqlens.numpy(), prob.anchors.numpy(),
                                           c.B, c.mode, rows=rows)
    hi = torch.as_tensor(heads, device="cuda")
    dq_all = torch.cat([grads[0].index_select(1, hi), grads[3].index_select(2, hi).reshape(-1, len(heads), c.d)])
    assert max_abs(_np(dq_all[torch.as_tensor(r2, device="cuda")]), dQ) <= TOL_GRAD
    del grads
    # sparse dO
    mask = torch.zeros(S + prob.Nb * c.B, dtype=torch.bool, device="cuda")
    mask[torch.as_tensor(rows, device="cuda")] = True
    do = prob.do * mask[:S, None, None]
    dob = prob.dob * mask[S:].view(prob.Nb, c.B)[..., None, None]
    grads = _fwd_bwd(ba, prob, do, dob)
    sub.do = do.index_select(1, hi)
    sub.dob = dob.index_select(2, hi)
    host = [t.cpu() for t in (sub.q, sub.k, sub.v, sub.qb, sub.kb, sub.vb, sub.do, sub.dob)]
    r2, dQ, dk, dv, dkb, dvb = orc.backward_rows(*host, prob.cu_seqlens.numpy(), prob.anchors.numpy(),
                                                 c.B, c.mode, rows=rows)
    gi = torch.as_tensor(groups, device="cuda")
    assert max_abs(_np(grads[1].index_select(1, gi)), dk) <= TOL_GRAD
    assert max_abs(_np(grads[2].index_select(1, gi)), dv) <= TOL_GRAD
    assert max_abs(_np(grads[4].index_select(2, gi)), dkb) <= TOL_GRAD
    assert max_abs(_np(grads[5].index_select(2, gi)), dvb) <= TOL_GRAD
