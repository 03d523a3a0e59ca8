"""GPU parity of the backward (dQ, dK, dV through the main-sequence and the
branch-local components) against the fp64 oracle, through the C ABI.

The device backward consumes the device forward's O and LSE (that is the
product path); the oracle recomputes everything from q, k, v and dO alone."""
import numpy as np
import pytest
import torch

import oracle as orc
import workloads as wl
from gpu_cases import (SMALL_CASES, TOL_GRAD, attn_for, config_rows, make_case, max_abs,
                       oracle_rows_by_group, to_device)

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


def test_bwd_branch_rows_exceed_shared_memory(ba):
    """B x G = 32 x 16 at d = 128: a branch's q / dO rows (256 KB) exceed one
    block's shared memory, so the branch-key backward takes its row-load form;
    every gradient matches the oracle.  With 16 query heads per KV head the
    gradients grow past 1, where one bf16 step of the outputs is already more
    than 5e-2, so the 5e-2 bound is scaled by max(1, |reference|)."""
    case = ("wide_group_deep_branch", [211, 120], "rand8", 16, 1, 128, 32, wl.CHAIN, 2)
    cpu = make_case(case)
    c = cpu.cfg
    _, dQ, dk, dv, dkb, dvb = orc.backward_rows(cpu.q, cpu.k, cpu.v, cpu.qb, cpu.kb, cpu.vb, cpu.do,
                                                cpu.dob, cpu.cu_seqlens.numpy(), cpu.anchors.numpy(),
                                                c.B, c.mode)
    prob = to_device(make_case(case))
    dq, dkd, dvd, dqb, dkbd, dvbd = _fwd_bwd(ba, prob)
    S = prob.S

    def within(got, ref):
        got = np.asarray(got, dtype=np.float64).reshape(ref.shape)
        return float(np.max(np.abs(got - ref) / np.maximum(1.0, np.abs(ref)))) <= TOL_GRAD

    assert within(_np(dq), dQ[:S]) and within(_np(dkd), dk) and within(_np(dvd), dv)
    assert within(_np(dqb).reshape(-1, c.Hq, c.d), dQ[S:])
    assert within(_np(dkbd), dkb) and within(_np(dvbd), dvb)


def test_bwd_bit_identical_across_R(ba):
    """The backward does not depend on R (it plans the same tiles for every
    R): gradients for R = 1, 3, 8 are bit-identical and match the oracle."""
    case = ("R_sweep_bwd", [700, 301, 5], "rand60", 4, 2, 128, 3, wl.CHAIN, 1)
    cpu = make_case(case)
    c = cpu.cfg
    _, dQ, dk, dv, dkb, dvb = orc.backward_rows(cpu.q, cpu.k, cpu.v, cpu.qb, cpu.kb, cpu.vb, cpu.do,
                                                cpu.dob, cpu.cu_seqlens.numpy(), cpu.anchors.numpy(),
                                                c.B, c.mode)
    prob = to_device(make_case(case))
    ref = None
    S = prob.S
    for R in (1, 3, 8):
        prob.cfg = wl.Config(**{**c.__dict__, "R": R})
        grads = _fwd_bwd(ba, prob)
        if ref is None:
            dq, dkd, dvd, dqb, dkbd, dvbd = grads
            assert max_abs(_np(dq), dQ[:S]) <= TOL_GRAD
            assert max_abs(_np(dkd), dk) <= TOL_GRAD
            assert max_abs(_np(dvd), dv) <= TOL_GRAD
            assert max_abs(_np(dqb).reshape(-1, c.Hq, c.d), dQ[S:]) <= TOL_GRAD
            ref = grads
        else:
            for x, y in zip(grads, ref):
                assert torch.equal(x, y)


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


@pytest.mark.parametrize("idx", [1, pytest.param(2, marks=pytest.mark.slow)])
def test_bwd_config_full(ba, idx):
    """8K chain and 32K block configs: every row, every key and every head
    against the oracle."""
    prob = wl.make_problem(idx, device="cuda")
    grads = _fwd_bwd(ba, prob)
    for g_ in grads:
        assert bool(torch.isfinite(g_.float()).all())
    _check_invariants(prob, grads)
    ref = oracle_rows_by_group(prob, backward=True)
    c = prob.cfg
    dq, dkd, dvd, dqb, dkbd, dvbd = grads
    S = prob.S
    assert max_abs(_np(dq), ref["dQ"][:S]) <= TOL_GRAD
    assert max_abs(_np(dqb).reshape(-1, c.Hq, c.d), ref["dQ"][S:]) <= TOL_GRAD
    assert max_abs(_np(dkd), ref["dk"]) <= TOL_GRAD
    assert max_abs(_np(dvd), ref["dv"]) <= TOL_GRAD
    assert max_abs(_np(dkbd), ref["dkb"]) <= TOL_GRAD
    assert max_abs(_np(dvbd), ref["dvb"]) <= TOL_GRAD


@pytest.mark.parametrize("idx,group", [(3, 6), pytest.param(4, 1, marks=pytest.mark.slow)])
def test_bwd_config_sampled(ba, idx, group):
    """64K and 256K configs on 4096 seeded, stratified rows.  (1) Full random
    dO: dQ of the sampled rows matches the oracle for every head (a row's dQ
    depends only on that row), and the gradient invariants hold.  (2) dO zero
    outside the sampled rows: then every dK, dV is exactly the oracle's sum
    over those rows, checked for every key of one KV group."""
    prob = wl.make_problem(idx, device="cuda")
    c = prob.cfg
    rows = config_rows(prob, 4096, seed=idx)
    assert len(rows) >= 4096
    S = prob.S
    grads = _fwd_bwd(ba, prob)
    _check_invariants(prob, grads)
    dq_all = torch.cat([grads[0], grads[3].reshape(-1, c.Hq, c.d)])
    got = _np(dq_all[torch.as_tensor(rows, device="cuda")])
    del grads, dq_all
    ref = oracle_rows_by_group(prob, rows, backward=True)
    assert max_abs(got, ref["dQ"]) <= TOL_GRAD
    del ref
    # sparse dO
    mask = torch.zeros(S + prob.Nb * c.B, dtype=torch.bool, device="cuda")
    mask[torch.as_tensor(rows, device="cuda")] = True
    prob.do = prob.do * mask[:S, None, None]
    prob.dob = prob.dob * mask[S:].view(prob.Nb, c.B)[..., None, None]
    grads = _fwd_bwd(ba, prob)
    ref = oracle_rows_by_group(prob, rows, groups=[group], backward=True)
    gi = torch.as_tensor([group], device="cuda")
    assert max_abs(_np(grads[1].index_select(1, gi)), ref["dk"]) <= TOL_GRAD
    assert max_abs(_np(grads[2].index_select(1, gi)), ref["dv"]) <= TOL_GRAD
    assert max_abs(_np(grads[4].index_select(2, gi)), ref["dkb"]) <= TOL_GRAD
    assert max_abs(_np(grads[5].index_select(2, gi)), ref["dvb"]) <= TOL_GRAD
