"""GPU parity of the forward path (steps a2, a3, a4 and the fused kernel)
against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle as orc
import workloads as wl
from gpu_cases import (SMALL_CASES, TOL_LSE, TOL_O, attn_for, gather_rows, make_case, max_abs,
                       oracle_fwd, sub_heads, to_device)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ba():
    from branch_attention_speculative_packed_b200 import build
    build.build()
    import branch_attention_speculative_packed_b200 as m
    return m


def _fused(ba, prob, R=None):
    a = attn_for(prob, ba, R)
    S, Nb, c = prob.S, prob.Nb, prob.cfg
    o = torch.full_like(prob.q, float("nan"))
    ob = torch.full((Nb, c.B, c.Hq, c.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((c.Hq, a.rows), float("nan"), dtype=torch.float32, device="cuda")
    a.fused_fwd(prob.q, prob.k, prob.v, prob.qb, prob.kb, prob.vb, out=(o, ob, lse))
    ba.sync_status()
    return o, ob, lse


@pytest.mark.parametrize("case", SMALL_CASES, ids=[c[0] for c in SMALL_CASES])
def test_fused_fwd_small(ba, case):
    cpu = make_case(case)
    rows, O, L = oracle_fwd(cpu)
    prob = to_device(make_case(case))
    o, ob, lse = _fused(ba, prob)
    got = gather_rows(o, ob, rows, prob.S)
    assert max_abs(got, O) <= TOL_O
    assert max_abs(lse.cpu().numpy()[:, rows], L) <= TOL_LSE


@pytest.mark.parametrize("case", SMALL_CASES[:6], ids=[c[0] for c in SMALL_CASES[:6]])
def test_main_and_branch_parts_and_merge(ba, case):
    cpu = make_case(case)
    c = cpu.cfg
    Om, Lm = orc.main_part(cpu.q, cpu.k, cpu.v, cpu.qb, cpu.cu_seqlens.numpy(), cpu.anchors.numpy(), c.B)
    prob = to_device(make_case(case))
    a = attn_for(prob, ba)
    om, lm = a.main_fwd(prob.q, prob.k, prob.v, prob.qb, prob.kb, prob.vb)
    ba.sync_status()
    assert max_abs(om.cpu().numpy(), Om) <= TOL_O
    assert max_abs(lm.cpu().numpy(), Lm) <= TOL_LSE
    if prob.Nb == 0:
        return
    Obr, Lbr = orc.branch_part(cpu.qb, cpu.kb, cpu.vb, c.B, c.mode)
    obr, lbr = a.branch_fwd(prob.q, prob.k, prob.v, prob.qb, prob.kb, prob.vb)
    ba.sync_status()
    assert max_abs(obr.cpu().numpy(), Obr) <= TOL_O
    assert max_abs(lbr.cpu().numpy(), Lbr) <= TOL_LSE
    # Eq. 2 on the device over the two device partials of the branch rows
    S = prob.S
    mo, ml = ba.lse_merge([om[S:], obr], [lm[:, S:], lbr])
    ba.sync_status()
    rows, O, L = oracle_fwd(cpu)
    assert max_abs(mo.double().cpu().numpy(), O[S:]) <= TOL_O
    assert max_abs(ml.cpu().numpy(), L[:, S:]) <= TOL_LSE


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("k", [1, 2, 3, 7])
def test_lse_merge_random_partials(ba, d, k):
    rs = np.random.default_rng(100 * k + d)
    rows, H = 1000 + k, 3
    O = [rs.standard_normal((rows, H, d)).astype(np.float32) for _ in range(k)]
    L = [rs.standard_normal((H, rows)).astype(np.float32) * 3 for _ in range(k)]
    for p in range(k):  # some empty partials, and some rows empty everywhere
        L[p][:, rs.random(rows) < 0.2] = -np.inf
    for p in range(k):
        L[p][:, :5] = -np.inf
        O[p][:5] = 0.0
    eo, el = orc.lse_merge([o for o in O], [l.T for l in L])
    do_ = [torch.from_numpy(o).cuda() for o in O]
    dl = [torch.from_numpy(l).cuda() for l in L]
    mo, ml = ba.lse_merge(do_, dl)
    ba.sync_status()
    assert max_abs(mo.double().cpu().numpy(), eo) <= 1e-2 * max(1.0, np.abs(eo).max())
    got_l = ml.cpu().numpy().T
    fin = np.isfinite(el)
    assert (np.isneginf(got_l) == ~fin).all()
    assert np.abs(got_l[fin] - el[fin]).max() <= TOL_LSE


def test_lse_merge_rejects_bad_args(ba):
    x = torch.zeros(10, 2, 128, device="cuda")
    l = torch.zeros(2, 10, device="cuda")
    with pytest.raises(ba.BAError):
        ba.lse_merge([x] * 17, [l] * 17)
    with pytest.raises(ba.BAError):
        ba.lse_merge([torch.zeros(10, 2, 96, device="cuda")], [l])


@pytest.mark.parametrize("R", [1, 2, 5, 8])
def test_result_independent_of_R(ba, R):
    case = ("R_sweep", [700, 301, 5], "rand60", 4, 2, 128, 3, wl.CHAIN, R)
    cpu = make_case(case)
    rows, O, L = oracle_fwd(cpu)
    prob = to_device(make_case(case))
    o, ob, lse = _fused(ba, prob)
    assert max_abs(gather_rows(o, ob, rows, prob.S), O) <= TOL_O
    assert max_abs(lse.cpu().numpy(), L) <= TOL_LSE


def test_fused_fwd_config_tiny(ba):
    cpu = wl.make_problem(0)
    rows, O, L = oracle_fwd(cpu)
    prob = to_device(wl.make_problem(0))
    o, ob, lse = _fused(ba, prob)
    assert max_abs(gather_rows(o, ob, rows, prob.S), O) <= TOL_O
    assert max_abs(lse.cpu().numpy(), L) <= TOL_LSE


@pytest.mark.parametrize("idx,groups", [(1, [0, 5]), (2, [3])])
def test_fused_fwd_config_full_rows(ba, idx, groups):
    """Configs at 8K (chain) and 32K (block): every row, the query heads of
    the listed KV groups (the oracle's cost), all heads computed on the GPU."""
    prob = to_device(wl.make_problem(idx))
    o, ob, lse = _fused(ba, prob)
    assert torch.isfinite(o.float()).all() and torch.isfinite(ob.float()).all()
    assert torch.isfinite(lse).all()
    sub, heads = sub_heads(prob, groups)
    cpu_sub = wl.Problem(sub.cfg, sub.seed, sub.cu_seqlens, sub.anchors,
                         *(t.cpu() for t in (sub.q, sub.k, sub.v, sub.qb, sub.kb, sub.vb)))
    c = prob.cfg
    rows, O, L = orc.forward_rows(cpu_sub.q, cpu_sub.k, cpu_sub.v, cpu_sub.qb, cpu_sub.kb, cpu_sub.vb,
                                  prob.cu_seqlens.numpy(), prob.anchors.numpy(), c.B, c.mode)
    got = gather_rows(o[:, heads], ob[:, :, heads], rows, prob.S)
    assert max_abs(got, O) <= TOL_O
    assert max_abs(lse[heads].cpu().numpy(), L) <= TOL_LSE


@pytest.mark.parametrize("idx,n_rows,groups", [(3, 2048, [0, 7]), (4, 512, [2])])
def test_fused_fwd_config_sampled_rows(ba, idx, n_rows, groups):
    """64K and 256K configs: seeded, stratified sample of rows (document ends,
    zigzag chunk edges, anchors at document ends), heads of the listed groups."""
    prob = wl.make_problem(idx, device="cuda", with_grad_inputs=False)
    o, ob, lse = _fused(ba, prob)
    c = prob.cfg
    edges = [e[2] for e in orc.zigzag_chunks(prob.cu_seqlens.numpy(), c.R)]
    rows = wl.sample_rows(prob.cu_seqlens, prob.anchors, c.B, n_rows, seed=idx, extra=edges).numpy()
    sub, heads = sub_heads(prob, groups)
    host = [t.cpu() for t in (sub.q, sub.k, sub.v, sub.qb, sub.kb, sub.vb)]
    r2, O, L = orc.forward_rows(*host, prob.cu_seqlens.numpy(), prob.anchors.numpy(), c.B, c.mode,
                                rows=rows)
    got = gather_rows(o[:, heads], ob[:, :, heads], r2, prob.S)
    assert max_abs(got, O) <= TOL_O
    assert max_abs(lse[heads][:, torch.as_tensor(r2, device="cuda")].cpu().numpy(), L) <= TOL_LSE
    # every output written (canaries were NaN)
    assert bool(torch.isfinite(lse).all())
