"""GPU parity of the forward path (steps a2, a3, a4 and the fused kernel)
against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle as orc
import workloads as wl
from gpu_cases import (SMALL_CASES, TOL_LSE, TOL_O, attn_for, config_rows, gather_rows, make_case,
                       max_abs, oracle_fwd, oracle_rows_by_group, to_device)

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


def test_full_rows_bit_identical_across_R(ba):
    """R labels the row tiles with their virtual ranks (the zigzag split) but
    does not change what the full-row forward computes: the tile list, the
    pairs and their order are the same for every R, so the outputs are
    bit-identical.  (The zigzag split itself is checked by the per-rank ring
    partials in test_gpu_variants.py.)"""
    case = ("R_sweep", [700, 301, 5], "rand60", 4, 2, 128, 3, wl.CHAIN, 1)
    cpu = make_case(case)
    rows, O, L = oracle_fwd(cpu)
    prob = to_device(make_case(case))
    ref = None
    for R in (1, 2, 5, 8):
        o, ob, lse = _fused(ba, prob, R)
        if ref is None:
            assert max_abs(gather_rows(o, ob, rows, prob.S), O) <= TOL_O
            assert max_abs(lse.cpu().numpy(), L) <= TOL_LSE
            ref = (o, ob, lse)
        else:
            for x, y in zip((o, ob, lse), ref):
                assert torch.equal(x, y)


def test_fused_fwd_config_tiny(ba):
    cpu = wl.make_problem(0)
    rows, O, L = oracle_fwd(cpu)
    prob = to_device(wl.make_problem(0))
    o, ob, lse = _fused(ba, prob)
    assert max_abs(gather_rows(o, ob, rows, prob.S), O) <= TOL_O
    assert max_abs(lse.cpu().numpy(), L) <= TOL_LSE


@pytest.mark.parametrize("idx", [1, pytest.param(2, marks=pytest.mark.slow)])
def test_fused_fwd_config_full_rows(ba, idx):
    """Configs at 8K (chain) and 32K (block): every row and every query head
    against the oracle."""
    prob = to_device(wl.make_problem(idx, with_grad_inputs=False))
    o, ob, lse = _fused(ba, prob)
    ref = oracle_rows_by_group(prob)
    assert ref["heads"] == list(range(prob.cfg.Hq))
    assert max_abs(gather_rows(o, ob, ref["rows"], prob.S), ref["O"]) <= TOL_O
    assert max_abs(lse.cpu().numpy(), ref["L"]) <= TOL_LSE


@pytest.mark.parametrize("idx", [3, pytest.param(4, marks=pytest.mark.slow)])
def test_fused_fwd_config_sampled_rows(ba, idx):
    """64K and 256K configs: 4096 seeded, stratified rows (plus document ends,
    zigzag chunk edges and anchors at document ends), every query head."""
    prob = wl.make_problem(idx, device="cuda", with_grad_inputs=False)
    o, ob, lse = _fused(ba, prob)
    rows = config_rows(prob, 4096, seed=idx)
    assert len(rows) >= 4096
    ref = oracle_rows_by_group(prob, rows)
    assert ref["heads"] == list(range(prob.cfg.Hq))
    assert max_abs(gather_rows(o, ob, rows, prob.S), ref["O"]) <= TOL_O
    assert max_abs(lse[:, torch.as_tensor(rows, device="cuda")].cpu().numpy(), ref["L"]) <= TOL_LSE
    # every output written (canaries were NaN)
    assert bool(torch.isfinite(lse).all())
    assert bool(torch.isfinite(o.float()).all()) and bool(torch.isfinite(ob.float()).all())
