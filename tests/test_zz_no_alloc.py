"""The fused forward for callers that cannot allocate device memory.

Some callers of this library cannot call cudaMalloc or pass a freshly
allocated workspace: a runtime whose allocator owns all device memory and
forbids side allocations, code under a device-memory budget fixed at start-up,
or a caller that must not trigger an allocation's implicit synchronisation
mid-stream.  ba_fused_fwd_noalloc serves them by taking its scratch space (the
plan) from a static device array inside the library.  These tests call it
through the C ABI and check it against ba_fused_fwd, which uses a caller
workspace, on two calls in a row with different problems (the shared array
keeps the first call's contents when the second one runs), and check that a
problem too large for the array is refused before anything is enqueued.

This file is collected last, so a run that stops at the first failure has run
every other test before it; it also passes when run alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import workloads as wl
from gpu_cases import SMALL_CASES, TOL_LSE, TOL_O, attn_for, make_case, max_abs, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ba():
    from branch_attention_speculative_packed_b200 import build
    build.build()
    import branch_attention_speculative_packed_b200 as m
    return m


def _nan_outputs(prob, a):
    c = prob.cfg
    return (torch.full_like(prob.q, float("nan")),
            torch.full((prob.Nb, c.B, c.Hq, c.d), float("nan"), dtype=torch.bfloat16, device="cuda"),
            torch.full((c.Hq, a.rows), float("nan"), dtype=torch.float32, device="cuda"))


def test_noalloc_matches_fused_fwd_two_calls_in_a_row(ba):
    problems = [to_device(make_case(SMALL_CASES[2])),           # block mask, 3 documents, GQA 8/2
                wl.make_problem(1, device="cuda", with_grad_inputs=False)]  # 8K chain, every position
    for prob in problems:
        a = attn_for(prob, ba)
        ref = a.fused_fwd(prob.q, prob.k, prob.v, prob.qb, prob.kb, prob.vb)
        got = a.fused_fwd_noalloc(prob.q, prob.k, prob.v, prob.qb, prob.kb, prob.vb,
                                  out=_nan_outputs(prob, a))
        ba.sync_status()
        for r, g, tol in zip(ref, got, (TOL_O, TOL_O, TOL_LSE)):
            assert bool(torch.isfinite(g.float()).all())
            assert max_abs(g.double().cpu().numpy(), r.double().cpu().numpy()) <= tol


def test_noalloc_refuses_problems_beyond_the_static_array(ba):
    from branch_attention_speculative_packed_b200._abi import BA_ERR_SCRATCH_LIMIT
    S = 1 << 21  # ~16 K row tiles: the plan needs more than 8 MiB
    a = ba.BranchAttention([0, S], [], Hq=1, Hkv=1, d=64, B=1, mode=0, R=1)
    assert a.workspace_size(ba.BA_WS_FWD) > 8 << 20
    t = torch.zeros(16, 1, 64, dtype=torch.bfloat16, device="cuda")  # never read: refused first
    with pytest.raises(ba.BAError) as e:
        a.fused_fwd_noalloc(t, t, t, t, t, t, out=(t, t, torch.zeros(4, device="cuda")))
    assert e.value.status == BA_ERR_SCRATCH_LIMIT
