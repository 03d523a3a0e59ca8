"""Failure detection on the GPU without a GPU fault.

Every wait inside the library's kernels is bounded.  These tests make waits
expire on purpose -- a one-thread check waiting on a barrier that nothing
arrives on, then the real forward and backward kernels run with a wait limit
of a few hundred cycles -- and check that the library reports BA_ERR_TIMEOUT
with a decodable error word, that the context stays usable and that the next
ordinary call gives correct results.  Nothing here traps, asserts on the
device or touches a bad address."""
import pytest
import torch

import oracle as orc
from gpu_cases import (SMALL_CASES, TOL_GRAD, TOL_LSE, TOL_O, attn_for, gather_rows, make_case,
                       max_abs, oracle_fwd, to_device)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ba():
    from branch_attention_speculative_packed_b200 import build
    build.build()
    import branch_attention_speculative_packed_b200 as m
    return m


def _expect_timeout(ba):
    from branch_attention_speculative_packed_b200._abi import BA_ERR_TIMEOUT
    with pytest.raises(ba.BAError) as e:
        ba.sync_status()
    assert e.value.status == BA_ERR_TIMEOUT
    return ba.error_word_fields(int(ba.lib().ba_last_error_word()))


def test_bounded_wait_on_a_barrier_nothing_sets(ba):
    ba.sync_status()
    ba.set_wait_limit(2000)
    try:
        stream = torch.cuda.current_stream()
        import ctypes
        assert ba.lib().ba_check_bounded_wait(ctypes.c_void_p(stream.cuda_stream)) == 0
        f = _expect_timeout(ba)
        assert f == {"expired": True, "kernel": 4, "role": 0, "site": 1, "parity": 0}
    finally:
        ba.set_wait_limit(0)
    ba.sync_status()  # the word was cleared by the report


def test_short_wait_limit_aborts_the_kernels_and_the_next_call_is_right(ba):
    case = SMALL_CASES[1]
    cpu = make_case(case)
    prob = to_device(make_case(case))
    a = attn_for(prob, ba)
    ba.sync_status()
    ba.set_wait_limit(300)
    try:
        o, ob, lse = a.fused_fwd(prob.q, prob.k, prob.v, prob.qb, prob.kb, prob.vb)
        a.bwd(prob.q, prob.k, prob.v, prob.qb, prob.kb, prob.vb, o, ob, lse, prob.do, prob.dob)
        f = _expect_timeout(ba)
    finally:
        ba.set_wait_limit(0)
    assert f["expired"] and f["kernel"] in (1, 2, 3) and f["role"] in (0, 1, 2)
    # the context is usable and an ordinary call is correct
    o, ob, lse = a.fused_fwd(prob.q, prob.k, prob.v, prob.qb, prob.kb, prob.vb)
    grads = a.bwd(prob.q, prob.k, prob.v, prob.qb, prob.kb, prob.vb, o, ob, lse, prob.do, prob.dob)
    ba.sync_status()
    rows, O, L = oracle_fwd(cpu)
    assert max_abs(gather_rows(o, ob, rows, prob.S), O) <= TOL_O
    assert max_abs(lse.cpu().numpy(), L) <= TOL_LSE
    c = cpu.cfg
    _, dQ, dk, dv, dkb, dvb = orc.backward_rows(cpu.q, cpu.k, cpu.v, cpu.qb, cpu.kb, cpu.vb, cpu.do,
                                                cpu.dob, cpu.cu_seqlens.numpy(), cpu.anchors.numpy(),
                                                c.B, c.mode)
    S = prob.S
    assert max_abs(grads[0].double().cpu().numpy(), dQ[:S]) <= TOL_GRAD
    assert max_abs(grads[1].double().cpu().numpy(), dk) <= TOL_GRAD
    assert max_abs(grads[2].double().cpu().numpy(), dv) <= TOL_GRAD
    assert max_abs(grads[4].double().cpu().numpy(), dkb) <= TOL_GRAD
