"""The TapChannel-style mailbox across processes: sources write taps with
sequence stamps into the draft stage's slots, the owner waits, reads and
releases them in order, a source cannot overwrite a tap that was not
released, and every wait is bounded (a stamp that never comes raises
TimeoutError).  On CPU with shared memory; on the GPU with CUDA IPC and peer
copies (host polling only: no kernel waits on another process)."""
import os
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

N_MB = 6
SHAPE = (64, 33)


def _tap(src, mb, device):
    g = torch.Generator(device="cpu").manual_seed(1000 * src + mb)
    return torch.randn(SHAPE, generator=g).to(torch.bfloat16).to(device)


def _source(handle, src, device, errq):
    sys.path.insert(0, ROOT)
    try:
        from branch_attention_speculative_packed_b200.tapchannel import TapWriter
        w = TapWriter(handle, src)
        for mb in range(1, N_MB + 1):
            w.write(_tap(src, mb, device), mb, timeout_s=60)
        del w, handle  # drop the mapped slots before telling the owner we are done
        errq.put((src, None))
    except Exception as e:  # reported to the owner
        errq.put((src, repr(e)))


def _run(device):
    sys.path.insert(0, ROOT)
    from branch_attention_speculative_packed_b200.tapchannel import TapMailbox
    ctx = mp.get_context("spawn")
    box = TapMailbox(2, SHAPE, dtype=torch.bfloat16, device=device)
    errq = ctx.Queue()
    procs = [ctx.Process(target=_source, args=(box.handle(), s, device, errq)) for s in range(2)]
    for p in procs:
        p.start()
    try:
        for mb in range(1, N_MB + 1):
            for s in (1, 0):  # the draft stage reads its sources in any order
                got = box.wait_and_read(s, mb, timeout_s=60).clone()
                assert torch.equal(got.cpu(), _tap(s, mb, "cpu")), (s, mb)
                box.release(s, mb)
        errs = sorted(errq.get(timeout=60) for _ in range(2))
        assert errs == [(0, None), (1, None)], errs
    finally:
        for p in procs:
            p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs)


def test_mailbox_across_processes_cpu():
    _run("cpu")


def test_waits_are_bounded_and_slots_are_not_overwritten():
    sys.path.insert(0, ROOT)
    from branch_attention_speculative_packed_b200.tapchannel import TapMailbox, TapWriter
    box = TapMailbox(1, (4,), dtype=torch.float32, device="cpu")
    with pytest.raises(TimeoutError):
        box.wait_and_read(0, 1, timeout_s=0.05)         # nothing was written
    w = TapWriter(box.handle(), 0)
    w.write(torch.ones(4), 1)
    assert torch.equal(box.wait_and_read(0, 1), torch.ones(4))
    with pytest.raises(TimeoutError):
        w.write(torch.full((4,), 2.0), 2, timeout_s=0.05)  # tap 1 not released yet
    assert torch.equal(box.data[0], torch.ones(4))       # untouched
    box.release(0, 1)
    w.write(torch.full((4,), 2.0), 2)
    assert torch.equal(box.wait_and_read(0, 2), torch.full((4,), 2.0))
    with pytest.raises(ValueError):
        w.write(torch.ones(5), 3)                         # wrong shape


@pytest.mark.gpu
def test_mailbox_across_processes_cuda_ipc():
    _run("cuda")
