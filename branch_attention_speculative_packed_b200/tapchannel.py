"""TapChannel-style mailbox: a one-way side path for pipeline "taps".

Paper: §3.3 (the rcap.io post, the paragraph on getting target hidden states
to the draft under pipeline parallelism, and its pseudocode; the evolve.pub
FAQ "What is TapChannel?").  The draft stage owns one pre-allocated slot per
source stage in its own device memory.  A source writes its tap into its slot
after its forward pass and publishes a sequence stamp; the draft stage waits
for the stamp it expects, reads the tap, and releases the slot for the next
microbatch.  Taps only flow one way, so the pipeline schedule never sees them.

B200 / single-node form: the slots are device tensors of the draft stage's
process; sources map them through CUDA IPC (torch.multiprocessing shares a
CUDA tensor between processes that way) and write with peer copies over
NVLink.  Cross-node GPUDirect RDMA is outside this library.

Handshake (per slot, two int64 stamps in the owner's memory):
  written  -- the source sets it to s after the tap of microbatch s has landed
              (the stamp copy is queued on the source's stream after the data
              copy, so it cannot overtake it);
  released -- the owner sets it to s when it no longer needs tap s.
The source writes tap s only once released == s - 1; the owner reads tap s
only once written == s.  Stamps start at 0 and count microbatches from 1.
Both sides poll the stamps from the host, each poll bounded by a timeout that
raises TimeoutError: no GPU kernel ever waits on another process.
"""
from __future__ import annotations

import time

import torch


class TapMailbox:
    """The draft stage's mailbox: ``n_sources`` slots of ``slot_shape`` and
    ``dtype`` on ``device`` (any torch device; the CPU form shares memory
    between processes the same way)."""

    def __init__(self, n_sources: int, slot_shape, dtype=torch.bfloat16, device="cuda"):
        self.data = torch.zeros((n_sources,) + tuple(slot_shape), dtype=dtype, device=device)
        self.stamps = torch.zeros(n_sources, 2, dtype=torch.int64, device=device)  # written, released
        if self.data.device.type == "cpu":
            self.data.share_memory_()
            self.stamps.share_memory_()

    def handle(self):
        """What a source process needs (send it through torch.multiprocessing)."""
        return self.data, self.stamps

    def wait_and_read(self, src: int, stamp: int, timeout_s: float = 10.0, poll_s: float = 1e-4):
        """Waits until source ``src`` has published tap ``stamp`` and returns
        its slot (a view; valid until ``release``)."""
        _wait_for(self.stamps, src, 0, stamp, timeout_s, poll_s, "tap", src)
        return self.data[src]

    def release(self, src: int, stamp: int) -> None:
        """Tap ``stamp`` of ``src`` is consumed: the source may write the next."""
        if self.stamps.device.type == "cuda":
            torch.cuda.current_stream(self.stamps.device).synchronize()  # reads of the slot done
        self.stamps[src, 1] = stamp


class TapWriter:
    """A source stage's end of one slot of a mailbox it received through
    torch.multiprocessing."""

    def __init__(self, handle, src: int):
        self.data, self.stamps = handle
        self.src = src

    def write(self, tap: torch.Tensor, stamp: int, timeout_s: float = 10.0, poll_s: float = 1e-4,
              stream=None) -> None:
        """Writes tap ``stamp`` (1, 2, ...) into the slot once the owner has
        released tap ``stamp - 1``, then publishes the stamp."""
        if tap.shape != self.data.shape[1:] or tap.dtype != self.data.dtype:
            raise ValueError(f"tap {tuple(tap.shape)} {tap.dtype} does not fit the slot "
                             f"{tuple(self.data.shape[1:])} {self.data.dtype}")
        _wait_for(self.stamps, self.src, 1, stamp - 1, timeout_s, poll_s, "slot release", self.src)
        slot = self.data[self.src]
        if self.data.device.type == "cuda":
            st = stream if stream is not None else torch.cuda.current_stream(tap.device)
            with torch.cuda.stream(st):
                slot.copy_(tap, non_blocking=True)                   # peer copy into the owner's memory
                self.stamps[self.src, 0].fill_(stamp)                # queued after the data copy
            st.synchronize()
        else:
            slot.copy_(tap)
            self.stamps[self.src, 0] = stamp


def _wait_for(stamps, src, col, value, timeout_s, poll_s, what, who):
    t0 = time.monotonic()
    while True:
        got = int(stamps[src, col].item())
        if got == value:
            return
        if got > value:
            raise RuntimeError(f"{what} of source {who}: stamp {got} already past {value}")
        if time.monotonic() - t0 > timeout_s:
            raise TimeoutError(f"{what} of source {who}: waited {timeout_s} s for stamp {value}, "
                               f"stamp is {got}")
        time.sleep(poll_s)
