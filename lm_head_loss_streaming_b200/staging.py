"""Double-buffered host-to-device staging of a step's inputs.

When a step's inputs (hidden states, target hidden states, labels) arrive in host memory,
each step has to copy them to the GPU before its kernels can run.  InputStager keeps two
device copies of the inputs and a copy stream: the copy of step k+1's inputs runs on the
copy stream while step k computes on the other copy.  Events order the two streams:

  * the compute stream waits for a set's copy to land before it reads the set (``get``);
  * the copy stream waits for the compute that last read a set before it overwrites the
    set (``done`` records that point).

Host tensors should be pinned (``tensor.pin_memory()``), or the copies are synchronous.
"""

from __future__ import annotations

import torch


class InputStager:
    """Two device buffer sets shaped like ``like`` ({name: tensor or None}) and a copy
    stream on ``like``'s device.  Typical loop::

        stager = InputStager({"h": h_dev, "labels": lab_dev})
        slot = stager.put(host_batches[0])
        for k in range(steps):
            nxt = stager.put(host_batches[k + 1]) if k + 1 < steps else None
            bufs = stager.get(slot)          # the current stream waits for the copy
            ... run the step on bufs ...
            stager.done(slot)                # the copy stream may now reuse the set
            slot = nxt
    """

    def __init__(self, like: dict, device=None):
        ref = next(t for t in like.values() if t is not None)
        self.device = torch.device(device) if device is not None else ref.device
        self.bufs = [{k: (None if t is None else torch.empty_like(t, device=self.device))
                      for k, t in like.items()} for _ in range(2)]
        self.copy_stream = torch.cuda.Stream(device=self.device)
        self.ready = [torch.cuda.Event(), torch.cuda.Event()]
        self.free: list = [None, None]
        self.next = 0

    def start_after_current(self):
        """Make the next copies wait for the work already enqueued on the current stream
        (so that a timing event recorded there brackets them)."""
        self.copy_stream.wait_stream(torch.cuda.current_stream(self.device))

    def put(self, host: dict) -> int:
        """Enqueue the copies of ``host`` ({name: host tensor}) into the next buffer set on
        the copy stream; returns the set's slot."""
        s = self.next
        self.next ^= 1
        with torch.cuda.stream(self.copy_stream):
            if self.free[s] is not None:
                self.copy_stream.wait_event(self.free[s])
            for k, h in host.items():
                if h is not None:
                    self.bufs[s][k].copy_(h, non_blocking=True)
            self.ready[s].record(self.copy_stream)
        return s

    def get(self, slot: int) -> dict:
        """The buffer set of ``slot``; the current stream waits for its copies."""
        torch.cuda.current_stream(self.device).wait_event(self.ready[slot])
        return self.bufs[slot]

    def done(self, slot: int):
        """Records that the work enqueued so far on the current stream is the last to read
        the set of ``slot``."""
        ev = torch.cuda.Event()
        ev.record(torch.cuda.current_stream(self.device))
        self.free[slot] = ev
