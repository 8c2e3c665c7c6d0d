"""Stream-level plumbing for the library's entry points: host-to-device input
staging that overlaps the next step's copy with this step's compute
(``InputPrefetcher``), and replay of a fixed call sequence as one CUDA graph
(``GraphedCall``).

Input staging
-------------

A training step reads a few per-step inputs from the host: hidden states,
targets, behaviour log-probs, advantages and the mask.  Copied on the compute
stream they serialise with the step.  ``InputPrefetcher`` keeps two device
copies of those inputs and fills one on a separate copy stream while the other
is in use:

    pf = InputPrefetcher(templates)          # device tensors giving names, shapes, dtypes
    pf.prefetch(host_batch_0)
    for i in range(steps):
        dev = pf.next()                       # the current stream waits for batch i's copy
        if i + 1 < steps:
            pf.prefetch(host_batch[i + 1])    # batch i+1 copies while step i runs
        step(**dev)
        pf.release()                          # the slot may be refilled once step i is done

Host tensors must be pinned for the copies to be asynchronous.  Ordering is
kept with CUDA events only, so the host never waits.  This is plumbing (streams
and copies); no arithmetic of the loss path happens here.
"""
from __future__ import annotations

import torch


class InputPrefetcher:
    def __init__(self, templates: dict, depth: int = 2, copy_stream: torch.cuda.Stream | None = None):
        if depth < 2:
            raise ValueError("InputPrefetcher needs at least two slots")
        self.names = list(templates)
        dev = next(iter(templates.values())).device
        self.slots = [{k: torch.empty_like(v, device=dev) for k, v in templates.items()} for _ in range(depth)]
        self.copied = [torch.cuda.Event() for _ in range(depth)]
        self.freed = [None] * depth
        self.copy_stream = copy_stream or torch.cuda.Stream(device=dev)
        self.head = 0          # next slot to fill
        self.tail = 0          # next slot to hand out
        self.inflight = 0
        self.current = None

    def prefetch(self, host: dict) -> None:
        """Starts copying `host` (name -> pinned CPU tensor) into the next free slot."""
        if self.inflight == len(self.slots):
            raise RuntimeError("InputPrefetcher: every slot is in flight; call next() first")
        s = self.head
        with torch.cuda.stream(self.copy_stream):
            if self.freed[s] is not None:
                self.copy_stream.wait_event(self.freed[s])
            for k in self.names:
                self.slots[s][k].copy_(host[k], non_blocking=True)
            self.copied[s].record(self.copy_stream)
        self.head = (s + 1) % len(self.slots)
        self.inflight += 1

    def next(self) -> dict:
        """The oldest prefetched batch, ready for use on the current stream."""
        if self.inflight == 0:
            raise RuntimeError("InputPrefetcher: nothing prefetched")
        s = self.tail
        torch.cuda.current_stream().wait_event(self.copied[s])
        self.tail = (s + 1) % len(self.slots)
        self.inflight -= 1
        self.current = s
        return self.slots[s]

    def release(self) -> None:
        """Marks the batch returned by the last next() as consumed by the work
        enqueued so far on the current stream."""
        if self.current is None:
            return
        ev = torch.cuda.Event()
        ev.record(torch.cuda.current_stream())
        self.freed[self.current] = ev
        self.current = None

    def finish(self) -> None:
        """Makes the current stream wait for every copy still in flight."""
        for i in range(self.inflight):
            torch.cuda.current_stream().wait_event(self.copied[(self.tail + i) % len(self.slots)])


class GraphedCall:
    """Captures `fn` (a call sequence of the library's entry points on fixed
    device buffers) into a CUDA graph and replays it with one launch.

    The library's one-time host work (kernel attributes, occupancy queries) and
    any workspace creation happen in the `warmup` eager calls before capture;
    the captured calls then contain only kernel launches on the capturing
    stream.  Replays read and write the same buffers as the captured call: copy
    new inputs into them before ``replay()``.  This replaces per-call launch
    overhead -- several kernels per fused step, one cooperative launch per loss
    call -- for small, launch-bound batches.
    """

    def __init__(self, fn, warmup: int = 2):
        stream = torch.cuda.Stream()
        stream.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(stream):
            for _ in range(warmup):
                fn()
        torch.cuda.current_stream().wait_stream(stream)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            fn()

    def replay(self) -> None:
        self.graph.replay()
