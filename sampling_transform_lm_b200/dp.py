"""Data-parallel weight-gradient sum for the scoring core's backward.

Every rank scores its own rows against the same W, so each rank's dW is a
partial sum; the loss layer's weight gradient is their sum over ranks ("What
this PR does", item 2, of the xorl PR "Consolidate sampling-transform scoring
on one shared chunked core"). The backward writes dW once per vocabulary slice
("Self-review pass"), so the sum can start slice by slice while the GEMMs of
the next slice run: ``SliceAllReduce`` is the ``on_dw_slice`` callback of
``sts_backward`` that does this with ``torch.distributed`` (NCCL over NVLink on
GPUs, gloo for CPU tensors in tests).
"""

from __future__ import annotations

import torch
import torch.distributed as dist


class SliceAllReduce:
    """Sum every dW slice over a process group as soon as its GEMM is enqueued.

    Per slice, on the host thread that runs the backward: an event recorded on
    the compute stream, the communication stream made to wait for it, and an
    asynchronous all-reduce of the slice issued under that stream. ``finish``
    makes the compute stream wait for every exchange; call it before reading
    dW. CPU tensors (gloo) take the same steps without streams.
    """

    def __init__(self, group=None, comm_stream=None, average=False):
        self.group = group
        self.average = average
        self.comm_stream = comm_stream
        self.works = []
        self.slices = []  # (v0, rows) in the order handed out

    def __call__(self, v0, rows, dW_slice):
        self.slices.append((int(v0), int(rows)))
        if dW_slice.is_cuda:
            compute = torch.cuda.current_stream(dW_slice.device)
            if self.comm_stream is None:
                self.comm_stream = torch.cuda.Stream(device=dW_slice.device)
            ready = torch.cuda.Event()
            ready.record(compute)
            self.comm_stream.wait_event(ready)
            with torch.cuda.stream(self.comm_stream):
                self.works.append((dist.all_reduce(dW_slice, group=self.group, async_op=True),
                                   dW_slice))
        else:
            self.works.append((dist.all_reduce(dW_slice, group=self.group, async_op=True), dW_slice))

    def finish(self):
        """Wait for every slice's exchange (on the device for CUDA tensors);
        returns the slices (v0, rows) exchanged since the last call."""
        world = dist.get_world_size(self.group)
        for work, sl in self.works:
            work.wait()
            if self.average and world > 1:
                sl.div_(world)
        if self.comm_stream is not None:
            torch.cuda.current_stream(self.comm_stream.device).wait_stream(self.comm_stream)
        self.works = []
        done, self.slices = self.slices, []
        return done
