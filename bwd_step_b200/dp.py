"""Data-parallel training step over ranks (one process per GPU).

Batch rows are independent, so each rank runs the fused step on its own rows
and the only exchange is the average of the fp32 gradients (each rank's are
the mean over its rows) and of the loss.  The library records one CUDA event
per gradient bucket as soon as the backward has finished it (LM head, then the
layers from last to first, then the token embedding); a communication stream
waits on each event and all-reduces that bucket while the backward goes on, so
the exchange overlaps the rest of the step.  Every rank must hold the same
number of rows; every rank issues the same collectives in the same order.
"""
from __future__ import annotations


def grad_buckets_from_layout(layout, n_layer):
    """The library's gradient buckets computed from the flat layout
    [(name, rows, cols, offset)] in layout order (wte, then wq wk wv wo wfc
    wproj per layer, then wlm): [(offset, count)] in backward order."""
    def span(first, last):
        off = layout[first][3]
        end = layout[last][3] + layout[last][1] * layout[last][2]
        return off, end - off
    out = [span(1 + 6 * n_layer, 1 + 6 * n_layer)]
    for l in range(n_layer - 1, -1, -1):
        out.append(span(1 + 6 * l, 6 + 6 * l))
    out.append(span(0, 0))
    return out


def average_buckets(views, group=None, before=None):
    """Average each tensor view over the ranks of `group`, in list order:
    sum-all-reduce, then scale by 1/world.  `before(i)` runs before view i is
    reduced (the step uses it to make the communication stream wait for the
    bucket's event).  Returns the async work handles of the all-reduces; the
    scaling is issued after each one completes on the same stream."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    works = []
    for i, v in enumerate(views):
        if before is not None:
            before(i)
        works.append(dist.all_reduce(v, op=dist.ReduceOp.SUM, group=group, async_op=True))
    for w, v in zip(works, views):
        w.wait()
        v.mul_(1.0 / world)
    return works


class DataParallelStep:
    """One data-parallel training step of `model` (a bwd_step_b200.Model) over
    the ranks of `group` (torch.distributed, NCCL on GPUs)."""

    def __init__(self, model, group=None):
        import torch
        import torch.distributed as dist
        self.model, self.group = model, group
        self.world = dist.get_world_size(group)
        self.buckets = model.grad_buckets()
        self.comm = torch.cuda.Stream()
        self.events = [torch.cuda.Event() for _ in self.buckets]
        s = torch.cuda.current_stream()
        for e in self.events:
            e.record(s)  # creates the CUDA event behind the handle
        model.set_grad_events(self.events)

    def step(self, tokens, targets, weights, grads, loss, workspace, stream=None):
        """Enqueue the local step and the overlapped gradient / loss averaging;
        on return `stream` is ordered after the whole exchange."""
        import torch
        stream = stream or torch.cuda.current_stream()
        self.model.forward_backward(tokens, targets, weights, grads, loss, workspace, stream)
        views = [grads[off:off + n] for off, n in self.buckets] + [loss]

        def before(i):
            if i < len(self.events):
                self.comm.wait_event(self.events[i])
            else:
                self.comm.wait_stream(stream)  # the loss is written at the end of the step

        with torch.cuda.stream(self.comm):
            average_buckets(views, self.group, before)
        stream.wait_stream(self.comm)

    def close(self):
        self.model.set_grad_events([])
