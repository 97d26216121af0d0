"""Data parallelism over processes, one GPU per process ("Let's reproduce GPT-2
(124M)", "Scaling to 8 GPUs with DistributedDataParallel"; "GPT-2 from
Scratch", "How to scale up").

Each rank runs the forward and backward of its own micro-batches. Before the
update the ranks sum their gradient vectors with one all-reduce, in place in
the library's gradient buffer (gpt2_grads_device). Every rank scales its
micro-batch losses by 1 / (n_micro * world), so the sum is the gradient of the
mean loss over all ranks' micro-batches; every rank then clips and applies
AdamW to that same gradient, and the replicas stay identical. The loss each
rank reports is summed over the ranks the same way. The exchange runs once per
optimiser step, in the last micro-batch's backward, as the pages' DDP does
(gradient sync on the last micro-step only). It is torch.distributed's
all-reduce: NCCL between GPUs, gloo in the CPU tests.

Buckets: the gradient vector is exchanged in the ranges the backward finishes
one after another (gpt2_grad_buckets: ln_f, the blocks from the last to the
first, then wte and wpe). On GPUs the library records a CUDA event as each
bucket becomes final (gpt2_set_grad_events); a communication stream waits for
each event in turn and all-reduces that bucket, so the exchange of the late
layers overlaps the backward of the early ones, and the update waits for the
communication stream. Each all-reduce sums the same elements as one all-reduce
of the whole vector would, so the result does not depend on the bucketing.

The model is any object with zero_grad(), accumulate(idx, targets,
loss_scale), grads_view() (a tensor that shares the gradient buffer),
update(lr) -> (loss, norm), get_params() and set_params(flat), as
native.GPT2 has; with grad_buckets() (and, for the overlap on GPUs,
set_grad_events(events)) the exchange is bucketed. Create the model on
torch's current stream, so that the collectives are ordered after the
backward and the update after the collectives.
"""
from __future__ import annotations


class DataParallel:
    """One optimiser step over all ranks' micro-batches (see the module docstring)."""

    def __init__(self, model, group=None, bucketed: bool = True):
        import torch
        import torch.distributed as dist
        self.model = model
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.buckets = model.grad_buckets() if bucketed and hasattr(model, "grad_buckets") else None
        self.events = None
        self.comm = None
        g = model.grads_view()
        if self.buckets is not None and g.is_cuda and hasattr(model, "set_grad_events"):
            # one event per bucket, recorded once so that the CUDA event exists
            self.events = [torch.cuda.Event() for _ in self.buckets]
            for ev in self.events:
                ev.record()
            model.set_grad_events(self.events)
            self.comm = torch.cuda.Stream(device=g.device)

    def broadcast_params(self):
        """Copy rank 0's parameters to every rank (the replicas start equal)."""
        import numpy as np
        import torch
        import torch.distributed as dist
        dev = self.model.grads_view().device
        flat = torch.from_numpy(np.ascontiguousarray(self.model.get_params())).to(dev)
        dist.broadcast(flat, src=dist.get_global_rank(self.group, 0) if self.group is not None else 0,
                       group=self.group)
        self.model.set_params(flat.cpu().numpy() if dev.type == "cpu" else flat)

    def step(self, micro_batches, lr: float):
        """zero_grad; accumulate each (idx, targets) of this rank with loss scale
        1 / (len(micro_batches) * world); all-reduce (sum) the gradients; update.
        Every rank must pass the same number of micro-batches. Returns (the mean
        loss over every rank's micro-batches, the pre-clip norm of the averaged
        gradient)."""
        import torch
        import torch.distributed as dist
        n = len(micro_batches)
        if n < 1:
            raise ValueError("at least one micro-batch per rank")
        m = self.model
        count = getattr(m, "last_launch_count", None)
        self.last_launches = 0
        m.zero_grad()
        scale = 1.0 / (n * self.world)
        for idx, targets in micro_batches:
            m.accumulate(idx, targets, scale)
            if count:
                self.last_launches += count()
        g = m.grads_view()
        if self.world > 1:
            self._exchange(g)
        loss, norm = m.update(lr)
        if count:
            self.last_launches += count()
        if self.world > 1:
            t = torch.tensor([loss], dtype=torch.float64, device=g.device)
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=self.group)
            loss = float(t.item())
        return loss, norm

    def _exchange(self, g):
        """Sum g over the ranks: whole, or bucket by bucket in the order the backward
        finishes them; on GPUs each bucket's all-reduce waits (on the communication
        stream) only for that bucket's event of the backward just enqueued."""
        import torch
        import torch.distributed as dist
        if self.buckets is None:
            dist.all_reduce(g, op=dist.ReduceOp.SUM, group=self.group)
            return
        if self.comm is None:
            for off, cnt in self.buckets:
                dist.all_reduce(g[off:off + cnt], op=dist.ReduceOp.SUM, group=self.group)
            return
        main = torch.cuda.current_stream(g.device)
        with torch.cuda.stream(self.comm):
            for (off, cnt), ev in zip(self.buckets, self.events):
                self.comm.wait_event(ev)
                dist.all_reduce(g[off:off + cnt], op=dist.ReduceOp.SUM, group=self.group)
        main.wait_stream(self.comm)
