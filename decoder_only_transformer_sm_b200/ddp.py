"""Data parallelism over processes, one GPU per process ("Let's reproduce GPT-2
(124M)", "Scaling to 8 GPUs with DistributedDataParallel"; "GPT-2 from
Scratch", "How to scale up").

Each rank runs the forward and backward of its own micro-batches. Before the
update the ranks sum their gradient vectors with one all-reduce, in place in
the library's gradient buffer (gpt2_grads_device). Every rank scales its
micro-batch losses by 1 / (n_micro * world), so the sum is the gradient of the
mean loss over all ranks' micro-batches; every rank then clips and applies
AdamW to that same gradient, and the replicas stay identical. The loss each
rank reports is summed over the ranks the same way. The all-reduce runs once
per optimiser step, after the last micro-batch's backward, as the pages' DDP
does (gradient sync on the last micro-step only). It is torch.distributed's
all-reduce: NCCL between GPUs, gloo in the CPU tests.

The model is any object with zero_grad(), accumulate(idx, targets,
loss_scale), grads_view() (a tensor that shares the gradient buffer),
update(lr) -> (loss, norm), get_params() and set_params(flat), as
native.GPT2 has. Create the model on torch's current stream, so that the
collective is ordered after the backward and the update after the collective.
"""
from __future__ import annotations


class DataParallel:
    """One optimiser step over all ranks' micro-batches (see the module docstring)."""

    def __init__(self, model, group=None):
        import torch.distributed as dist
        self.model = model
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

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
        m.zero_grad()
        scale = 1.0 / (n * self.world)
        for idx, targets in micro_batches:
            m.accumulate(idx, targets, scale)
        g = m.grads_view()
        if self.world > 1:
            dist.all_reduce(g, op=dist.ReduceOp.SUM, group=self.group)
        loss, norm = m.update(lr)
        if self.world > 1:
            t = torch.tensor([loss], dtype=torch.float64, device=g.device)
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=self.group)
            loss = float(t.item())
        return loss, norm
