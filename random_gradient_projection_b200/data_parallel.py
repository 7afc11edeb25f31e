"""Data-parallel DP-GRAPE step: one process per GPU, samples sharded across ranks.

Per-sample work (projection, norms, clipping) needs no exchange: every rank
clips its own samples.  The one exchange is the sum of the clipped projected
gradients S_l = sum_i c_i R_{i,l} over all ranks (an all-reduce of r x d_out
fp32 per layer).  Every rank then adds the same noise (the same Philox key),
divides by the global batch, runs Adam and back-projects, so the replicas
stay identical.
"""
from __future__ import annotations


def dp_step(g, A, Gout, W, step: int, group=None, stream=None, batch_total=None):
    """One step of context ``g`` (a GrapeStep or an object with the same methods)
    inside ``torch.distributed`` process group ``group``.

    ``batch_total`` is the global batch the noisy sum is averaged over.  By default
    every rank holds ``g.B`` samples (B x world); ranks whose shards differ in size
    pass the sum of their shard sizes, the same number on every rank."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    if batch_total is None:
        batch_total = g.B * world
    g.accumulate(A, Gout, step, stream)
    if world > 1:
        if hasattr(g, "S_all_tensor"):
            # every S_l lies back to back: one all-reduce for the whole step
            dist.all_reduce(g.S_all_tensor(), op=dist.ReduceOp.SUM, group=group)
        else:
            for l in range(len(g.layers)):
                dist.all_reduce(g.S_tensor(l), op=dist.ReduceOp.SUM, group=group)
    g.apply(W, step, batch_total, stream)
