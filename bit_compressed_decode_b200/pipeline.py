"""Pipeline parallelism over GPUs: the layers of a stack split into contiguous stages, one stage
per rank, with the block's sequences cut into micro-batches that flow from stage to stage
("A 175B-parameter model on one GPU, if you can wait", key highlights: pipeline parallelism
across GPUs; the layer order within a stage is the stack's).

One decode step, GPipe order: stage r receives micro-batch j from stage r-1 (a point-to-point
receive: NCCL over NVLink between GPUs), runs its layers on it, and sends the result to stage
r+1 without waiting for the send, so the transfer of j overlaps the compute of j+1.  Stage r
works on micro-batch j while stage r+1 works on j-1: m micro-batches over n stages take
m + n - 1 stage slots.  Rows of different sequences never mix, so the result of every sequence
is the same as running all layers in one process.

The stage's computation is a callable ``run_layers(x, s0, n)`` over the rows of sequences
[s0, s0+n): for GPUs, :func:`layer_runner` wraps ``fg_layer_decode`` over the stage's layers
(weights resident in the GPU's memory, each layer's 4-bit KV cache viewed at those sequences).
"""
from __future__ import annotations

from . import replicas


def split_layers(num_layers: int, world: int, rank: int) -> tuple[int, int]:
    """(first layer, count) of `rank`'s stage: contiguous, balanced to within one layer."""
    return replicas.shard(num_layers, world, rank)


def micro_batches(num_seqs: int, parts: int) -> list[tuple[int, int]]:
    """(first sequence, count) of each micro-batch: `parts` contiguous, balanced pieces (empty
    pieces dropped)."""
    if parts < 1:
        raise ValueError("parts must be >= 1")
    out = [replicas.shard(num_seqs, parts, j) for j in range(parts)]
    return [(s, n) for s, n in out if n > 0]


class PipelineStage:
    """This rank's stage of a layer pipeline.

    run_layers(x, s0, n) -> y: the stage's layers applied to the rows `x` ([n, hidden]) of
    sequences [s0, s0+n); y has x's shape and dtype and stays valid until the step returns.
    """

    def __init__(self, run_layers, hidden: int, rank: int, world: int, group=None):
        if not 0 <= rank < world:
            raise ValueError("bad rank")
        self.run_layers, self.hidden, self.rank, self.world, self.group = run_layers, hidden, rank, world, group

    def step(self, x, parts: list[tuple[int, int]], dtype=None, device=None):
        """One decode step of the block.  Stage 0 takes the block's rows `x` ([S, hidden]); the
        other stages pass x=None and give the activations' dtype and device.  Returns the block's
        output ([S, hidden]) on the last stage, None elsewhere.  Every stage must use the same
        `parts`."""
        import torch
        import torch.distributed as dist

        first, last = self.rank == 0, self.rank == self.world - 1
        if first:
            if x is None:
                raise ValueError("stage 0 needs the block's rows")
            dtype, device = x.dtype, x.device
        outs, pending = [], []
        for s0, n in parts:
            if first:
                xin = x[s0:s0 + n]
            else:
                xin = torch.empty((n, self.hidden), dtype=dtype, device=device)
                dist.recv(xin, src=self.rank - 1, group=self.group)
            y = self.run_layers(xin, s0, n)
            if last:
                outs.append(y)
            else:
                pending.append((dist.isend(y.contiguous(), dst=self.rank + 1, group=self.group), y))
        for work, _ in pending:
            work.wait()
        return torch.cat(outs, dim=0) if last else None


def layer_runner(cfg, weights, caches, positions, workspace, stream=None):
    """run_layers for a GPU stage: ``fg_layer_decode`` of each of the stage's layers in order on a
    micro-batch (one GPU batch of its sequences), with each layer's cache viewed at those
    sequences.  weights, caches: the stage's LayerWeights and KVCaches (all sequences of the
    block); positions: int32 device [S]; workspace: device scratch for the largest micro-batch
    (``cfg.workspace_bytes(n)``)."""
    import torch

    from . import _binding as fg

    def run(x, s0, n):
        cur = x
        for w, c in zip(weights, caches):
            out = torch.empty_like(cur)
            fg.fg_layer_decode(cfg, w, c.view(s0, n), cur, positions[s0:s0 + n], num_gpu_batches=1,
                               gpu_batch_size=n, out=out, workspace=workspace, stream=stream)
            cur = out
        return cur

    return run
