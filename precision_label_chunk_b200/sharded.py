"""The classifier head split by labels over the ranks of a process group.

"ELMO: Efficiency via Low-precision and Peak Memory Optimization in Large
Output Spaces" (abstract) names the head as the part of the model that grows
with the label count and drives its compute and memory.  Split by label rows,
one rank per GPU, the head scales past one GPU's memory:

* rank r holds the rows [label_base, label_base + L_r) of W and runs the whole
  fused step on them (``elmo_init_head_shard``): every label's logits,
  gradient and SR update need only that label's row, X and whether the label
  is positive, and the stochastic rounding draws by the element's index in
  the whole head, so the rows come out bit-identical to an unsplit head's;
* the only exchange of a training step is the sum of the ranks' input
  gradients dX [B, d] (one all-reduce, B * d * 4 bytes);
* prediction ranks each rank's rows, gathers the ranks' [B, k] lists and
  merges them on the device (``elmo_topk_merge``).

torch.distributed carries the two collectives (NCCL between GPUs); the
library's kernels do all of the arithmetic.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (elmo_init_head_shard, elmo_topk_merge, elmo_topk_predict, elmo_train_step_chunked)

TILE = 128   # labels of one tensor-core tile: shard boundaries fall on tile boundaries


def label_shard(labels_total: int, rank: int, world: int, align: int = TILE) -> tuple[int, int]:
    """(label_base, rows) of `rank`: the head's `align`-label tiles split into
    `world` contiguous runs as evenly as possible (the ragged last tile goes to
    the last rank)."""
    if not (0 <= rank < world):
        raise ValueError(f"rank {rank} outside [0, {world})")
    tiles = -(-labels_total // align)
    if tiles < world:
        raise ValueError(f"{labels_total} labels make {tiles} tiles of {align}: fewer than {world} ranks")
    t0, t1 = tiles * rank // world, tiles * (rank + 1) // world
    base = min(t0 * align, labels_total)
    return base, min(t1 * align, labels_total) - base


def _group_info(group):
    if dist.is_available() and dist.is_initialized():
        return dist.get_rank(group), dist.get_world_size(group)
    return 0, 1


def reduce_input_grad(dX: torch.Tensor, group=None) -> torch.Tensor:
    """dX <- the sum over ranks of dX (each rank's contribution of its labels)."""
    if _group_info(group)[1] > 1:
        dist.all_reduce(dX, op=dist.ReduceOp.SUM, group=group)
    return dX


def gather_topk(idx: torch.Tensor, score: torch.Tensor, group=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Every rank's [B, k] lists, stacked to [P, B, k] on every rank."""
    P = _group_info(group)[1]
    if P == 1:
        return idx.unsqueeze(0), score.unsqueeze(0)
    gi = idx.new_empty((P,) + tuple(idx.shape))
    gs = score.new_empty((P,) + tuple(score.shape))
    dist.all_gather(list(gi.unbind(0)), idx.contiguous(), group=group)
    dist.all_gather(list(gs.unbind(0)), score.contiguous(), group=group)
    return gi, gs


class ShardedHead:
    """This rank's rows of a head of `labels_total` labels split by labels.

    W_local: this rank's rows, [rows, d] on this rank's GPU, with
    (label_base, rows) = label_shard(labels_total, rank, world) unless
    `label_base` is given.
    """

    def __init__(self, W_local: torch.Tensor, labels_total: int, dtype=None, group=None, fill: bool = False,
                 init_std: float = 0.02, seed: int = 0, label_base: int | None = None, stream=None):
        self.group = group
        self.rank, self.world = _group_info(group)
        if label_base is None:
            label_base, rows = label_shard(labels_total, self.rank, self.world)
            if W_local.shape[0] != rows:
                raise ValueError(f"rank {self.rank} holds {rows} rows of {labels_total}, W has {W_local.shape[0]}")
        self.label_base = label_base
        self.labels_total = labels_total
        self.head = elmo_init_head_shard(W_local, label_base, labels_total, dtype, fill, init_std, seed, stream)

    def train_step(self, X, rowptr, cols, lr, chunk, seed, step, dX, stream=None):
        """One step of the whole head: this rank's rows are updated in place and
        dX (fp32 [B, d]) receives the input gradient of all labels."""
        elmo_train_step_chunked(self.head, X, rowptr, cols, lr, chunk, seed, step, dX, stream)
        reduce_input_grad(dX, self.group)

    def topk_predict(self, X, k, chunk, idx, score, stream=None):
        """Top-k labels of the whole head (label ids in [0, labels_total))."""
        if self.world == 1:
            elmo_topk_predict(self.head, X, k, chunk, idx, score, stream)
            return
        li = torch.empty_like(idx)
        ls = torch.empty_like(score)
        elmo_topk_predict(self.head, X, k, chunk, li, ls, stream)
        gi, gs = gather_topk(li, ls, self.group)
        elmo_topk_merge(gi, gs, idx, score, stream)

    def close(self):
        self.head.close()
