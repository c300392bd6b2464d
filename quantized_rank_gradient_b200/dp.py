"""Layer-sharded data parallelism around the optimizer step (host side).

Every weight matrix's optimizer state (its INT4 projection, INT8 moments and
schedule) is independent of the others, so in a data-parallel trainer each
matrix can be owned by one rank:

1. every rank holds the full model's gradients of its own slice of the batch;
2. the gradients are reduce-scattered by ownership: the owner of a matrix
   receives the mean over the ranks, summed in float32 and rounded once to
   bf16;
3. each rank runs the optimizer step (qg_step_batch) on the matrices it owns;
4. the updated INT8 weights are all-gathered, so that every rank holds the
   whole model for the next forward pass.  Each matrix's group scales sit
   right after its codes in the same buffer: with qg_config.w_rescale = 1 the
   owner's step changes them, and the one all-gather carries them too.

Matrices go to ranks longest first, each to the rank with the least work so far
(work = 4 m n r, the step's FLOPs), ties to the lowest rank.  Gradients and
weights live in flat buffers laid out shard by shard, rank after rank, every
shard padded to the same size, so steps 2 and 4 are one reduce-scatter and one
all-gather of contiguous tensors (NCCL over NVLink on B200).  With a backend
that has no reduce-scatter (gloo), step 2 is an all-reduce followed by taking
the own shard, which gives the same values.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

GRAD_ALIGN = 8      # bf16 elements: every gradient starts on a 16-byte boundary
WEIGHT_ALIGN = 256  # bytes: every weight matrix and every scale array starts on a 256-byte boundary


def _round(x, a):
    return -(-x // a) * a


@dataclass
class ShardPlan:
    """Where every matrix lives in the flat gradient and weight buffers."""
    world: int
    owner: list            # rank owning matrix i
    grad_offset: list      # element offset of matrix i's gradient (m x ldg) in the flat gradient buffer
    weight_offset: list    # byte offset of matrix i's codes (m x ldw) in the flat weight buffer
    scale_offset: list     # byte offset of matrix i's ceil(m n / 256) float32 group scales, after its codes
    ldg: list              # gradient row stride (elements)
    ldw: list              # weight row stride (bytes)
    grad_shard: int        # elements per rank shard of the gradient buffer
    weight_shard: int      # bytes per rank shard of the weight buffer
    work: list             # per rank, sum of 4 m n r over its matrices

    def owned(self, rank):
        return [i for i, o in enumerate(self.owner) if o == rank]


def plan_shards(shapes, ranks_r, world) -> ShardPlan:
    """shapes: [(m, n)] per matrix; ranks_r: [r] per matrix (projection rank)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    cost = [4.0 * m * n * r for (m, n), r in zip(shapes, ranks_r)]
    order = sorted(range(len(shapes)), key=lambda i: (-cost[i], i))
    work = [0.0] * world
    owner = [0] * len(shapes)
    for i in order:
        w = min(range(world), key=lambda k: (work[k], k))
        owner[i] = w
        work[w] += cost[i]
    ldg = [_round(n, GRAD_ALIGN) for (_, n) in shapes]
    ldw = [_round(n, 16) for (_, n) in shapes]
    goff, woff, soff = [0] * len(shapes), [0] * len(shapes), [0] * len(shapes)
    gsize, wsize = [0] * world, [0] * world
    for i, (m, n) in enumerate(shapes):  # within a shard, matrices keep their order
        k = owner[i]
        goff[i], woff[i] = gsize[k], wsize[k]
        gsize[k] += _round(m * ldg[i], GRAD_ALIGN)
        wsize[k] += _round(m * ldw[i], WEIGHT_ALIGN)
        soff[i] = wsize[k]
        wsize[k] += _round(4 * -(-(m * n) // 256), WEIGHT_ALIGN)
    gshard, wshard = _round(max(gsize), GRAD_ALIGN), _round(max(wsize), WEIGHT_ALIGN)
    for i in range(len(shapes)):
        goff[i] += owner[i] * gshard
        woff[i] += owner[i] * wshard
        soff[i] += owner[i] * wshard
    return ShardPlan(world, owner, goff, woff, soff, ldg, ldw, gshard, wshard, work)


def grad_view(flat, plan, i, shape):
    """Matrix i's gradient (m x ldg) inside the flat gradient buffer."""
    m, _n = shape
    return flat[plan.grad_offset[i]: plan.grad_offset[i] + m * plan.ldg[i]].view(m, plan.ldg[i])


def weight_view(flat, plan, i, shape):
    """Matrix i's INT8 codes (m x ldw) inside the flat weight buffer."""
    m, _n = shape
    return flat[plan.weight_offset[i]: plan.weight_offset[i] + m * plan.ldw[i]].view(m, plan.ldw[i])


def scale_view(flat, plan, i, shape):
    """Matrix i's ceil(m n / 256) float32 group scales inside the flat weight
    buffer (a uint8 tensor): the d_Wscale array of its qg_layer."""
    m, n = shape
    ng = -(-(m * n) // 256)
    return flat[plan.scale_offset[i]: plan.scale_offset[i] + 4 * ng].view(torch.float32)


def reduce_scatter_gradients(flat, plan, rank, group=None):
    """Mean over the ranks of every gradient, delivered to its owner: afterwards
    this rank's shard of the bf16 buffer `flat` holds the means of the
    gradients it owns (the other shards are left unspecified).

    Numerics: the local bf16 gradients are widened to float32, summed over the
    ranks in float32 (in the collective's own order), divided by the rank count
    in float32, and rounded once to bf16 (nearest, ties to even) on the owner:
    G = bf16(fl32(fl32(sum_k G_k) / world)).  A bf16 sum on the wire would round
    at every hop of a ring or tree, so its result would depend on the algorithm
    and the rank count; in float32 the only order-dependent rounding is the
    sum's, at most (world - 1) 2^-24 sum_k |G_k| per element, and for two ranks
    the sum is exact whenever the two exponents are within 15 of each other.
    The float32 copy doubles the bytes on the wire and, for the time of the
    call, the gradient memory (26 GB for the LLaMA-7B stack)."""
    n = plan.grad_shard
    mine = flat[rank * n: (rank + 1) * n]
    if plan.world == 1:
        return mine
    if flat.dtype != torch.bfloat16:
        raise TypeError("the gradient buffer holds bf16, the dtype qg_step takes")
    wide = flat.to(torch.float32)
    if dist.get_backend(group) == "nccl":
        total = torch.empty(n, dtype=torch.float32, device=flat.device)
        dist.reduce_scatter_tensor(total, wide, op=dist.ReduceOp.SUM, group=group)
    else:
        dist.all_reduce(wide, op=dist.ReduceOp.SUM, group=group)
        total = wide[rank * n: (rank + 1) * n]
    total.div_(plan.world)
    mine.copy_(total)  # float32 -> bf16, round to nearest even
    return mine


def all_gather_weights(flat, plan, rank, group=None):
    """Every rank's shard of the flat weight buffer (codes and group scales) to
    every rank."""
    n = plan.weight_shard
    if plan.world == 1:
        return flat
    mine = flat[rank * n: (rank + 1) * n]
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(flat, mine, group=group)
    else:
        parts = [torch.empty_like(mine) for _ in range(plan.world)]
        dist.all_gather(parts, mine.clone(), group=group)
        for k, p in enumerate(parts):
            flat[k * n: (k + 1) * n].copy_(p)
    return flat
