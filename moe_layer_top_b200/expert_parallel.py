"""Expert parallelism of the fused MoE layer over ``torch.distributed``.

"Hosting von Qwen auf Blackwell" (perplexity.ai), section "MoE Dispatch -
Combine", "Experten-Parallel": the layer's inputs are replicated on every
rank; the dispatch keeps only the tokens routed to the rank's own experts, the
combine first accumulates their contributions per token on the rank, and an
all-reduce over the ranks then completes the layer.

Here the rank-local part is one ``moe_fused_forward`` call whose problem names
the rank's expert range (``num_global_experts`` / ``first_expert``): the
library routes over all experts, its alignment keeps the local assignments and
its combine sums only their rows.  The reduction is a ``torch.distributed``
all-reduce (NCCL over NVLink between GPUs).  Each rank holds the weights of its
experts only: ``E / world_size`` of them, contiguous.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import ops


def expert_shard(E: int, world_size: int, rank: int) -> tuple:
    """Experts ``(first, count)`` of ``rank``: ``[floor(rank*E/N), floor((rank+1)*E/N))``,
    contiguous, sizes differing by at most one."""
    if not 1 <= world_size <= E:
        raise ValueError(f"need 1 <= world_size <= E (world_size {world_size}, E {E})")
    if not 0 <= rank < world_size:
        raise ValueError(f"rank {rank} outside [0, {world_size})")
    first = (rank * E) // world_size
    return first, ((rank + 1) * E) // world_size - first


class ExpertParallelMoE:
    """One rank's share of an expert-parallel MoE layer of ``E`` experts.

    ``problem_kw`` are the other :func:`ops.problem` options (``fp8``, ``mx``,
    ``mode``, ...).  :meth:`forward` takes x [T, H], the routing over all
    experts (``logits`` [T, E] or global ``topk_ids`` / ``topk_weights``) and
    this rank's weights (:meth:`local_experts` of the full tensors), and
    returns the whole layer's output on every rank.  ``rank`` / ``world_size``
    default to the process group's (one rank without one); given explicitly
    they select a share without a group, for :meth:`local_forward` alone.
    """

    def __init__(self, T: int, E: int, topk: int, H: int, I: int, *, group=None, rank=None, world_size=None,
                 **problem_kw):
        self.group = group
        if (rank is None) != (world_size is None):
            raise ValueError("give both rank and world_size, or neither")
        if rank is not None:
            self.world_size, self.rank = int(world_size), int(rank)
        elif dist.is_available() and dist.is_initialized():
            self.world_size = dist.get_world_size(group)
            self.rank = dist.get_rank(group)
        else:
            self.world_size, self.rank = 1, 0
        self.E, self.T = int(E), int(T)
        self.first_expert, self.num_local = expert_shard(self.E, self.world_size, self.rank)
        self.problem = ops.problem(T, self.num_local, topk, H, I, num_global_experts=self.E,
                                   first_expert=self.first_expert, **problem_kw)
        self._ws = None

    def local_experts(self, w: torch.Tensor) -> torch.Tensor:
        """This rank's experts of a full per-expert tensor [E, ...] (weights or their scales)."""
        if w.shape[0] != self.E:
            raise ValueError(f"expected {self.E} experts, got {w.shape[0]}")
        return w[self.first_expert:self.first_expert + self.num_local]

    def local_forward(self, x, w13, w2, **kw) -> torch.Tensor:
        """This rank's partial output: the sum over each token's assignments to local experts."""
        if x.shape[0] != self.T:
            raise ValueError(f"x has {x.shape[0]} tokens, the problem {self.T}")
        if self._ws is None or self._ws.device != x.device:
            self._ws = ops.alloc_workspace(self.problem, x.device)
        return ops.fused_forward(self.problem, x, w13, w2, ws=self._ws, **kw)

    def forward(self, x, w13, w2, **kw) -> torch.Tensor:
        out = self.local_forward(x, w13, w2, **kw)
        if self.world_size > 1:
            if not (dist.is_available() and dist.is_initialized()):
                raise RuntimeError("forward of a rank of several needs the process group; use local_forward")
            dist.all_reduce(out, op=dist.ReduceOp.SUM, group=self.group)
        return out

    __call__ = forward
