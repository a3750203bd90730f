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
        self._shape = (int(topk), int(H), int(I), dict(problem_kw))
        self._problems, self._workspaces = {}, {}
        self.problem = self.problem_for(self.T)

    def problem_for(self, T: int):
        """This rank's moe_problem for a batch of T tokens."""
        if T not in self._problems:
            topk, H, I, kw = self._shape
            self._problems[T] = ops.problem(T, self.num_local, topk, H, I, num_global_experts=self.E,
                                            first_expert=self.first_expert, **kw)
        return self._problems[T]

    def workspace_for(self, T: int, device) -> torch.Tensor:
        """The workspace of this rank's T-token problem on ``device`` (allocated on first use)."""
        dev = torch.device(device)
        if dev.type == "cuda" and dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        key = (T, str(dev))
        if key not in self._workspaces:
            self._workspaces[key] = ops.alloc_workspace(self.problem_for(T), dev)
        return self._workspaces[key]

    def local_experts(self, w: torch.Tensor) -> torch.Tensor:
        """This rank's experts of a full per-expert tensor [E, ...] (weights or their scales)."""
        if w.shape[0] != self.E:
            raise ValueError(f"expected {self.E} experts, got {w.shape[0]}")
        return w[self.first_expert:self.first_expert + self.num_local]

    def local_forward(self, x, w13, w2, **kw) -> torch.Tensor:
        """This rank's partial output for x [T', H] (any T'): the sum over each token's assignments
        to local experts."""
        T = x.shape[0]
        return ops.fused_forward(self.problem_for(T), x, w13, w2, ws=self.workspace_for(T, x.device), **kw)

    def forward(self, x, w13, w2, *, chunks: int = 1, **kw) -> torch.Tensor:
        """The layer's output on every rank.  ``chunks`` > 1 splits the batch into that many
        contiguous token ranges: the all-reduce of a range is issued asynchronously (NCCL runs it
        on its own stream) while the next range computes, so the exchange overlaps the GEMMs
        (every output row depends only on its own token, so the result is the same layer)."""
        if self.world_size > 1 and not (dist.is_available() and dist.is_initialized()):
            raise RuntimeError("forward of a rank of several needs the process group; use local_forward")
        T = x.shape[0]
        chunks = max(1, min(int(chunks), T))
        if chunks == 1:
            out = self.local_forward(x, w13, w2, **kw)
            if self.world_size > 1:
                dist.all_reduce(out, op=dist.ReduceOp.SUM, group=self.group)
            return out
        out = kw.pop("out", None)
        if out is None:
            out = torch.empty((T, x.shape[1]), dtype=torch.bfloat16, device=x.device)
        per_token = ("logits", "topk_ids", "topk_weights")
        bounds = [(c * T) // chunks for c in range(chunks + 1)]
        pending = []
        for c0, c1 in zip(bounds, bounds[1:]):
            sub = {k: (v[c0:c1] if k in per_token and v is not None else v) for k, v in kw.items()}
            self.local_forward(x[c0:c1], w13, w2, out=out[c0:c1], **sub)
            if self.world_size > 1:
                pending.append(dist.all_reduce(out[c0:c1], op=dist.ReduceOp.SUM, group=self.group,
                                               async_op=True))
        for work in pending:
            work.wait()
        return out

    __call__ = forward
