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
all-reduce (NCCL over NVLink between GPUs), or, with ``fused_allreduce``, the
library's own kernel that does the combine and the all-reduce together over
peer memory (symmetric buffers from ``torch.distributed._symmetric_memory``).
Each rank holds the weights of its experts only: ``E / world_size`` of them,
contiguous.
"""

from __future__ import annotations

import os

import torch
import torch.distributed as dist

from . import ops


NO_MULTICAST_ENV = "TORCH_SYMM_MEM_DISABLE_MULTICAST"


def force_no_multicast() -> None:
    """Make torch's symmetric memory bind no NVLink multicast object to its buffers.

    The fused exchange reads and writes peers with plain loads and stores only, and a rank
    that ends while its memory is bound to a multicast object can fault the other GPUs.  A
    caller who set the switch to anything but "1" gets an error instead of a silent override
    (torch may already have read the value)."""
    v = os.environ.get(NO_MULTICAST_ENV)
    if v is not None and v != "1":
        raise RuntimeError(f"{NO_MULTICAST_ENV}={v!r}: the fused combine + all-reduce needs symmetric "
                           f"buffers without multicast; unset it or set it to 1")
    os.environ[NO_MULTICAST_ENV] = "1"
    assert os.environ[NO_MULTICAST_ENV] == "1"


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

    ``data_parallel``: every rank brings its OWN batch of T tokens (the page's
    decoders: data parallel and expert parallel together).  The ranks' x and
    routing inputs are gathered, each rank runs its share on the gathered batch
    of world * T tokens, and a reduce-scatter leaves each rank the layer for its
    own tokens.  (The page's decoders exchange only the chosen (token, expert)
    rows with a sparse all-to-all; the gather sends every token to every rank,
    which costs the same bytes when a token's k experts span most ranks.)
    """

    def __init__(self, T: int, E: int, topk: int, H: int, I: int, *, group=None, rank=None, world_size=None,
                 fused_allreduce: bool = False, data_parallel: bool = False, **problem_kw):
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
        self.data_parallel = bool(data_parallel)
        self.problem = self.problem_for(self.T * (self.world_size if self.data_parallel else 1))
        self.fused_allreduce = bool(fused_allreduce)
        self._exchange = {}

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

    def _exchange_for(self, T: int, device):
        """Symmetric buffers (partial, out, flags) of the fused combine + all-reduce for T tokens
        (per rank, with ``data_parallel``), their peer addresses, and the call counter (collective
        on first use for a T)."""
        if T in self._exchange:
            return self._exchange[T]
        force_no_multicast()
        import torch.distributed._symmetric_memory as symm_mem
        group = self.group if self.group is not None else dist.group.WORLD
        if not symm_mem.is_symm_mem_enabled_for_group(group.group_name):
            symm_mem.enable_symm_mem_for_group(group.group_name)
        H = self._shape[1]
        rows = T * self.world_size if self.data_parallel else T     # the batch the share runs on
        count = (ops.combine_reduce_scatter_flag_count if self.data_parallel else ops.combine_allreduce_flag_count)
        assert os.environ.get(NO_MULTICAST_ENV) == "1", "symmetric buffers must not be multicast-bound"
        partial = symm_mem.empty((rows, H), dtype=torch.bfloat16, device=device)
        out = symm_mem.empty((T, H), dtype=torch.bfloat16, device=device)
        flags = symm_mem.empty((count(T, self.world_size),), dtype=torch.int32, device=device)
        flags.zero_()
        handles = [symm_mem.rendezvous(t, group) for t in (partial, out, flags)]
        torch.cuda.synchronize(device)
        dist.barrier(group)      # every rank's flags are zero before any rank signals
        p = self.problem_for(rows)
        ws = self.workspace_for(rows, device)
        lay = ops.workspace_layout(p)
        base = ws.data_ptr()
        ranks = []
        for r in range(self.world_size):
            d = {"partial": handles[0].buffer_ptrs[r], "out": handles[1].buffer_ptrs[r],
                 "flags": handles[2].buffer_ptrs[r]}
            if r == self.rank:
                d.update(y=base + lay.y, status=base + lay.status,
                         pos_of_flat=base + lay.pos_of_flat if lay.pos_of_flat >= 0 else None)
            ranks.append(d)
        ex = {"partial": partial, "out": out, "flags": flags, "handles": handles, "ranks": ranks, "epoch": 0}
        self._exchange[T] = ex
        return ex

    def _fused_forward(self, T, x, w13, w2, **kw) -> torch.Tensor:
        """x: the batch the share runs on (the gathered one with ``data_parallel``); T: tokens of
        this rank's output."""
        rows = x.shape[0]
        user_out = kw.pop("out", None)
        ex = self._exchange_for(T, x.device)
        p = self.problem_for(rows)
        ops.forward_stages(p, x, w13, w2, ops.STAGE_ROUTE, ops.STAGE_COMBINE, out=ex["out"],
                           ws=self.workspace_for(rows, x.device), **kw)
        ex["epoch"] += 1
        topk, H = self._shape[0], self._shape[1]
        exchange = ops.combine_reduce_scatter if self.data_parallel else ops.combine_allreduce
        exchange(T, topk, H, self.rank, ex["ranks"], ex["epoch"])
        if user_out is None:
            return ex["out"]
        user_out.copy_(ex["out"])
        return user_out

    def _gather(self, x, kw):
        """The ranks' batches and per-token routing inputs, concatenated in rank order."""
        if self.world_size == 1:
            return x, dict(kw)

        def gather(t):
            full = torch.empty((t.shape[0] * self.world_size,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
            dist.all_gather_into_tensor(full, t.contiguous(), group=self.group)
            return full
        kw = dict(kw)
        for key in ("logits", "topk_ids", "topk_weights"):
            if kw.get(key) is not None:
                kw[key] = gather(kw[key])
        return gather(x), kw

    def _data_parallel_forward(self, x, w13, w2, **kw) -> torch.Tensor:
        T = x.shape[0]
        xg, kw = self._gather(x, kw)
        if self.fused_allreduce:
            return self._fused_forward(T, xg, w13, w2, **kw)
        user_out = kw.pop("out", None)
        full = self.local_forward(xg, w13, w2, **kw)      # this rank's partial for every rank's tokens
        out = user_out if user_out is not None else torch.empty((T, x.shape[1]), dtype=full.dtype,
                                                                device=full.device)
        if self.world_size == 1:
            return out.copy_(full) if user_out is not None else full
        dist.reduce_scatter_tensor(out, full, op=dist.ReduceOp.SUM, group=self.group)
        return out

    def forward(self, x, w13, w2, *, chunks: int = 1, **kw) -> torch.Tensor:
        """The layer's output on every rank.  ``chunks`` > 1 splits the batch into that many
        contiguous token ranges: the all-reduce of a range is issued asynchronously (NCCL runs it
        on its own stream) while the next range computes, so the exchange overlaps the GEMMs
        (every output row depends only on its own token, so the result is the same layer).
        With ``fused_allreduce`` the stages up to GEMM2 run, then one kernel per rank sums the
        local rows and all-reduces (with ``data_parallel``: reduce-scatters) them over peer
        memory; the result is then a symmetric buffer that the next call of the same T
        overwrites, unless ``out`` is given.  ``chunks`` applies to the NCCL all-reduce only."""
        if self.world_size > 1 and not (dist.is_available() and dist.is_initialized()):
            raise RuntimeError("forward of a rank of several needs the process group; use local_forward")
        if self.data_parallel:
            return self._data_parallel_forward(x, w13, w2, **kw)
        if self.fused_allreduce:
            return self._fused_forward(x.shape[0], x, w13, w2, **kw)
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
