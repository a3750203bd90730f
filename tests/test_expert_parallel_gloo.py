"""Host logic of the expert-parallel layer with real ranks: gloo process groups
on the CPU, 2 and 3 ranks.  Each rank's local part is replaced by the oracle's
partial for the rank's expert range (the CUDA library needs a B200); what runs
for real is the sharding, the per-rank problem, the weight slicing and the
all-reduce that completes the layer ("Hosting von Qwen auf Blackwell",
"Experten-Parallel")."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from moe_layer_top_b200 import inputs
from moe_layer_top_b200.expert_parallel import ExpertParallelMoE, expert_shard
from oracle import moe_oracle as O


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _OracleLocal(ExpertParallelMoE):
    """The rank-local part from the oracle (CPU); everything else is the product class."""

    def local_forward(self, x, w13, w2, out=None, **kw):
        p = self.problem_for(x.shape[0])
        assert p.T == x.shape[0] and w13.shape[0] == p.E == self.num_local and w2.shape[0] == p.E
        logits = kw.get("logits")
        assert logits is None or logits.shape == (p.T, self.E)
        r = O.moe_forward(x.double().numpy(), w13.double().numpy(), w2.double().numpy(), p.topk,
                          logits=None if logits is None else logits.numpy(),
                          expert_range=(p.first_expert, p.E))
        res = torch.from_numpy(r["out"]).to(torch.bfloat16)
        if out is None:
            return res
        out.copy_(res)
        return out


def _worker(rank, world, port, T, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        cfg = inputs.make_custom_config("ep_tiny", E=7, topk=3, H=256, I=128)
        w13, w2 = inputs.make_weights(cfg, 11)
        x = inputs.make_tokens(cfg, T, 11)
        logits = inputs.make_routing(cfg, T, 11)["logits"]
        layer = _OracleLocal(T, cfg.E, cfg.topk, cfg.H, cfg.I)
        out = layer.forward(x, layer.local_experts(w13), layer.local_experts(w2), logits=logits)
        # the chunked form: three token ranges, each all-reduced asynchronously
        chunked = layer.forward(x, layer.local_experts(w13), layer.local_experts(w2), logits=logits, chunks=3)
        torch.save({"out": out, "chunked": chunked, "first": layer.first_expert, "count": layer.num_local,
                    "problem": (layer.problem.E, layer.problem.num_global_experts, layer.problem.first_expert)},
                   os.path.join(out_dir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_expert_parallel_ranks_complete_the_layer(tmp_path, world):
    T = 9
    mp.spawn(_worker, args=(world, _free_port(), T, str(tmp_path)), nprocs=world, join=True)
    res = [torch.load(os.path.join(tmp_path, f"rank{r}.pt")) for r in range(world)]
    cfg = inputs.make_custom_config("ep_tiny", E=7, topk=3, H=256, I=128)
    # the ranks' ranges partition the experts and each rank's problem names its own
    assert [(r["first"], r["count"]) for r in res] == O.expert_shards(cfg.E, world)
    for r in res:
        assert r["problem"] == (r["count"], cfg.E, r["first"])
    # every rank ends with the same, complete layer
    w13, w2 = inputs.make_weights(cfg, 11)
    x = inputs.make_tokens(cfg, T, 11).double().numpy()
    logits = inputs.make_routing(cfg, T, 11)["logits"].numpy()
    full = O.moe_forward(x, w13.double().numpy(), w2.double().numpy(), cfg.topk, logits=logits)["out"]
    for r in res:
        torch.testing.assert_close(r["out"], res[0]["out"], rtol=0, atol=0)
        torch.testing.assert_close(r["chunked"], r["out"], rtol=0, atol=0)
    got = res[0]["out"].double().numpy()
    assert np.abs(got).max() > 0
    # partials rounded to bf16, summed in bf16 by the collective: a few bf16 ulps of the layer
    assert np.linalg.norm(got - full) <= 8e-3 * np.linalg.norm(full)


def test_expert_shard_matches_the_oracle_reading():
    for E, N in [(128, 8), (10, 4), (7, 3), (256, 16)]:
        assert [expert_shard(E, N, r) for r in range(N)] == O.expert_shards(E, N)
    with pytest.raises(ValueError):
        expert_shard(4, 5, 0)
    with pytest.raises(ValueError):
        expert_shard(8, 2, 2)


def _dp_worker(rank, world, port, T, out_dir):
    """Data parallel + expert parallel: rank r brings tokens [r*T, (r+1)*T) of one global batch."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        cfg = inputs.make_custom_config("ep_tiny", E=7, topk=3, H=256, I=128)
        w13, w2 = inputs.make_weights(cfg, 12)
        x = inputs.make_tokens(cfg, world * T, 12)[rank * T:(rank + 1) * T]
        logits = inputs.make_routing(cfg, world * T, 12)["logits"][rank * T:(rank + 1) * T]
        layer = _OracleLocal(T, cfg.E, cfg.topk, cfg.H, cfg.I, data_parallel=True)
        assert layer.problem.T == world * T                    # the share runs on the gathered batch
        out = layer.forward(x, layer.local_experts(w13), layer.local_experts(w2), logits=logits)
        torch.save({"out": out}, os.path.join(out_dir, f"dp{rank}.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_data_parallel_ranks_get_their_own_tokens(tmp_path, world):
    T = 5
    mp.spawn(_dp_worker, args=(world, _free_port(), T, str(tmp_path)), nprocs=world, join=True)
    cfg = inputs.make_custom_config("ep_tiny", E=7, topk=3, H=256, I=128)
    w13, w2 = inputs.make_weights(cfg, 12)
    x = inputs.make_tokens(cfg, world * T, 12).double().numpy()
    logits = inputs.make_routing(cfg, world * T, 12)["logits"].numpy()
    full = O.moe_forward(x, w13.double().numpy(), w2.double().numpy(), cfg.topk, logits=logits)["out"]
    for r in range(world):
        got = torch.load(os.path.join(tmp_path, f"dp{r}.pt"))["out"].double().numpy()
        ref = full[r * T:(r + 1) * T]
        assert got.shape == ref.shape and np.abs(ref).max() > 0
        assert np.linalg.norm(got - ref) <= 8e-3 * np.linalg.norm(ref)


def test_share_construction_without_a_group():
    """Shares chosen explicitly (no process group): ranges, per-share problems, weight slicing and
    the errors a caller can make."""
    w = torch.zeros((10, 4, 2))
    shares = [ExpertParallelMoE(6, 10, 3, 256, 128, rank=r, world_size=4) for r in range(4)]
    assert [(m.first_expert, m.num_local) for m in shares] == [(0, 2), (2, 3), (5, 2), (7, 3)]
    for m in shares:
        p = m.problem
        assert (p.T, p.E, p.num_global_experts, p.first_expert, p.topk) == (6, m.num_local, 10, m.first_expert, 3)
        assert m.local_experts(w).shape[0] == m.num_local
        assert m.local_experts(torch.arange(10))[0].item() == m.first_expert
        assert m.problem_for(17).T == 17 and m.problem_for(17) is m.problem_for(17)
    dp = ExpertParallelMoE(6, 10, 3, 256, 128, rank=1, world_size=4, data_parallel=True)
    assert dp.problem.T == 24                             # the share runs on the gathered batch
    with pytest.raises(ValueError):
        shares[0].local_experts(torch.zeros((9, 4)))
    with pytest.raises(ValueError):
        ExpertParallelMoE(6, 10, 3, 256, 128, rank=1)     # rank without world_size
    with pytest.raises(ValueError):
        ExpertParallelMoE(6, 3, 1, 256, 128, rank=0, world_size=4)   # more ranks than experts
    with pytest.raises(RuntimeError):
        shares[1].forward(torch.zeros((6, 256), dtype=torch.bfloat16), None, None)   # no process group


def test_multicast_switch_is_forced(monkeypatch):
    """The fused exchange's symmetric buffers are never bound to a multicast object: the switch is
    set to 1 when unset, and a caller's other value is an error, not silently kept."""
    from moe_layer_top_b200.expert_parallel import NO_MULTICAST_ENV, force_no_multicast
    monkeypatch.delenv(NO_MULTICAST_ENV, raising=False)
    force_no_multicast()
    assert os.environ[NO_MULTICAST_ENV] == "1"
    force_no_multicast()                                  # idempotent
    monkeypatch.setenv(NO_MULTICAST_ENV, "0")
    with pytest.raises(RuntimeError):
        force_no_multicast()
    assert os.environ[NO_MULTICAST_ENV] == "0"
