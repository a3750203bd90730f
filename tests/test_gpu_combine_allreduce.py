"""The fused combine + all-reduce of expert parallelism ("Hosting von Qwen auf
Blackwell", "Experten-Parallel" and "All-Reduce"), on one B200: every rank's
part runs in ONE cooperative launch over all ranks' buffers in this GPU's
memory (the same device code and flag protocol as one launch per GPU; ranks
whose kernels wait on one another never run as separate launches here).

Checked: each rank's partial equals its share's own combine stage bit for bit;
every rank's out is the same and equals the bf16 rounding of the partials'
fp32 sum in rank order bit for bit; out matches the oracle's layer within the
layer tolerance; a second call with the next epoch reuses the flags; a rank
whose peer never runs gives up after the time limit with a status code and
leaves the context usable.
"""

import numpy as np
import pytest
import torch

from gpu_helpers import assert_close
from moe_layer_top_b200 import inputs, ops
from test_gpu_expert_parallel import Sharded

pytestmark = pytest.mark.gpu


def _run_shares(s, scatter=False):
    """Stages route .. GEMM2 of every rank's share, the share's own combine (for reference),
    and the per-rank buffers of the fused exchange (reduce-scatter: s.T is the gathered batch,
    out holds s.T / world rows)."""
    T, H = s.T, s.cfg.H
    T_out = T // s.world if scatter else T
    count = ops.combine_reduce_scatter_flag_count if scatter else ops.combine_allreduce_flag_count
    dev = torch.device("cuda")
    ranks, plain, probs = [], [], []
    for m in s.ranks:
        p, ws = m.problem_for(T), m.workspace_for(T, dev)
        sl = lambda w: None if w is None else m.local_experts(w)
        kw = dict(logits=s.routing.get("logits"), topk_ids=s.routing.get("topk_ids"),
                  topk_weights=s.routing.get("topk_weights"), w13_scale=sl(s.s13), w2_scale=sl(s.s2), ws=ws)
        ref = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        ops.forward_stages(p, s.x, sl(s.w13), sl(s.w2), ops.STAGE_ROUTE, ops.NUM_STAGES, out=ref, **kw)
        v = ops.workspace_views(p, ws)
        ranks.append(dict(y=v["y"], pos_of_flat=v["pos_of_flat"], status=v["status"],
                          partial=torch.full((T, H), float("nan"), dtype=torch.bfloat16, device=dev),
                          out=torch.full((T_out, H), float("nan"), dtype=torch.bfloat16, device=dev),
                          flags=torch.zeros(count(T_out, s.world), dtype=torch.int32, device=dev)))
        plain.append(ref)
        probs.append(p)
    torch.cuda.synchronize()
    return ranks, plain, probs


def _check(s, ranks, plain, probs, epoch, scatter=False):
    torch.cuda.synchronize()
    for r, p, m in zip(ranks, probs, s.ranks):
        assert ops.read_status(p, m.workspace_for(s.T, "cuda")) == ops.MOE_STATUS_OK
        nflags = r["flags"].numel()
        assert torch.all(r["flags"][:nflags - 1] == epoch) and int(r["flags"][nflags - 1]) == 0
    for r, ref in zip(ranks, plain):
        assert torch.equal(r["partial"], ref)                 # phase 1 is the share's combine
    total = torch.zeros((s.T, s.cfg.H), dtype=torch.float32, device="cuda")
    for r in ranks:
        total += r["partial"].float()                         # rank order, fp32, one rounding
    expect = total.to(torch.bfloat16)
    rows = s.T // s.world
    for i, r in enumerate(ranks):
        assert torch.equal(r["out"], expect[i * rows:(i + 1) * rows] if scatter else expect)


CASES = [
    ("decode_bf16", inputs.CONFIGS["decode_bf16"], 16, 4, {}),
    ("fp8_normal", inputs.make_custom_config("ar_fp8", E=16, topk=4, H=512, I=256, fp8=True, routing="logits",
                                             tokens=(300,)), 300, 2, dict(mode=ops.MODE_NORMAL)),
    ("mxfp8", inputs.make_custom_config("ar_mx", E=16, topk=4, H=512, I=256, fp8=True, mx=True, routing="logits",
                                        tokens=(200,)), 200, 4, {}),
    ("wide_router_8_ranks", inputs.make_custom_config("ar_wide", E=512, topk=8, H=256, I=128, routing="logits",
                                                      tokens=(64,)), 64, 8, {}),
    ("uneven_shards", inputs.make_custom_config("ar_uneven", E=10, topk=3, H=256, I=128, routing="logits",
                                                tokens=(33,)), 33, 4, {}),
    ("one_expert_per_rank_16", inputs.make_custom_config("ar_16", E=16, topk=2, H=384, I=128, routing="logits",
                                                         tokens=(40,)), 40, 16, dict(mode=ops.MODE_SWAP_AB)),
    ("many_chunks", inputs.make_custom_config("ar_chunks", E=8, topk=2, H=256, I=128, routing="logits",
                                              tokens=(3000,)), 3000, 2, {}),
]


@pytest.mark.parametrize("name,cfg,T,world,kw", CASES, ids=[c[0] for c in CASES])
def test_fused_combine_allreduce_emulated(name, cfg, T, world, kw):
    s = Sharded(cfg, T, world, seed=4, **kw)
    ranks, plain, probs = _run_shares(s)
    ops.combine_allreduce_emulated(T, cfg.topk, cfg.H, ranks, epoch=1)
    _check(s, ranks, plain, probs, 1)
    tokens = None if T <= 64 else np.sort(np.random.default_rng(0).choice(T, 48, replace=False))
    ref = s.oracle(tokens=tokens)["out"]
    got = ranks[0]["out"].float().cpu().numpy()
    assert_close(got if tokens is None else got[tokens], ref, cfg.fp8)
    # the next call reuses the flags: epoch 2, outputs rewritten from scratch
    for r in ranks:
        r["out"].fill_(float("nan"))
        r["partial"].fill_(float("nan"))
    ops.combine_allreduce_emulated(T, cfg.topk, cfg.H, ranks, epoch=2)
    _check(s, ranks, plain, probs, 2)


def test_rank_whose_peer_never_runs_gives_up():
    """Rank 0 of two runs alone: its wait for rank 1's chunks runs out after 20 ms, it records the
    site in its status word and returns; the context then runs the layer normally."""
    cfg = inputs.make_custom_config("ar_alone", E=8, topk=2, H=256, I=128, routing="logits", tokens=(24,))
    s = Sharded(cfg, 24, 2, seed=5)
    ranks, plain, probs = _run_shares(s)
    ops.combine_allreduce(24, cfg.topk, cfg.H, 0, ranks, epoch=1, timeout_us=20_000)
    torch.cuda.synchronize()
    st = ops.read_status(probs[0], s.ranks[0].workspace_for(24, "cuda"))
    assert st == (ops.MOE_STATUS_WAIT_TIMEOUT | 0x31)
    flags = ranks[0]["flags"]
    assert int(flags[-1]) == 1                                # the abort word holds the epoch
    assert torch.equal(ranks[0]["partial"], plain[0])         # its own part was done
    # the context is usable: the shares again, through the ordinary path
    again = s.run()
    for a, b in zip(again, plain):
        assert torch.equal(a, b)


RS_CASES = [
    ("decode_bf16", inputs.CONFIGS["decode_bf16"], 4, 4, {}),
    ("fp8_normal", inputs.make_custom_config("rs_fp8", E=16, topk=4, H=512, I=256, fp8=True, routing="logits",
                                             tokens=(300,)), 150, 2, dict(mode=ops.MODE_NORMAL)),
    ("wide_router_8_ranks", inputs.make_custom_config("rs_wide", E=512, topk=8, H=256, I=128, routing="logits",
                                                      tokens=(64,)), 8, 8, {}),
    ("uneven_shards", inputs.make_custom_config("rs_uneven", E=10, topk=3, H=256, I=128, routing="logits",
                                                tokens=(36,)), 9, 4, {}),
    ("many_chunks", inputs.make_custom_config("rs_chunks", E=8, topk=2, H=256, I=128, routing="logits",
                                              tokens=(3000,)), 1500, 2, {}),
]


@pytest.mark.parametrize("name,cfg,T,world,kw", RS_CASES, ids=[c[0] for c in RS_CASES])
def test_fused_combine_reduce_scatter_emulated(name, cfg, T, world, kw):
    """Data parallel + expert parallel: T tokens per rank, every share runs on the gathered batch of
    world * T tokens, each rank keeps the layer of its own rows."""
    s = Sharded(cfg, world * T, world, seed=7, **kw)
    ranks, plain, probs = _run_shares(s, scatter=True)
    ops.combine_reduce_scatter_emulated(T, cfg.topk, cfg.H, ranks, epoch=1)
    _check(s, ranks, plain, probs, 1, scatter=True)
    rows = np.arange(T) if T <= 64 else np.sort(np.random.default_rng(1).choice(T, 32, replace=False))
    for r in (0, world - 1):
        ref = s.oracle(tokens=r * T + rows)["out"]
        assert_close(ranks[r]["out"].float().cpu().numpy()[rows], ref, cfg.fp8)
    for r in ranks:
        r["out"].fill_(float("nan"))
    ops.combine_reduce_scatter_emulated(T, cfg.topk, cfg.H, ranks, epoch=2)
    _check(s, ranks, plain, probs, 2, scatter=True)


_SYMMETRIC_CHILD = r"""
import os, sys
import torch
import torch.distributed as dist
sys.path.insert(0, os.environ["MOE_TEST_ROOT"])
from moe_layer_top_b200 import inputs, ops
from moe_layer_top_b200.expert_parallel import ExpertParallelMoE

torch.cuda.set_device(0)
dist.init_process_group("nccl", rank=0, world_size=1, init_method="tcp://127.0.0.1:" + os.environ["MOE_TEST_PORT"],
                        device_id=torch.device("cuda:0"))
cfg = inputs.make_custom_config("ar_symm", E=16, topk=4, H=512, I=256, routing="logits", tokens=(40,))
T, dev = 40, torch.device("cuda:0")
w13, w2 = inputs.make_weights(cfg, 6, device=dev)
x = inputs.make_tokens(cfg, T, 6, device=dev)
logits = inputs.make_routing(cfg, T, 6, device=dev)["logits"]
plain = ops.fused_forward(ops.problem(T, cfg.E, cfg.topk, cfg.H, cfg.I), x, w13, w2, logits=logits)
m = ExpertParallelMoE(T, cfg.E, cfg.topk, cfg.H, cfg.I, fused_allreduce=True)
a = m.forward(x, w13, w2, logits=logits).clone()
b = m.forward(x, w13, w2, logits=logits, out=torch.empty_like(plain))
torch.cuda.synchronize()
assert torch.equal(a, plain) and torch.equal(b, plain), "fused path differs from the plain layer"
flags = m._exchange[T]["flags"]
assert int(flags[:-1].min()) == 2 and int(flags[:-1].max()) == 2 and int(flags[-1]) == 0, flags
assert ops.read_status(m.problem, m.workspace_for(T, dev)) == ops.MOE_STATUS_OK
# data parallel + expert parallel, fused reduce-scatter and the NCCL form
m2 = ExpertParallelMoE(T, cfg.E, cfg.topk, cfg.H, cfg.I, fused_allreduce=True, data_parallel=True)
c = m2.forward(x, w13, w2, logits=logits).clone()
m3 = ExpertParallelMoE(T, cfg.E, cfg.topk, cfg.H, cfg.I, data_parallel=True)
d = m3.forward(x, w13, w2, logits=logits)
torch.cuda.synchronize()
assert torch.equal(c, plain) and torch.equal(d, plain), "data-parallel paths differ from the plain layer"
del m, m2, m3, a, b, c, d
torch.cuda.synchronize()
dist.destroy_process_group()
print("SYMMETRIC-OK")
"""


def test_fused_allreduce_through_symmetric_memory_one_rank():
    """The production wiring (symmetric buffers, rendezvous, peer addresses, epochs) on a one-rank
    NCCL group: the fused kernel then reduces one partial, so the result is the plain layer bit for
    bit.  Run in a child process so its process group ends with it."""
    import os
    import socket
    import subprocess
    import sys
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, MOE_TEST_ROOT=root, MOE_TEST_PORT=str(port), MASTER_ADDR="127.0.0.1",
               TORCH_SYMM_MEM_DISABLE_MULTICAST="1", NCCL_NVLS_ENABLE="0")
    res = subprocess.run([sys.executable, "-c", _SYMMETRIC_CHILD], env=env, capture_output=True, text=True,
                         timeout=240)
    assert res.returncode == 0 and "SYMMETRIC-OK" in res.stdout, (res.stdout[-2000:], res.stderr[-3000:])
