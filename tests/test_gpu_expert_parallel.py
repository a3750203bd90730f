"""Expert parallelism on one B200: every rank's share of the layer run in turn
through the C ABI ("Hosting von Qwen auf Blackwell", "Experten-Parallel":
replicated inputs, each rank accumulates its own experts, an all-reduce sums
the ranks).  Checked against the oracle:

* routing (global ids) and each rank's alignment bit-exact;
* each rank's partial output within the layer tolerance of the oracle's
  partial for the same expert range;
* the sum of the partials (the all-reduce, here one fp32 sum on the device)
  within the layer tolerance of the oracle's layer;
* edge cases: a rank no token reaches, an invalid global id, the persistent
  decode switch (not taken for a rank's share), top-1 with the router weight
  on the input.
"""

import numpy as np
import pytest
import torch

from gpu_helpers import LazyExperts, assert_close
from moe_layer_top_b200 import inputs, ops
from moe_layer_top_b200.expert_parallel import ExpertParallelMoE
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


class _Shifted:
    """Local expert e of a rank -> global expert first + e of a lazy oracle table."""

    def __init__(self, table, first):
        self.table, self.first = table, first

    def __getitem__(self, e):
        return self.table[self.first + int(e)]


class Sharded:
    """A workload on the GPU, its weights quantised once, split over `world` emulated ranks."""

    def __init__(self, cfg, T, world, seed=0, routing=None, **problem_kw):
        dev = torch.device("cuda")
        self.cfg, self.T, self.world = cfg, T, world
        self.w13_bf16, self.w2_bf16 = inputs.make_weights(cfg, seed, device=dev)
        self.x = inputs.make_tokens(cfg, T, seed, device=dev)
        self.routing = routing if routing is not None else inputs.make_routing(cfg, T, seed, device=dev)
        if cfg.mx:
            self.w13, self.s13 = ops.quantize_weights_mxfp8(self.w13_bf16)
            self.w2, self.s2 = ops.quantize_weights_mxfp8(self.w2_bf16)
        elif cfg.fp8:
            self.w13, self.s13 = ops.quantize_weights_fp8(self.w13_bf16)
            self.w2, self.s2 = ops.quantize_weights_fp8(self.w2_bf16)
        else:
            self.w13, self.w2, self.s13, self.s2 = self.w13_bf16, self.w2_bf16, None, None
        self.problem_kw = dict(fp8=cfg.fp8, mx=cfg.mx, **problem_kw)
        self.ranks = [ExpertParallelMoE(T, cfg.E, cfg.topk, cfg.H, cfg.I, rank=r, world_size=world,
                                        **self.problem_kw) for r in range(world)]
        self.l13 = LazyExperts(self.w13_bf16, cfg.fp8, cfg.mx)
        self.l2 = LazyExperts(self.w2_bf16, cfg.fp8, cfg.mx)

    def run(self):
        parts = []
        for m in self.ranks:
            sl = lambda w: None if w is None else m.local_experts(w)
            out = m.local_forward(self.x, sl(self.w13), sl(self.w2), logits=self.routing.get("logits"),
                                  topk_ids=self.routing.get("topk_ids"),
                                  topk_weights=self.routing.get("topk_weights"), w13_scale=sl(self.s13),
                                  w2_scale=sl(self.s2))
            parts.append(out.clone())
        torch.cuda.synchronize()
        return parts

    def oracle(self, expert_range=None, tokens=None):
        kw = {}
        if "logits" in self.routing:
            kw["logits"] = self.routing["logits"].cpu().numpy()
        else:
            kw["topk_ids"] = self.routing["topk_ids"].cpu().numpy()
            kw["topk_weights"] = self.routing["topk_weights"].cpu().numpy()
        kw["router_weight_on_input"] = self.problem_kw.get("router_weight_on_input", False)
        first = 0 if expert_range is None else expert_range[0]
        w13, w2 = _Shifted(self.l13.codes, first), _Shifted(self.l2.codes, first)
        if self.cfg.fp8:
            kw.update(w13_scale=_Shifted(self.l13.scales, first), w2_scale=_Shifted(self.l2.scales, first),
                      mx=self.cfg.mx)
        x = self.x.float().cpu().double().numpy()
        return O.moe_forward(x, w13, w2, self.cfg.topk, tokens=tokens, expert_range=expert_range, **kw)


def _check_routing_and_alignment(s, m, ref_ids):
    v = ops.workspace_views(m.problem, m.workspace_for(s.T, "cuda"))
    q = v["problem"]
    if "logits" in s.routing:
        np.testing.assert_array_equal(v["topk_ids"].cpu().numpy(), ref_ids)
    ref = O.align(ref_ids, q.E, q.block_m, first_expert=m.first_expert, num_global_experts=s.cfg.E)
    ntpp = int(v["num_tokens_post_padded"].item())
    assert ntpp == ref["num_tokens_post_padded"]
    np.testing.assert_array_equal(v["sorted_token_ids"].cpu().numpy()[:ntpp], ref["sorted_token_ids"][:ntpp])
    np.testing.assert_array_equal(v["expert_ids"].cpu().numpy()[:ntpp // q.block_m],
                                  ref["expert_ids"][:ntpp // q.block_m])
    np.testing.assert_array_equal(v["expert_counts"].cpu().numpy(), ref["expert_counts"])
    pos = v["pos_of_flat"].cpu().numpy()
    local = (ref_ids.reshape(-1) >= m.first_expert) & (ref_ids.reshape(-1) < m.first_expert + q.E)
    assert np.all(pos[~local] == -1)
    st = v["sorted_token_ids"].cpu().numpy()
    np.testing.assert_array_equal(st[pos[local]], np.nonzero(local)[0])
    assert ops.read_status(m.problem, m.workspace_for(s.T, "cuda")) == ops.MOE_STATUS_OK


CASES = [
    # (name, config, T, world, problem options)
    ("decode_bf16_swap", inputs.CONFIGS["decode_bf16"], 16, 4, {}),
    ("fp8_normal", inputs.make_custom_config("ep_fp8", E=16, topk=4, H=512, I=256, fp8=True,
                                             routing="logits", tokens=(300,)), 300, 2,
     dict(mode=ops.MODE_NORMAL)),
    ("fp8_swap_split", inputs.make_custom_config("ep_fp8s", E=16, topk=4, H=512, I=256, fp8=True,
                                                 routing="uniform_ids", tokens=(37,)), 37, 4,
     dict(mode=ops.MODE_SWAP_AB)),
    ("mxfp8", inputs.make_custom_config("ep_mx", E=16, topk=4, H=512, I=256, fp8=True, mx=True,
                                        routing="logits", tokens=(200,)), 200, 4, {}),
    ("wide_router_multi_cta_align", inputs.make_custom_config("ep_wide", E=512, topk=8, H=256, I=128,
                                                              routing="logits", tokens=(64,)), 64, 8, {}),
    ("uneven_shards", inputs.make_custom_config("ep_uneven", E=10, topk=3, H=256, I=128,
                                                routing="logits", tokens=(33,)), 33, 4, {}),
]


@pytest.mark.parametrize("name,cfg,T,world,kw", CASES, ids=[c[0] for c in CASES])
def test_expert_parallel_shares_and_sum(name, cfg, T, world, kw):
    s = Sharded(cfg, T, world, seed=3, **kw)
    parts = s.run()
    full_ref = s.oracle()
    ref_ids = full_ref["topk_ids"]
    for m, part in zip(s.ranks, parts):
        _check_routing_and_alignment(s, m, ref_ids)
        ref = s.oracle(expert_range=(m.first_expert, m.num_local))["out"]
        got = part.float().cpu().numpy()
        if np.abs(ref).max() == 0:
            assert np.all(got == 0)
        else:
            assert_close(got, ref, cfg.fp8)
    total = torch.stack([p.float() for p in parts]).sum(0).to(torch.bfloat16)
    assert_close(total.float().cpu().numpy(), full_ref["out"], cfg.fp8)


def test_rank_without_tokens_writes_zeros():
    cfg = inputs.make_custom_config("ep_skew", E=8, topk=2, H=256, I=128, routing="uniform_ids", tokens=(20,))
    dev = torch.device("cuda")
    ids = torch.randint(0, 4, (20, 2), generator=torch.Generator(device=dev).manual_seed(1), device=dev,
                        dtype=torch.int32)                       # every id on the first half of the experts
    w = torch.full((20, 2), 0.5, device=dev)
    s = Sharded(cfg, 20, 2, seed=1, routing={"topk_ids": ids, "topk_weights": w})
    parts = s.run()
    assert torch.count_nonzero(parts[1]).item() == 0
    assert ops.read_status(s.ranks[1].problem, s.ranks[1].workspace_for(s.T, "cuda")) == ops.MOE_STATUS_OK
    assert_close(parts[0].float().cpu().numpy(), s.oracle()["out"], False)


def test_invalid_global_id_is_reported_and_skipped():
    cfg = inputs.make_custom_config("ep_bad", E=8, topk=2, H=256, I=128, routing="uniform_ids", tokens=(12,))
    dev = torch.device("cuda")
    ids = torch.randint(0, 8, (12, 2), generator=torch.Generator(device=dev).manual_seed(2), device=dev,
                        dtype=torch.int32)
    ids[3, 1] = 8                                                # outside [0, num_global_experts)
    w = torch.full((12, 2), 0.5, device=dev)
    s = Sharded(cfg, 12, 2, seed=2, routing={"topk_ids": ids, "topk_weights": w})
    s.run()
    for m in s.ranks:
        assert ops.read_status(m.problem, m.workspace_for(s.T, "cuda")) == ops.MOE_STATUS_BAD_EXPERT_ID
        pos = ops.workspace_views(m.problem, m.workspace_for(s.T, "cuda"))["pos_of_flat"].cpu().numpy()
        assert pos[3 * 2 + 1] == -1


def test_persistent_decode_switch_is_not_taken_for_a_share():
    cfg = inputs.CONFIGS["decode_bf16"]
    a = Sharded(cfg, 4, 2, seed=5)
    b = Sharded(cfg, 4, 2, seed=5, persistent_decode=True)
    for m, pa, pb in zip(b.ranks, a.run(), b.run()):
        assert torch.equal(pa, pb)                               # the same stage pipeline ran
        assert_close(pb.float().cpu().numpy(), b.oracle(expert_range=(m.first_expert, m.num_local))["out"], False)


def test_router_weight_on_input_top1():
    cfg = inputs.make_custom_config("ep_top1", E=8, topk=1, H=256, I=128, fp8=True, routing="logits",
                                    tokens=(24,))
    s = Sharded(cfg, 24, 2, seed=6, router_weight_on_input=True, mode=ops.MODE_SWAP_AB)
    parts = s.run()
    for m, part in zip(s.ranks, parts):
        assert_close(part.float().cpu().numpy(), s.oracle(expert_range=(m.first_expert, m.num_local))["out"], True)


def test_one_share_is_the_plain_layer_bit_for_bit():
    cfg = inputs.CONFIGS["decode_bf16"]
    s = Sharded(cfg, 16, 1, seed=7)
    part = s.run()[0]
    p = ops.problem(16, cfg.E, cfg.topk, cfg.H, cfg.I)
    plain = ops.fused_forward(p, s.x, s.w13, s.w2, logits=s.routing["logits"])
    torch.cuda.synchronize()
    assert torch.equal(part, plain)


def test_chunked_forward_is_the_layer():
    """forward(chunks=3) on one rank: three token ranges, each its own problem and workspace."""
    cfg = inputs.make_custom_config("ep_chunks", E=16, topk=4, H=512, I=256, fp8=True, routing="logits",
                                    tokens=(50,))
    s = Sharded(cfg, 50, 1, seed=8)
    m = s.ranks[0]
    kw = dict(logits=s.routing["logits"], w13_scale=s.s13, w2_scale=s.s2)
    whole = m.forward(s.x, s.w13, s.w2, **kw).clone()
    chunked = m.forward(s.x, s.w13, s.w2, chunks=3, **kw)
    torch.cuda.synchronize()
    ref = s.oracle()["out"]
    assert_close(chunked.float().cpu().numpy(), ref, True)
    assert_close(whole.float().cpu().numpy(), ref, True)
    assert sorted(m._problems) == [16, 17, 50]


def test_share_of_a_token_range_is_those_rows():
    cfg = inputs.make_custom_config("ep_rows", E=12, topk=3, H=256, I=128, routing="logits", tokens=(40,))
    s = Sharded(cfg, 40, 3, seed=9)
    s.run()
    m = s.ranks[1]
    sub = m.local_forward(s.x[8:29], m.local_experts(s.w13), m.local_experts(s.w2),
                          logits=s.routing["logits"][8:29])
    torch.cuda.synchronize()
    ref = s.oracle(expert_range=(m.first_expert, m.num_local), tokens=np.arange(8, 29))["out"]
    assert_close(sub.float().cpu().numpy(), ref, False)
