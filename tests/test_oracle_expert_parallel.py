"""Pins of the oracle's expert-parallel reading ("Hosting von Qwen auf
Blackwell", "MoE Dispatch - Combine" / "Experten-Parallel": replicated inputs,
each rank accumulates its own experts' contributions, an all-reduce sums them).

* the shard ranges partition the experts (hand-worked examples);
* a shard's alignment equals the matching segments of the full alignment;
* a shard's partial output equals the dense brute force with the other
  ranks' assignments masked out;
* the partials sum to the full layer within bf16 rounding, and one rank is
  the full layer bit for bit.
"""

import numpy as np
import pytest

from moe_layer_top_b200 import inputs
from oracle import moe_oracle as O
from test_oracle_mlp import _dense_reference


def test_expert_shards_examples():
    assert O.expert_shards(128, 8) == [(16 * r, 16) for r in range(8)]
    assert O.expert_shards(10, 4) == [(0, 2), (2, 3), (5, 2), (7, 3)]
    assert O.expert_shards(5, 1) == [(0, 5)]
    for E, N in [(128, 3), (7, 7), (256, 16), (9, 2)]:
        sh = O.expert_shards(E, N)
        covered = np.concatenate([np.arange(f, f + c) for f, c in sh])
        np.testing.assert_array_equal(covered, np.arange(E))
        sizes = [c for _, c in sh]
        assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    with pytest.raises(ValueError):
        O.expert_shards(4, 5)


@pytest.mark.parametrize("block_m", [1, 4, 16])
def test_shard_alignment_is_the_full_alignment_restricted(block_m):
    rng = np.random.default_rng(7)
    E, T, k = 12, 40, 3
    ids = rng.integers(0, E, size=(T, k))
    ids[5] = [4, 4, 4]
    full = O.align(ids, E, block_m)
    fo = full["expert_offsets"]
    for first, count in O.expert_shards(E, 3):
        sh = O.align(ids, count, block_m, first_expert=first, num_global_experts=E)
        np.testing.assert_array_equal(sh["expert_counts"], full["expert_counts"][first:first + count])
        so = sh["expert_offsets"]
        for e in range(count):
            c = sh["expert_counts"][e]
            g = first + e
            np.testing.assert_array_equal(sh["sorted_token_ids"][so[e]:so[e] + c],
                                          full["sorted_token_ids"][fo[g]:fo[g] + c])
        # every slot that is not a local assignment holds the sentinel
        n = T * k
        real = np.concatenate([np.arange(so[e], so[e] + sh["expert_counts"][e]) for e in range(count)])
        pad = np.setdiff1d(np.arange(sh["capacity"]), real)
        assert np.all(sh["sorted_token_ids"][pad] == n)
        assert sh["num_tokens_post_padded"] == so[count]
    with pytest.raises(ValueError):
        O.align(np.array([[E]]), 4, block_m, first_expert=0, num_global_experts=E)


def _tiny_fp8_case(seed=4):
    cfg = inputs.make_custom_config("tiny_ep", E=6, topk=3, H=256, I=256, fp8=True,
                                    routing="uniform_ids", tokens=(12,))
    w13, w2 = inputs.make_weights(cfg, seed)
    x = inputs.make_tokens(cfg, 12, seed).double().numpy()
    r = inputs.make_routing(cfg, 12, seed)
    ids = r["topk_ids"].numpy().copy()
    ids[0] = [2, 2, 2]
    ids[1] = [0, 1, 0]                       # a token with no expert on the last shards
    wts = r["topk_weights"].numpy()
    q13, s13 = O.quantize_weight_block128(w13.double().numpy())
    q2, s2 = O.quantize_weight_block128(w2.double().numpy())
    return cfg, x, ids, wts, q13, s13, q2, s2


def test_shard_partial_matches_masked_dense_bruteforce():
    cfg, x, ids, wts, q13, s13, q2, s2 = _tiny_fp8_case()
    for first, count in O.expert_shards(cfg.E, 3):
        sl = slice(first, first + count)
        part = O.moe_forward(x, q13[sl], q2[sl], cfg.topk, topk_ids=ids, topk_weights=wts,
                             w13_scale=s13[sl], w2_scale=s2[sl], expert_range=(first, count))["out"]
        local = (ids >= first) & (ids < first + count)
        ref = _dense_reference(x, q13[sl], q2[sl], np.where(local, ids - first, 0),
                               np.where(local, wts, 0.0), fp8=True, w13_scale=s13[sl], w2_scale=s2[sl])
        np.testing.assert_array_equal(part, ref)
        if first >= 2:
            assert np.all(part[1] == 0.0)        # token 1 has no expert here


@pytest.mark.parametrize("world", [2, 3, 6])
def test_partials_sum_to_the_layer(world):
    cfg, x, ids, wts, q13, s13, q2, s2 = _tiny_fp8_case(5)
    full = O.moe_forward(x, q13, q2, cfg.topk, topk_ids=ids, topk_weights=wts, w13_scale=s13, w2_scale=s2)["out"]
    ep = O.moe_forward_expert_parallel(x, q13, q2, cfg.topk, world, topk_ids=ids, topk_weights=wts,
                                       w13_scale=s13, w2_scale=s2)
    assert len(ep["partials"]) == world
    # each partial is one bf16 rounding (2^-9 relative) of its exact sum, and so is each result
    mag = np.sum(np.abs(ep["partials"]), axis=0)
    bound = 2.0 ** -8 * (mag + np.abs(full)) + 1e-30
    assert np.all(np.abs(ep["out"] - full) <= bound)
    assert np.abs(full).max() > 0


def test_one_rank_is_the_layer_bit_for_bit():
    cfg = inputs.CONFIGS["tiny"]
    w13, w2 = inputs.make_weights(cfg, 2)
    x = inputs.make_tokens(cfg, 16, 2).double().numpy()
    logits = inputs.make_routing(cfg, 16, 2)["logits"].numpy()
    w13n, w2n = w13.double().numpy(), w2.double().numpy()
    full = O.moe_forward(x, w13n, w2n, cfg.topk, logits=logits)["out"]
    one = O.moe_forward_expert_parallel(x, w13n, w2n, cfg.topk, 1, logits=logits)
    np.testing.assert_array_equal(one["out"], full)
    every = O.moe_forward(x, w13n, w2n, cfg.topk, logits=logits, expert_range=(0, cfg.E))["out"]
    np.testing.assert_array_equal(every, full)
