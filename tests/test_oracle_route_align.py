"""Pins of the oracle's router and alignment: brute force on small inputs,
a torch library path for the weights, and the invariants of the method."""

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O


def _brute_route_ids(logits, k):
    t, e = logits.shape
    return np.array([sorted(range(e), key=lambda j: (-float(logits[r, j]), j))[:k] for r in range(t)],
                    dtype=np.int32)


@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (16, 8, 2), (37, 128, 8), (5, 256, 8), (3, 4, 4)])
def test_route_matches_brute_force_and_torch(T, E, k):
    rng = np.random.default_rng(T * 1000 + E)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    # plant exact ties so that the lower index must win
    logits[0, E - 1] = logits[0, 0]
    if T > 1:
        logits[1, :] = 0.5
    ids, w = O.route(logits, k)
    np.testing.assert_array_equal(ids, _brute_route_ids(logits, k))
    # weights: torch's softmax, the chosen entries, renormalised (float64 library path)
    p = torch.softmax(torch.from_numpy(logits).double(), dim=-1)
    chosen = torch.gather(p, 1, torch.from_numpy(ids).long())
    ref = (chosen / chosen.sum(-1, keepdim=True)).float().numpy()
    np.testing.assert_allclose(w, ref, rtol=1e-6, atol=0)
    np.testing.assert_allclose(w.astype(np.float64).sum(-1), 1.0, atol=k * 2.0 ** -23)
    assert np.all(np.diff(w, axis=1) <= 0), "weights follow the descending logits"
    # without renormalisation the weights are the plain softmax probabilities
    _, w_raw = O.route(logits, k, renormalize=False)
    np.testing.assert_allclose(w_raw, chosen.float().numpy(), rtol=1e-6)


def test_route_all_equal_logits_picks_lowest_indices():
    ids, w = O.route(np.zeros((2, 16), dtype=np.float32), 4)
    np.testing.assert_array_equal(ids, [[0, 1, 2, 3]] * 2)
    np.testing.assert_allclose(w, 0.25)


def _brute_align(ids, E, bm):
    """Counting sort written as the dumbest loop: walk experts, then flat ids."""
    flat = [int(v) for v in np.asarray(ids).reshape(-1)]
    n = len(flat)
    sorted_ids, expert_of_block = [], []
    for e in range(E):
        members = [f for f in range(n) if flat[f] == e]
        if not members:
            continue
        while len(members) % bm:
            members.append(n)
        for b in range(len(members) // bm):
            expert_of_block.append(e)
        sorted_ids += members
    return sorted_ids, expert_of_block


@pytest.mark.parametrize("T,E,k,bm,dist", [
    (16, 8, 2, 16, "uniform"), (1, 128, 8, 16, "uniform"), (4, 128, 8, 32, "uniform"),
    (64, 128, 8, 64, "uniform"), (100, 16, 4, 128, "dup"), (33, 256, 8, 16, "skew"),
    (7, 1, 1, 16, "uniform"), (50, 8, 8, 16, "dup"),
])
def test_align_matches_brute_force(T, E, k, bm, dist):
    rng = np.random.default_rng(T + 7 * E + bm)
    if dist == "uniform":
        ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]) if k <= E else None
    elif dist == "dup":                                       # with replacement: repeats allowed
        ids = rng.integers(0, E, (T, k))
    else:                                                     # a few hot experts, many empty ones
        ids = np.minimum(rng.zipf(1.5, (T, k)) - 1, E - 1)
    ids = ids.astype(np.int32)
    a = O.align(ids, E, bm)
    ref_sorted, ref_blocks = _brute_align(ids, E, bm)
    ntpp = a["num_tokens_post_padded"]
    assert ntpp == len(ref_sorted)
    np.testing.assert_array_equal(a["sorted_token_ids"][:ntpp], ref_sorted)
    np.testing.assert_array_equal(a["expert_ids"][:ntpp // bm], ref_blocks)
    # invariants
    n = T * k
    cap = a["capacity"]
    assert cap == O.align_capacity(T, k, E, bm) and cap % bm == 0 and cap >= ntpp
    assert np.all(a["sorted_token_ids"][ntpp:] == n)
    assert np.all(a["expert_ids"][ntpp // bm:] == -1)
    real = a["sorted_token_ids"][a["sorted_token_ids"] != n]
    np.testing.assert_array_equal(np.sort(real), np.arange(n))          # a permutation
    assert a["expert_counts"].sum() == n
    assert np.all(a["expert_offsets"] % bm == 0)
    np.testing.assert_array_equal(np.diff(a["expert_offsets"]),
                                  -(-a["expert_counts"] // bm) * bm)
    flat = ids.reshape(-1)
    for b in range(ntpp // bm):                                         # one expert per block
        blk = a["sorted_token_ids"][b * bm:(b + 1) * bm]
        assert np.all(flat[blk[blk != n]] == a["expert_ids"][b])


def test_align_capacity_bound_is_tight_for_single_token_per_expert():
    # every expert gets exactly one assignment: each pads to a whole block
    ids = np.arange(8, dtype=np.int32).reshape(1, 8)
    a = O.align(ids, 128, 16)
    assert a["num_tokens_post_padded"] == 8 * 16 == a["capacity"]


def test_align_empty_input():
    a = O.align(np.zeros((0, 8), dtype=np.int32), 128, 16)
    assert a["num_tokens_post_padded"] == 0 and a["capacity"] == 0


def test_identity_expert_through_align_reproduces_x():
    """With f_e(x) = x for every expert, gather -> sort -> scatter -> weighted
    combine must give back x (the weights of a row sum to one)."""
    rng = np.random.default_rng(9)
    T, E, k, bm = 40, 16, 4, 16
    x = O.round_bf16(rng.standard_normal((T, 64)))
    ids = rng.integers(0, E, (T, k)).astype(np.int32)
    z = rng.standard_normal((T, k))
    w = (np.exp(z) / np.exp(z).sum(1, keepdims=True)).astype(np.float32)
    a = O.align(ids, E, bm)
    s = a["sorted_token_ids"]
    y = np.zeros((T * k, 64))
    for r in range(a["num_tokens_post_padded"]):
        if s[r] != T * k:
            y[s[r]] = x[s[r] // k]                  # identity expert on the gathered row
    out = (w.astype(np.float64)[:, :, None] * y.reshape(T, k, 64)).sum(1)
    np.testing.assert_allclose(out, x, rtol=1e-6, atol=1e-7)


def test_align_random_shapes_match_brute_force():
    """Sixty random (T, E, k, BM, id distribution) draws, including empty and single-expert cases,
    against the counting sort written as a loop."""
    rng = np.random.default_rng(2024)
    for case in range(60):
        E = int(rng.integers(1, 65))
        k = int(rng.integers(1, min(8, E) + 1))
        T = int(rng.integers(0, 41))
        bm = int(rng.choice([16, 32, 64, 128]))
        kind = case % 3
        if kind == 0 and T > 0:
            ids = np.stack([rng.permutation(E)[:k] for _ in range(T)])
        elif kind == 1:
            ids = rng.integers(0, E, (T, k))
        else:
            ids = np.minimum(rng.zipf(1.3, (T, k)) - 1, E - 1)
        ids = np.asarray(ids, dtype=np.int32).reshape(T, k)
        a = O.align(ids, E, bm)
        ref_sorted, ref_blocks = _brute_align(ids, E, bm)
        ntpp = a["num_tokens_post_padded"]
        assert ntpp == len(ref_sorted), case
        np.testing.assert_array_equal(a["sorted_token_ids"][:ntpp], ref_sorted, err_msg=str(case))
        np.testing.assert_array_equal(a["expert_ids"][:ntpp // bm], ref_blocks, err_msg=str(case))
        assert a["capacity"] == O.align_capacity(T, k, E, bm) >= ntpp
        np.testing.assert_array_equal(a["expert_counts"], np.bincount(ids.reshape(-1), minlength=E))
