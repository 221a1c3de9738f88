"""Pins for the oracle's group-aware sigmoid top-k router (S1).

Definition ("Supporting MegaKernel for DeepSeek Models", layer table,
moe_topk_sigmoid_routing_layer: logits + bias -> topk_weight, indices;
num_groups=8, topk_group=4, routed_scaling_factor=2.5).  Readings: score =
sigmoid(logit); selection on score + bias; group score = sum of the group's
two best; weights = unbiased scores normalised over the chosen k, times the
scaling factor; ties go to the lower index.
"""
import itertools

import numpy as np
import torch

import oracle


def _sig32(lg):
    return (1.0 / (1.0 + np.exp(-lg.astype(np.float64)))).astype(np.float32)


def test_single_group_reduces_to_plain_topk():
    rng = np.random.default_rng(0)
    lg = rng.standard_normal((200, 64)).astype(np.float32)
    bias = (rng.standard_normal(64) * 0.1).astype(np.float32)
    idx, w = oracle.route_sigmoid_grouped(lg, bias, 1, 1, 6, 2.5)
    c = torch.from_numpy(_sig32(lg)) + torch.from_numpy(bias)
    ref = torch.sort(c, dim=1, descending=True, stable=True).indices[:, :6].numpy()
    assert np.array_equal(idx, ref)
    s = _sig32(lg)[np.arange(200)[:, None], idx].astype(np.float64)
    np.testing.assert_allclose(w, s / s.sum(1, keepdims=True) * 2.5, rtol=3e-7)
    np.testing.assert_allclose(w.sum(1), 2.5, rtol=1e-6)


def test_exhaustive_small_groups():
    """E=8 in 4 groups of 2, keep 2 groups, pick 3: brute force over subsets."""
    rng = np.random.default_rng(1)
    for trial in range(200):
        lg = rng.standard_normal((1, 8)).astype(np.float32)
        bias = (rng.standard_normal(8) * 0.3).astype(np.float32)
        idx, w = oracle.route_sigmoid_grouped(lg, bias, 4, 2, 3, 1.0)
        c = (_sig32(lg)[0] + bias).astype(np.float32)
        gscore = [float(np.float32(c[2 * g] + c[2 * g + 1])) for g in range(4)]
        groups = max(itertools.combinations(range(4), 2), key=lambda gs: sum(gscore[g] for g in gs))
        cand = [e for e in range(8) if e // 2 in groups]
        best = max(itertools.combinations(cand, 3), key=lambda es: sum(float(c[e]) for e in es))
        assert sorted(idx[0].tolist()) == sorted(best)
        assert all(c[idx[0][i]] >= c[idx[0][i + 1]] for i in range(2))


def test_group_score_is_sum_of_top_two():
    # group 0: {0.9, 0.0}, group 1: {0.8, 0.7}; top-1 would keep group 0,
    # the top-2 sum keeps group 1
    s = np.array([0.9, 0.0 + 1e-3, 0.8, 0.7], np.float64)
    lg = np.log(s / (1 - s)).astype(np.float32)[None]
    idx, _ = oracle.route_sigmoid_grouped(lg, np.zeros(4, np.float32), 2, 1, 1, 1.0)
    assert idx[0, 0] == 2


def test_bias_selects_but_does_not_weight():
    lg = np.zeros((1, 4), np.float32)          # all sigmoid = 0.5
    bias = np.array([0.0, 0.3, 0.0, 0.2], np.float32)
    idx, w = oracle.route_sigmoid_grouped(lg, bias, 1, 1, 2, 2.5)
    assert idx[0].tolist() == [1, 3]
    assert w[0].tolist() == [1.25, 1.25]


def test_ties_go_to_lower_index():
    lg = np.zeros((1, 16), np.float32)
    idx, w = oracle.route_sigmoid_grouped(lg, np.zeros(16, np.float32), 4, 2, 4, 1.0)
    assert idx[0].tolist() == [0, 1, 2, 3]
