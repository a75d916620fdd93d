"""Pins of the oracle's pooling and hierarchical Top-K selection.

Each test checks the oracle against something other than itself: closed forms,
brute force written a different way, or the pages' worked examples (fixtures
under tests/golden/, each with its citation).
"""

import json
import os

import numpy as np
import pytest

import oracle
from hierarchical_top_sparse_llsa_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_examples.json")


def _pixel_xy(t):
    """Z-order decode by direct bit picking (x: bits 0,2,4..; y: bits 1,3,5..)."""
    x = y = 0
    for b in range(16):
        x += ((t >> (2 * b)) & 1) << b
        y += ((t >> (2 * b + 1)) & 1) << b
    return x, y


# ----------------------------------------------------------------- pooling
def test_pool_constant_is_constant():
    X = np.full((1, 2, 4096, 8), 1.5, dtype=np.float32)
    pyr = oracle.pool(X, 3)
    for l in (1, 2, 3):
        assert pyr[l].shape == (1, 2, 4096 // 16**l, 8)
        assert np.all(pyr[l] == np.float32(1.5))


def test_pool_zorder_ramp_gives_tile_centroids():
    # channel 0 holds the pixel x, channel 1 the pixel y; a level-l token is a
    # 4**l x 4**l pixel tile whose mean coordinate is origin + (4**l - 1) / 2.
    N = 4096
    X = np.zeros((1, 1, N, 2), dtype=np.float32)
    for t in range(N):
        X[0, 0, t] = _pixel_xy(t)
    pyr = oracle.pool(X, 3)
    for l in (1, 2, 3):
        side = 4**l
        for t in range(N // 16**l):
            x0, y0 = _pixel_xy(t * 16**l)
            assert x0 % side == 0 and y0 % side == 0
            assert pyr[l][0, 0, t, 0] == x0 + (side - 1) / 2
            assert pyr[l][0, 0, t, 1] == y0 + (side - 1) / 2


def test_pool_matches_fp64_direct_mean_within_rounding_bound():
    rng = np.random.default_rng(7)
    X = rng.standard_normal((2, 3, 4096, 16)).astype(np.float32)
    pyr = oracle.pool(X, 3)
    for l in (1, 2, 3):
        span = 16**l
        g = X.astype(np.float64).reshape(2, 3, 4096 // span, span, 16)
        exact = g.mean(axis=3)
        # each level adds at most 15 roundings of relative size 2^-24 on sums
        # of absolute values, plus the final rounding of the stored mean
        bound = (15 * l + 1) * 2.0**-24 * np.abs(g).mean(axis=3) * 1.01 + 1e-30
        assert np.all(np.abs(pyr[l] - exact) <= bound)


def test_pool_factor2_levels_page_example():
    ex = json.load(open(GOLDEN))["pool_levels_factor2"]
    X = np.arange(ex["N"], dtype=np.float32).reshape(1, 1, ex["N"], 1)
    pyr = oracle.pool(X, ex["L"], factor=ex["factor"])
    sizes = [ex["N"]] + [pyr[l].shape[2] for l in range(1, ex["L"] + 1)]
    assert sizes == ex["tokens_per_level"]
    assert list(pyr[1][0, 0, :, 0]) == [0.5, 2.5, 4.5, 6.5]
    assert list(pyr[2][0, 0, :, 0]) == [1.5, 5.5]


# --------------------------------------------------------------- selection
def _brute_topk(qrow, keys, cand, k):
    """Top-k of exact scores by Python sorting: score descending, index ascending."""
    scored = sorted(((-float(np.dot(qrow, keys[c])), int(c)) for c in cand))
    kept = sorted(c for _, c in scored[:k])
    return kept + [-1] * (k - len(kept))


def _integer_inputs(seed, B, H, N, D, lo=-3, hi=3):
    rng = np.random.default_rng(seed)
    q = rng.integers(lo, hi + 1, size=(B, H, N, D)).astype(np.float32)
    k = rng.integers(lo, hi + 1, size=(B, H, N, D)).astype(np.float32)
    return q, k


@pytest.mark.parametrize("N,L,topk", [(1024, 2, 4), (4096, 3, 16)])
def test_select_equals_flat_exhaustive_topk_when_upper_levels_keep_all(N, L, topk):
    # Integer inputs make every pooled value a multiple of 16**-l and every
    # score exact in fp32 and fp64, so brute force in fp64 is the exact answer.
    # Ties are frequent, which also exercises the lower-index rule.
    q, k = _integer_inputs(11 + N, 1, 2, N, 16)
    pq, pk = oracle.pool(q, L), oracle.pool(k, L)
    idx = oracle.select_all(pq, pk, L, topk)
    for l in range(2, L + 1):  # every upper level keeps every candidate
        n = N // 16**l
        assert np.all((idx[l] >= 0).sum(-1) == min(topk, n))
    n1 = N // 16
    for h in range(2):
        for qq in range(0, n1, 7):
            want = _brute_topk(pq[1][0, h, qq].astype(np.float64),
                               pk[1][0, h].astype(np.float64), range(n1), topk)
            assert list(idx[1][0, h, qq]) == want


def test_select_hierarchical_descent_differs_from_flat_planted():
    # Level-2 block 8 is the best region on average; inside it level-1 block
    # 137 is best.  A decoy level-1 block 3 (in level-2 block 0) is the best
    # level-1 block overall, but its level-2 parent looks poor, so the
    # hierarchy never scores it.
    N, D = 4096, 4
    q = np.zeros((1, 1, N, D), dtype=np.float32)
    q[..., 0] = 1.0
    k = np.zeros((1, 1, N, D), dtype=np.float32)
    k[0, 0, 8 * 256:9 * 256, 0] = 1.0
    k[0, 0, 137 * 16:138 * 16, 0] = 2.0
    k[0, 0, 3 * 16:4 * 16, 0] = 3.0
    pq, pk = oracle.pool(q, 3), oracle.pool(k, 3)
    idx = oracle.select_all(pq, pk, 3, 1)
    assert np.all(idx[3] == 0)
    assert np.all(idx[2] == 8)
    assert np.all(idx[1] == 137)
    flat = oracle.select_level(pq[1], pk[1], None, 1)
    assert np.all(flat == 3)


def test_select_ties_go_to_lower_index():
    N, D = 4096, 8
    q = np.ones((1, 1, N, D), dtype=np.float32)
    k = np.ones((1, 1, N, D), dtype=np.float32)
    pq, pk = oracle.pool(q, 3), oracle.pool(k, 3)
    idx = oracle.select_all(pq, pk, 3, 4)
    assert np.all(idx[3][..., 0] == 0) and np.all(idx[3][..., 1:] == -1)  # one token, K_eff = 1
    assert np.all(idx[2] == np.arange(4))
    assert np.all(idx[1] == np.arange(4))  # children 0..15 of token 0, lowest four


def test_select_negative_zero_ties_with_positive_zero():
    # -0.0 == +0.0 under IEEE comparison, so the lower index wins.
    ql = np.array([[[[1.0, 0.0], [1.0, 0.0]]]], dtype=np.float32)  # [1,1,2,2]
    kl = np.array([[[[0.0, 5.0], [-0.0, 1.0]]]], dtype=np.float32)
    assert oracle.select_level(ql, kl, None, 1)[0, 0, 0, 0] == 0
    kl2 = np.array([[[[-0.0, 5.0], [0.0, 1.0]]]], dtype=np.float32)
    assert oracle.select_level(ql, kl2, None, 1)[0, 0, 0, 0] == 0


def test_select_page_descent_example_factor2():
    ex = json.load(open(GOLDEN))["descent_factor2_k1"]
    q = np.array(ex["q_fine"], dtype=np.float32).reshape(1, 1, -1, 1)
    k = np.array(ex["k_fine"], dtype=np.float32).reshape(1, 1, -1, 1)
    pq = oracle.pool(q, ex["L"], factor=ex["factor"])
    pk = oracle.pool(k, ex["L"], factor=ex["factor"])
    assert list(pk[1][0, 0, :, 0]) == ex["level1_means"]
    assert list(pk[2][0, 0, :, 0]) == ex["level2_means"]
    idx = oracle.select_all(pq, pk, ex["L"], ex["topk"], factor=ex["factor"])
    assert idx[2][0, 0].tolist() == ex["expected_I2"]
    assert idx[1][0, 0].tolist() == ex["expected_I1"]
    flat = oracle.select_level(pq[1], pk[1], None, 1, factor=ex["factor"])
    assert flat[0, 0, 0, 0] == ex["flat_best_level1_block"]


def test_select_parent_padding_limits_candidates():
    # A parent row with one kept key and one pad offers only 16 candidates;
    # with K = 20 the child rows hold those 16 and four pads.
    rng = np.random.default_rng(3)
    ql = rng.standard_normal((1, 1, 32, 4)).astype(np.float32)
    kl = rng.standard_normal((1, 1, 32, 4)).astype(np.float32)
    parent = np.array([[[[1, -1], [0, 1]]]], dtype=np.int32)  # [1,1,2,2]
    idx = oracle.select_level(ql, kl, parent, 20)
    assert np.all(idx[0, 0, :16, :16] == np.arange(16, 32))
    assert np.all(idx[0, 0, :16, 16:] == -1)
    assert np.all(idx[0, 0, 16:, :20] == np.sort(idx[0, 0, 16:, :20], axis=-1))
    assert np.all((idx[0, 0, 16:] >= 0).sum(-1) == 20)


def test_select_fp32_score_order_is_left_to_right():
    # Scores are summed d = 0..D-1 in fp32 with one rounding per operation.
    # With q = (1, 1, 1) the sum of k = (2^24, 1, 1) is 2^24 after rounding
    # (each +1 is lost), while (1, 1, 2^24) sums to 2^24 + 2 exactly, so the
    # second key ranks first although both have the same exact score.
    ql = np.ones((1, 1, 2, 3), dtype=np.float32)
    big = np.float32(2.0**24)
    kl = np.array([[[[big, 1, 1], [1, 1, big]]]], dtype=np.float32)
    idx = oracle.select_level(ql, kl, None, 1)
    assert idx[0, 0, 0, 0] == 1


def test_workload_keys_per_query_matches_page_example():
    ex = json.load(open(GOLDEN))["enriched_key_count"]
    w = workloads.WORKLOADS["img256_bf16"]
    assert w.topk == ex["topk"] and w.L - 1 == ex["coarse_levels"]
    assert w.keys_per_query() == ex["total_keys"]
    fine, coarse = oracle.key_sets(
        {l: np.zeros((1, 1, w.n_level(l), w.topk), dtype=np.int32) for l in range(1, w.L + 1)},
        w.L, w.n_level(1))
    assert fine.shape[-1] == ex["fine_keys"]
    assert all(c.shape[-1] == ex["coarse_keys_per_level"] for c in coarse.values())
