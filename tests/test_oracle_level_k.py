"""Pins of a Top-K per level (K_l kept keys at level l, the descent
unchanged): the level-to-K rule, flat exhaustive Top-K_1 when the upper
levels keep every candidate, a planted descent whose answer turns on K_2,
candidate padding, and attention/backward at mixed widths against dense
masked attention and finite differences."""

import numpy as np
import pytest

import oracle
from test_oracle_attn_bwd import _fp64_pyramid, _masked_dense
from test_oracle_pool_select import _brute_topk, _integer_inputs


def test_level_topk_rule():
    assert oracle.level_topk(8, 1) == 8 and oracle.level_topk(8, 3) == 8
    assert oracle.level_topk({1: 5, 2: 3}, 2) == 3
    assert oracle.level_topk([0, 4, 2, 1], 1) == 4


def test_widths_follow_the_levels():
    q, k = _integer_inputs(51, 1, 2, 4096, 8)
    pq, pk = oracle.pool(q, 3), oracle.pool(k, 3)
    idx = oracle.select_all(pq, pk, 3, {1: 6, 2: 3, 3: 1})
    assert idx[3].shape == (1, 2, 1, 1)
    assert idx[2].shape == (1, 2, 16, 3) and np.all((idx[2] >= 0).sum(-1) == 3)
    assert idx[1].shape == (1, 2, 256, 6) and np.all((idx[1] >= 0).sum(-1) == 6)
    # nesting: every kept level-1 block is a child of a key its parent kept
    for h in range(2):
        for b in range(256):
            parents = set(int(c) for c in idx[2][0, h, b // 16] if c >= 0)
            assert all(int(c) // 16 in parents for c in idx[1][0, h, b] if c >= 0)


@pytest.mark.parametrize("k1", [3, 11])
def test_flat_exhaustive_when_upper_levels_keep_all(k1):
    # 4096 tokens, L = 3: K_3 = 1 keeps the one top token, K_2 = 16 keeps all
    # of its children, so level 1 scores all 256 blocks: a flat Top-K_1.
    N = 4096
    q, k = _integer_inputs(52 + k1, 1, 2, N, 16)
    pq, pk = oracle.pool(q, 3), oracle.pool(k, 3)
    idx = oracle.select_all(pq, pk, 3, {1: k1, 2: 16, 3: 1})
    assert np.all(idx[2] == np.arange(16))
    for h in range(2):
        for qq in range(0, 256, 5):
            want = _brute_topk(pq[1][0, h, qq].astype(np.float64),
                               pk[1][0, h].astype(np.float64), range(256), k1)
            assert list(idx[1][0, h, qq]) == want


def _planted():
    # Level-2 region 8 is best on average and holds level-1 block 137 (2.0);
    # region 5 is second (average 5/16) and holds block 84 (5.0); region 0 is
    # third (3/16) and holds block 3 (3.0).  Every query is (1, 0, 0, 0).
    N, D = 4096, 4
    q = np.zeros((1, 1, N, D), dtype=np.float32)
    q[..., 0] = 1.0
    k = np.zeros((1, 1, N, D), dtype=np.float32)
    k[0, 0, 8 * 256:9 * 256, 0] = 1.0
    k[0, 0, 137 * 16:138 * 16, 0] = 2.0
    k[0, 0, 84 * 16:85 * 16, 0] = 5.0
    k[0, 0, 3 * 16:4 * 16, 0] = 3.0
    return oracle.pool(q, 3), oracle.pool(k, 3)


@pytest.mark.parametrize("k2,k1,want2,want1", [
    (1, 1, [8], [137]),
    (2, 1, [5, 8], [84]),
    (2, 2, [5, 8], [84, 137]),
    (3, 2, [0, 5, 8], [3, 84]),
    (3, 3, [0, 5, 8], [3, 84, 137]),
])
def test_planted_descent_turns_on_k2(k2, k1, want2, want1):
    pq, pk = _planted()
    idx = oracle.select_all(pq, pk, 3, {1: k1, 2: k2, 3: 1})
    assert np.all(idx[3] == 0)
    assert np.all(idx[2] == np.array(want2))
    assert np.all(idx[1] == np.array(want1))


def test_k1_above_candidates_pads():
    # K_2 = 1 leaves 16 candidates per query block; K_1 = 20 keeps them all
    # and pads four slots.
    rng = np.random.default_rng(53)
    q = rng.standard_normal((1, 1, 4096, 8)).astype(np.float32)
    k = rng.standard_normal((1, 1, 4096, 8)).astype(np.float32)
    pq, pk = oracle.pool(q, 3), oracle.pool(k, 3)
    idx = oracle.select_all(pq, pk, 3, {1: 20, 2: 1, 3: 1})
    for b in range(256):
        p = int(idx[2][0, 0, b // 16, 0])
        assert list(idx[1][0, 0, b, :16]) == list(range(16 * p, 16 * p + 16))
        assert np.all(idx[1][0, 0, b, 16:] == -1)


def _mixed_problem(seed, N, H, D):
    rng = np.random.default_rng(seed)
    Q, K, V = (rng.standard_normal((1, H, N, D)) for _ in range(3))
    pq, pk = oracle.pool(Q.astype(np.float32), 3), oracle.pool(K.astype(np.float32), 3)
    idx = oracle.select_all(pq, pk, 3, {1: 3, 2: 5, 3: 2})
    return Q, K, V, idx


def test_fwd_mixed_widths_equals_masked_dense():
    Q, K, V, idx = _mixed_problem(54, 8192, 2, 8)
    lw = [1, 1, 16.0, 256.0]
    pk, pv = _fp64_pyramid(K, 3), _fp64_pyramid(V, 3)
    O, LSE = oracle.attn_fwd(Q, K, V, pk, pv, idx, 3, 0.4, lw)
    Od, LSEd = _masked_dense(Q, K, V, pk, pv, idx, 3, 0.4, lw)
    assert np.allclose(O, Od, rtol=1e-10, atol=1e-12)
    assert np.allclose(LSE, LSEd, rtol=1e-10, atol=1e-12)


def test_bwd_mixed_widths_matches_finite_differences():
    Q, K, V, idx = _mixed_problem(55, 8192, 1, 4)
    scale = 0.5
    rng = np.random.default_rng(56)
    dO = rng.standard_normal(Q.shape)

    def loss(Q_, K_, V_):
        pk_, pv_ = _fp64_pyramid(K_, 3), _fp64_pyramid(V_, 3)
        O_, _ = oracle.attn_fwd(Q_, K_, V_, pk_, pv_, idx, 3, scale)
        return float((O_ * dO).sum())

    pk, pv = _fp64_pyramid(K, 3), _fp64_pyramid(V, 3)
    O, LSE = oracle.attn_fwd(Q, K, V, pk, pv, idx, 3, scale)
    grads = oracle.attn_bwd(Q, K, V, pk, pv, O, LSE, dO, idx, 3, scale)
    h = 1e-6
    for pos, G in enumerate(grads):
        for t in rng.integers(0, 8192, size=4):
            d = int(rng.integers(0, 4))
            args_p, args_m = [Q, K, V], [Q, K, V]
            Xp = args_p[pos].copy(); Xp[0, 0, t, d] += h
            Xm = args_m[pos].copy(); Xm[0, 0, t, d] -= h
            args_p[pos], args_m[pos] = Xp, Xm
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - G[0, 0, t, d]) <= 1e-6 * max(1.0, abs(fd))
