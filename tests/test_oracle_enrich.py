"""Pins of the enrichment depth Le (the number of coarse levels whose pooled
tokens join the keys): the depth-to-level rule, dense masked attention with
only the enriched levels, agreement with padding the dropped levels' index
lists, and central finite differences of the backward."""

import numpy as np
import pytest

import oracle
from test_oracle_attn_bwd import _fp64_pyramid, _masked_dense, _random_problem


def test_depth_to_top_level():
    assert oracle.enriched_top(3, None) == 3
    assert oracle.enriched_top(3, 0) == 3
    assert oracle.enriched_top(3, 1) == 2
    assert oracle.enriched_top(3, 2) == 3
    assert oracle.enriched_top(3, 7) == 3
    assert oracle.enriched_top(3, -1) == 1
    assert oracle.enriched_top(1, None) == 1


@pytest.mark.parametrize("enrich,top", [(-1, 1), (1, 2), (2, 3)])
def test_fwd_equals_masked_dense_over_the_enriched_levels(enrich, top):
    # _masked_dense builds its score matrix over levels 2..L' for the L' it is
    # given: with L' = the top enriched level it is the reference for depth Le
    L, scale, lw = 3, 0.4, [1, 1, 16.0, 256.0]
    Q, K, V, idx = _random_problem(41, N=4096, H=1, D=8, L=L, topk=3, pad_rows=5)
    pk, pv = _fp64_pyramid(K, L), _fp64_pyramid(V, L)
    O, LSE = oracle.attn_fwd(Q, K, V, pk, pv, idx, L, scale, lw, enrich=enrich)
    Od, LSEd = _masked_dense(Q, K, V, pk, pv, idx, top, scale, lw)
    assert np.allclose(O, Od, rtol=1e-10, atol=1e-12)
    assert np.allclose(LSE, LSEd, rtol=1e-10, atol=1e-12, equal_nan=False)


def test_depth_equals_padding_the_dropped_levels():
    L, scale = 3, 0.3
    Q, K, V, idx = _random_problem(42, N=4096, H=2, D=8, L=L, topk=4)
    pk, pv = _fp64_pyramid(K, L), _fp64_pyramid(V, L)
    O1, L1 = oracle.attn_fwd(Q, K, V, pk, pv, idx, L, scale, enrich=1)
    padded = dict(idx)
    padded[3] = np.full_like(idx[3], -1)
    O2, L2 = oracle.attn_fwd(Q, K, V, pk, pv, padded, L, scale)
    # the padded run reduces over K more (masked, zero) terms, so the fp64
    # sums may differ in rounding order only
    assert np.allclose(O1, O2, rtol=1e-12, atol=1e-14)
    assert np.allclose(L1, L2, rtol=1e-12, atol=1e-14)
    rng = np.random.default_rng(43)
    dO = rng.standard_normal(Q.shape)
    g1 = oracle.attn_bwd(Q, K, V, pk, pv, O1, L1, dO, idx, L, scale, enrich=1)
    g2 = oracle.attn_bwd(Q, K, V, pk, pv, O2, L2, dO, padded, L, scale)
    for a, b in zip(g1, g2):
        assert np.allclose(a, b, rtol=1e-11, atol=1e-13)


def test_bwd_with_depth_one_matches_finite_differences():
    L, scale, enrich = 3, 0.5, 1
    Q, K, V, idx = _random_problem(44, N=4096, H=1, D=4, L=L, topk=2)
    rng = np.random.default_rng(45)
    dO = rng.standard_normal(Q.shape)

    def loss(Q_, K_, V_):
        pk_, pv_ = _fp64_pyramid(K_, L), _fp64_pyramid(V_, L)
        O_, _ = oracle.attn_fwd(Q_, K_, V_, pk_, pv_, idx, L, scale, enrich=enrich)
        return float((O_ * dO).sum())

    pk, pv = _fp64_pyramid(K, L), _fp64_pyramid(V, L)
    O, LSE = oracle.attn_fwd(Q, K, V, pk, pv, idx, L, scale, enrich=enrich)
    grads = oracle.attn_bwd(Q, K, V, pk, pv, O, LSE, dO, idx, L, scale, enrich=enrich)
    h = 1e-6
    for pos, G in enumerate(grads):
        for t in rng.integers(0, 4096, size=5):
            d = int(rng.integers(0, 4))
            args_p = [Q, K, V]
            args_m = [Q, K, V]
            Xp = args_p[pos].copy(); Xp[0, 0, t, d] += h
            Xm = args_m[pos].copy(); Xm[0, 0, t, d] -= h
            args_p[pos], args_m[pos] = Xp, Xm
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - G[0, 0, t, d]) <= 1e-6 * max(1.0, abs(fd))
