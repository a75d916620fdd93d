"""Pins of the oracle's enriched sparse attention, index transpose and backward.

Independent routes: dense attention over an explicit N x (N + coarse) mask,
torch's fp64 scaled_dot_product_attention, scipy's softmax/logsumexp,
duplicated key rows, a dense block mask, and central finite differences.
"""

import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp, softmax

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_examples.json")


def _random_indices(rng, n_q, n_k, topk, pad_rows=0):
    """Random valid index lists: ascending, unique, -1 tail padding."""
    I = np.full((n_q, topk), -1, dtype=np.int32)
    for q in range(n_q):
        kk = topk if q >= pad_rows else rng.integers(0, topk)
        kk = min(kk, n_k)
        I[q, :kk] = np.sort(rng.choice(n_k, size=kk, replace=False))
    return I


def _random_problem(seed, B=1, H=2, N=1024, D=8, L=2, topk=3, pad_rows=0):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((B, H, N, D))
    K = rng.standard_normal((B, H, N, D))
    V = rng.standard_normal((B, H, N, D))
    idx = {}
    for l in range(1, L + 1):
        n = N // 16**l
        idx[l] = np.stack([np.stack([_random_indices(rng, n, n, topk, pad_rows)
                                     for _ in range(H)]) for _ in range(B)])
    return Q, K, V, idx


def _fp64_pyramid(X, L):
    B, H, N, D = X.shape
    return {l: X.reshape(B, H, N // 16**l, 16**l, D).mean(axis=3) for l in range(1, L + 1)}


def _dense_reference(Q, K, V, pk, pv, idx, L, scale, level_w, dup=False):
    """Dense attention of every query over all N fine keys plus every coarse
    token of every level, with an explicit mask built from the index lists.
    With dup=True a coarse key of weight w is instead appended w times."""
    B, H, N, D = Q.shape
    O = np.zeros((B, H, N, D))
    LSE = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            for i in range(N):
                blk = i // 16
                keys, vals, bias = [], [], []
                for c in idx[1][b, h, blk]:
                    if c >= 0:
                        for t in range(16 * c, 16 * c + 16):
                            keys.append(K[b, h, t]); vals.append(V[b, h, t]); bias.append(0.0)
                for l in range(2, L + 1):
                    w = 1.0 if level_w is None else level_w[l]
                    for c in idx[l][b, h, blk // 16 ** (l - 1)]:
                        if c >= 0:
                            reps = int(w) if dup else 1
                            for _ in range(reps):
                                keys.append(pk[l][b, h, c]); vals.append(pv[l][b, h, c])
                                bias.append(0.0 if dup else math.log(w))
                s = scale * np.array(keys) @ Q[b, h, i] + np.array(bias)
                O[b, h, i] = softmax(s) @ np.array(vals)
                LSE[b, h, i] = logsumexp(s)
    return O, LSE


def _masked_dense(Q, K, V, pk, pv, idx, L, scale, level_w):
    """One dense score matrix per head over [fine tokens | coarse tokens of
    levels 2..L]; unselected entries masked to -inf, coarse ones offset by ln w."""
    B, H, N, D = Q.shape
    O = np.zeros((B, H, N, D))
    LSE = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            keys = [K[b, h]] + [pk[l][b, h] for l in range(2, L + 1)]
            vals = [V[b, h]] + [pv[l][b, h] for l in range(2, L + 1)]
            Kall, Vall = np.concatenate(keys), np.concatenate(vals)
            mask = np.full((N, Kall.shape[0]), -np.inf)
            for i in range(N):
                for c in idx[1][b, h, i // 16]:
                    if c >= 0:
                        mask[i, 16 * c:16 * c + 16] = 0.0
                off = N
                for l in range(2, L + 1):
                    w = 1.0 if level_w is None else level_w[l]
                    for c in idx[l][b, h, (i // 16) // 16 ** (l - 1)]:
                        if c >= 0:
                            mask[i, off + c] = math.log(w)
                    off += N // 16**l
            S = scale * Q[b, h] @ Kall.T + mask
            empty = np.all(np.isneginf(S), axis=-1)  # no key at all: O = 0, LSE = -inf
            S[empty] = 0.0
            O[b, h] = np.where(empty[:, None], 0.0, softmax(S, axis=-1) @ Vall)
            LSE[b, h] = np.where(empty, -np.inf, logsumexp(S, axis=-1))
    return O, LSE


# ------------------------------------------------------------------ forward
def test_fwd_full_selection_no_coarse_equals_full_softmax_attention():
    rng = np.random.default_rng(5)
    N, D = 512, 16
    Q, K, V = (rng.standard_normal((1, 2, N, D)) for _ in range(3))
    idx = {1: np.broadcast_to(np.arange(N // 16, dtype=np.int32), (1, 2, N // 16, N // 16)).copy()}
    scale = oracle.default_scale(D)
    O, LSE = oracle.attn_fwd(Q, K, V, {}, {}, idx, 1, scale)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q), torch.from_numpy(K), torch.from_numpy(V), scale=scale).numpy()
    np.testing.assert_allclose(O, ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(LSE, logsumexp(scale * Q @ K.transpose(0, 1, 3, 2), axis=-1), rtol=1e-12)


@pytest.mark.parametrize("level_w", [None, [1, 1, 16.0**2, 16.0**3]])
def test_fwd_equals_masked_dense_attention(level_w):
    Q, K, V, idx = _random_problem(9, N=4096, L=3, topk=3, pad_rows=40)
    pk, pv = _fp64_pyramid(K, 3), _fp64_pyramid(V, 3)
    scale = 0.37
    O, LSE = oracle.attn_fwd(Q, K, V, pk, pv, idx, 3, scale, level_w)
    Od, LSEd = _masked_dense(Q, K, V, pk, pv, idx, 3, scale, level_w)
    np.testing.assert_allclose(O, Od, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(LSE, LSEd, rtol=1e-12, atol=1e-12)


def test_fwd_weight_equals_duplicated_coarse_rows():
    Q, K, V, idx = _random_problem(10, N=1024, H=1, L=2, topk=2)
    pk, pv = _fp64_pyramid(K, 2), _fp64_pyramid(V, 2)
    w = [1, 1, 3]
    O, LSE = oracle.attn_fwd(Q, K, V, pk, pv, idx, 2, 0.5, w)
    Od, LSEd = _dense_reference(Q, K, V, pk, pv, idx, 2, 0.5, w, dup=True)
    np.testing.assert_allclose(O, Od, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(LSE, LSEd, rtol=1e-12)


def test_fwd_reweighting_page_example_closed_form():
    # One fine key and one coarse key with equal scores; the coarse key weighs
    # 16, so it carries 16/17 of the attention.
    ex = json.load(open(GOLDEN))["reweighting"]
    w = ex["weight"]
    Q = np.zeros((1, 1, 256, 2)); K = np.zeros((1, 1, 256, 2)); V = np.zeros((1, 1, 256, 2))
    V[0, 0, :, 0] = 1.0  # fine tokens carry value (1, 0)
    pk = {2: np.zeros((1, 1, 1, 2))}
    pv = {2: np.array([[[[0.0, 1.0]]]])}  # the coarse token carries (0, 1)
    idx = {1: np.array([[[[0]]] * 16]).reshape(1, 1, 16, 1).astype(np.int32),
           2: np.zeros((1, 1, 1, 1), dtype=np.int32)}
    O, LSE = oracle.attn_fwd(Q, K, V, pk, pv, idx, 2, 1.0, [1, 1, w])
    # query 0 sees the 16 fine tokens of block 0 (value (1,0)) and the coarse token
    np.testing.assert_allclose(O[0, 0, 0], [16 / (16 + w), w / (16 + w)], rtol=1e-14)
    np.testing.assert_allclose(LSE[0, 0, 0], math.log(16 + w), rtol=1e-14)
    assert ex["weight"] == ex["factor"] ** ex["level"]


def test_fwd_empty_key_set_gives_zero_and_minus_inf():
    Q, K, V, idx = _random_problem(12, N=1024, H=1, L=2, topk=2)
    idx[1][0, 0, 5] = -1
    idx[2][0, 0, 0] = -1  # block 5 is under level-2 token 0
    pk, pv = _fp64_pyramid(K, 2), _fp64_pyramid(V, 2)
    O, LSE = oracle.attn_fwd(Q, K, V, pk, pv, idx, 2, 0.5)
    assert np.all(O[0, 0, 80:96] == 0) and np.all(np.isneginf(LSE[0, 0, 80:96]))
    assert np.all(np.isfinite(LSE[0, 0, :80]))


# ---------------------------------------------------------------- transpose
def test_transpose_matches_dense_block_mask():
    rng = np.random.default_rng(13)
    I = np.stack([_random_indices(rng, 64, 64, 5, pad_rows=10) for _ in range(3)])[None]
    row_ptr, col = oracle.index_transpose(I, 64)
    for h in range(3):
        M = np.zeros((64, 64), dtype=bool)  # M[q, c]
        for q in range(64):
            for c in I[0, h, q]:
                if c >= 0:
                    M[q, c] = True
        Mt = M.T
        for c in range(64):
            got = col[0, h, row_ptr[0, h, c]:row_ptr[0, h, c + 1]]
            assert got.tolist() == np.nonzero(Mt[c])[0].tolist()
        nvalid = int((I[0, h] >= 0).sum())
        assert row_ptr[0, h, -1] == nvalid
        assert np.all(col[0, h, nvalid:] == -1)


def test_transpose_page_example_pair_count():
    ex = json.load(open(GOLDEN))["transpose_pairs"]
    rng = np.random.default_rng(14)
    I = _random_indices(rng, ex["queries"], 128, ex["topk"])[None, None]
    row_ptr, col = oracle.index_transpose(I, 128)
    assert row_ptr[0, 0, -1] == ex["pairs"]
    pairs_in = sorted((int(c), q) for q in range(ex["queries"]) for c in I[0, 0, q])
    pairs_out = sorted((c, int(col[0, 0, p])) for c in range(128)
                       for p in range(row_ptr[0, 0, c], row_ptr[0, 0, c + 1]))
    assert pairs_in == pairs_out
    assert np.all(np.diff(row_ptr[0, 0]) >= 0)


# ----------------------------------------------------------------- backward
def _loss(Q, K, V, dO, idx, L, scale, level_w):
    pk, pv = _fp64_pyramid(K, L), _fp64_pyramid(V, L)
    O, _ = oracle.attn_fwd(Q, K, V, pk, pv, idx, L, scale, level_w)
    return float((O * dO).sum())


@pytest.mark.parametrize("level_w", [None, [1, 1, 256.0]])
def test_bwd_matches_central_finite_differences(level_w):
    L, scale = 2, 0.45
    Q, K, V, idx = _random_problem(15, N=1024, H=1, D=4, L=L, topk=2, pad_rows=6)
    rng = np.random.default_rng(16)
    dO = rng.standard_normal(Q.shape)
    pk, pv = _fp64_pyramid(K, L), _fp64_pyramid(V, L)
    O, LSE = oracle.attn_fwd(Q, K, V, pk, pv, idx, L, scale, level_w)
    dQ, dK, dV = oracle.attn_bwd(Q, K, V, pk, pv, O, LSE, dO, idx, L, scale, level_w)
    # fine tokens that no query block selects: their gradient comes only from
    # the coarse keys, so the spread-down term is exercised by these samples
    selected = np.zeros(64, dtype=bool)
    selected[idx[1][0, 0][idx[1][0, 0] >= 0]] = True
    unsel_tok = [t for t in range(1024) if not selected[t // 16]]
    assert unsel_tok
    samples = list(rng.integers(0, 1024, size=12)) + unsel_tok[:4]
    h = 1e-6
    for name, X, G in (("q", Q, dQ), ("k", K, dK), ("v", V, dV)):
        for t in samples:
            d = int(rng.integers(0, 4))
            Xp = X.copy(); Xp[0, 0, t, d] += h
            Xm = X.copy(); Xm[0, 0, t, d] -= h
            args = {"q": (Q, K, V), "k": (Q, K, V), "v": (Q, K, V)}[name]
            ap = list(args); am = list(args)
            pos = "qkv".index(name)
            ap[pos] = Xp; am[pos] = Xm
            fd = (_loss(*ap, dO, idx, L, scale, level_w) - _loss(*am, dO, idx, L, scale, level_w)) / (2 * h)
            assert abs(fd - G[0, 0, t, d]) <= 1e-6 * max(1.0, abs(fd)), (name, t, d, fd, G[0, 0, t, d])
    if name == "v":
        assert np.any(dV[0, 0, unsel_tok[0]] != 0)
