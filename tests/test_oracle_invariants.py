"""Property pins of the oracle on random small inputs (hypothesis): what the
Top-K selection and the index transpose must satisfy whatever the values,
checked by brute force rather than by restating the oracle's steps.

- select_level: each row holds min(K, #candidates) distinct candidates in
  ascending order, padded with -1; every kept candidate scores at least as
  high as every candidate left out (ties: the kept one has the lower index),
  scores taken in fp32 in the order the selection fixes (d = 0..D-1, one
  rounding per multiply and per add).
- index_transpose: row_ptr is the running count of every key's occurrences,
  each key's list is ascending, and the (query, key) pairs are exactly those
  of the index lists.
"""

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle


def _fp32_score(q, k):
    s = np.float32(0.0)
    for d in range(q.shape[0]):
        s = np.float32(s + np.float32(q[d] * k[d]))
    return s


@settings(max_examples=40, deadline=None)
@given(seed=st.integers(0, 2**31 - 1), n=st.sampled_from([16, 32, 48]), D=st.integers(1, 6),
       K=st.integers(1, 20), n_par=st.integers(0, 3))
def test_select_level_is_a_top_k(seed, n, D, K, n_par):
    rng = np.random.default_rng(seed)
    # small integers make ties frequent, which exercises the index rule
    ql = rng.integers(-2, 3, size=(1, 1, n, D)).astype(np.float32)
    kl = rng.integers(-2, 3, size=(1, 1, n, D)).astype(np.float32)
    n_parent_rows = n // 16
    kp = max(1, n_par)
    parent = np.full((1, 1, n_parent_rows, kp), -1, dtype=np.int32)
    for r in range(n_parent_rows):
        chosen = np.sort(rng.choice(n_parent_rows, size=min(n_par, n_parent_rows), replace=False))
        parent[0, 0, r, :chosen.size] = chosen
    idx = oracle.select_level(ql, kl, parent, K)
    for q in range(n):
        par = [int(p) for p in parent[0, 0, q // 16] if p >= 0]
        cand = [16 * p + j for p in par for j in range(16)]
        row = idx[0, 0, q]
        kept = [int(c) for c in row if c >= 0]
        assert len(kept) == min(K, len(cand))
        assert all(c == -1 for c in row[len(kept):])
        assert kept == sorted(set(kept)) and set(kept) <= set(cand)
        sc = {c: _fp32_score(ql[0, 0, q], kl[0, 0, c]) for c in cand}
        for a in kept:
            for b in set(cand) - set(kept):
                assert sc[a] > sc[b] or (sc[a] == sc[b] and a < b)


@settings(max_examples=60, deadline=None)
@given(seed=st.integers(0, 2**31 - 1), nq=st.integers(1, 40), n_keys=st.integers(1, 40),
       K=st.integers(1, 8), pad=st.floats(0.0, 0.8))
def test_index_transpose_lists_every_pair_once_in_order(seed, nq, n_keys, K, pad):
    rng = np.random.default_rng(seed)
    I = np.full((1, 2, nq, K), -1, dtype=np.int32)
    for h in range(2):
        for q in range(nq):
            m = min(K, n_keys, int(round(K * (1 - pad))))
            I[0, h, q, :m] = np.sort(rng.choice(n_keys, size=m, replace=False))
    row_ptr, col = oracle.index_transpose(I, n_keys)
    for h in range(2):
        pairs = {(q, int(c)) for q in range(nq) for c in I[0, h, q] if c >= 0}
        assert row_ptr[0, h, 0] == 0 and row_ptr[0, h, -1] == len(pairs)
        listed = set()
        for c in range(n_keys):
            qs = [int(x) for x in col[0, h, row_ptr[0, h, c]:row_ptr[0, h, c + 1]]]
            assert qs == sorted(qs)
            assert len(qs) == sum(1 for q in range(nq) if c in I[0, h, q])
            listed |= {(q, c) for q in qs}
        assert listed == pairs
        assert np.all(col[0, h, row_ptr[0, h, -1]:] == -1)
