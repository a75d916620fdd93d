"""The near-tie adjudication that the GPU parity tests apply to selected
indices (spec: indices bit-exact, near-tie mismatches adjudicated).

A GPU selection may order two candidates whose fp32 scores differ by a
rounding error differently from the oracle's fixed left-to-right order; the
check accepts such a swap only within the recursive-summation bound
gamma_D * sum |q_d k_d| and rejects anything larger."""

import numpy as np
import pytest

import oracle
from llsa_testlib import adjudicate_selection


def _two_level(seed=7, D=64):
    rng = np.random.default_rng(seed)
    N = 16 * 16 * 4  # 4 level-2 tokens, 64 level-1 blocks
    Q1 = rng.standard_normal((1, 1, N // 16, D)).astype(np.float32)
    K1 = rng.standard_normal((1, 1, N // 16, D)).astype(np.float32)
    Q2 = Q1.reshape(1, 1, -1, 16, D).mean(3).astype(np.float32)
    K2 = K1.reshape(1, 1, -1, 16, D).mean(3).astype(np.float32)
    return {1: Q1, 2: Q2}, {1: K1, 2: K2}


def test_identical_indices_need_no_adjudication():
    pq, pk = _two_level()
    idx = oracle.select_all(pq, pk, 2, 4)
    assert adjudicate_selection(pq, pk, idx, 2, 4) == 0


def test_a_swapped_near_tie_is_accepted_and_counted():
    # one level (every query scores every block), query 0 = e_0, so its score
    # for key c is K[c, 0]: keys 0..3 clearly best, keys 4 and 5 one rounding
    # step apart for the fifth place
    D, n = 64, 16
    pq = {1: np.zeros((1, 1, n, D), np.float32)}
    pk = {1: np.zeros((1, 1, n, D), np.float32)}
    pq[1][0, 0, :, 0] = 1.0
    pk[1][0, 0, :, 0] = np.linspace(0.0, 1.0, n, dtype=np.float32)
    pk[1][0, 0, :4, 0] = [10.0, 9.0, 8.0, 7.0]
    pk[1][0, 0, 4, 0] = 5.0
    pk[1][0, 0, 5, 0] = np.nextafter(np.float32(5.0), np.float32(6.0))
    idx = oracle.select_all(pq, pk, 1, 5)
    assert list(idx[1][0, 0, 0]) == [0, 1, 2, 3, 5]
    gpu = {1: idx[1].copy()}
    gpu[1][0, 0, 0] = [0, 1, 2, 3, 4]
    assert adjudicate_selection(pq, pk, gpu, 1, 5) == 1
    # the same swap with a real gap is not a tie
    pk[1][0, 0, 5, 0] = 5.5
    with pytest.raises(AssertionError, match="beyond the rounding bound"):
        adjudicate_selection(pq, pk, gpu, 1, 5)


def test_a_wrong_key_is_rejected():
    pq, pk = _two_level()
    idx = oracle.select_all(pq, pk, 2, 4)
    gpu = {l: v.copy() for l, v in idx.items()}
    # replace the best key of row 3 by a candidate the oracle ranks last
    from oracle.llsa_oracle import _scores_fp32, candidates_for_level

    cand = candidates_for_level(idx[2], 16)[0, 0, 3 // 16]
    cand = cand[cand >= 0]
    s = _scores_fp32(pq[1][0, 0, 3:4], pk[1][0, 0][cand][None])[0]
    worst, best = int(cand[np.argmin(s)]), int(cand[np.argmax(s)])
    row = [c for c in gpu[1][0, 0, 3] if c >= 0 and c != best] + [worst]
    gpu[1][0, 0, 3, :len(row)] = sorted(row)
    with pytest.raises(AssertionError, match="beyond the rounding bound"):
        adjudicate_selection(pq, pk, gpu, 2, 4)
