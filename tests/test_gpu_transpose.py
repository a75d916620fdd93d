"""GPU parity of the sparse index transpose (llsa_index_transpose) against the
oracle's stable counting sort, bit for bit, on index rows built directly:
every row width from 1 to 32, ragged row counts, skewed key popularity,
garbage entries, levels of up to 32768 keys."""

import numpy as np
import pytest
import torch

import hierarchical_top_sparse_llsa_b200 as llsa
from llsa_testlib import clean_indices
from oracle import llsa_oracle as oracle

pytestmark = pytest.mark.gpu


def _rows(rng, B, H, n, K, hot=0.5):
    """Canonical rows (ascending, -1 tail) of random length 0..K; a share
    `hot` of the draws comes from 64 popular keys, so some keys collect long
    lists."""
    shape = (B, H, n, K)
    keys = rng.integers(0, n, size=shape)
    hot_keys = rng.integers(0, n, size=64)
    pick = rng.random(shape) < hot
    keys[pick] = hot_keys[rng.integers(0, 64, size=int(pick.sum()))]
    big = np.iinfo(np.int64).max
    s = np.sort(keys, axis=-1)
    dup = np.zeros(shape, bool)
    dup[..., 1:] = s[..., 1:] == s[..., :-1]
    s[dup] = big
    lens = rng.integers(0, K + 1, size=shape[:-1])
    s[np.arange(K) >= lens[..., None]] = big
    s = np.sort(s, axis=-1)
    s[s == big] = -1
    return s.astype(np.int32)


def _gpu_transpose(B, H, N, L, K, idx, topk_l=None):
    desc = llsa.make_desc(B, H, N, 64, L, K, llsa.BF16, topk_l=topk_l)
    buf = llsa.LlsaBuffers(desc, "cuda")
    for l in range(1, L + 1):
        buf.idx[l].copy_(torch.from_numpy(idx[l]))
        buf.col[l].fill_(-7)  # every slot must be written
        buf.row_ptr[l].fill_(-7)
    llsa.llsa_index_transpose(desc, buf.indices, buf.csr, buf.tr_ws.data_ptr(), buf.tr_ws_bytes,
                              buf.status.data_ptr(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    out = {l: (buf.row_ptr[l].cpu().numpy(), buf.col[l].cpu().numpy()) for l in range(1, L + 1)}
    return out, int(buf.status.item())


def _check(out, idx, N, L, want_flags=0, status=0):
    assert status == want_flags
    for l in range(1, L + 1):
        n = N // 16**l
        clean, _ = clean_indices(idx[l], n) if want_flags else (idx[l], 0)
        rp, col = oracle.index_transpose(clean, n)
        assert np.array_equal(out[l][0], rp), f"row_ptr level {l}"
        assert np.array_equal(out[l][1], col), f"col level {l}"


@pytest.mark.parametrize("K", [1, 3, 5, 8, 12, 16, 31, 32])
def test_row_widths(K):
    # n = 1000 level-1 keys: rows split unevenly over the CTAs of a cluster
    B, H, N = 2, 3, 16000
    rng = np.random.default_rng(100 + K)
    idx = {1: _rows(rng, B, H, N // 16, K)}
    out, st = _gpu_transpose(B, H, N, 1, K, idx)
    _check(out, idx, N, 1, status=st)


@pytest.mark.parametrize("B,H,N,L,K", [
    (1, 16, 65536, 3, 8),      # 256x256 pixels, three levels
    (1, 2, 262144, 4, 32),     # 512x512 pixels, K = 32: 16384 level-1 keys of 32 entries
    (1, 1, 16, 1, 4),          # a single key
    (3, 1, 4096 * 16, 2, 2),   # more (b, h) than one key's list is long
])
def test_levels(B, H, N, L, K):
    rng = np.random.default_rng(7 + N + K)
    idx = {l: _rows(rng, B, H, N // 16**l, K, hot=0.3) for l in range(1, L + 1)}
    out, st = _gpu_transpose(B, H, N, L, K, idx)
    _check(out, idx, N, L, status=st)


@pytest.mark.parametrize("n", [20480, 32768])
def test_large_levels(n):
    # more keys than one 8192-key shared-memory range of the count and fill
    B, H, N, K = 1, 2, n * 16, 8
    rng = np.random.default_rng(31 + n)
    idx = {1: _rows(rng, B, H, N // 16, K)}
    out, st = _gpu_transpose(B, H, N, 1, K, idx)
    _check(out, idx, N, 1, status=st)


def test_per_level_width_and_garbage():
    B, H, N, L = 1, 2, 65536, 3
    topk_l = [0, 12, 5, 3]
    rng = np.random.default_rng(41)
    idx = {}
    for l in range(1, L + 1):
        n, K = N // 16**l, topk_l[l]
        I = _rows(rng, B, H, n, K)
        bad = rng.random(I.shape) < 0.02
        I[bad] = rng.integers(-3, n + 3, size=int(bad.sum()))
        idx[l] = I
    idx[1][0, 1, 5] = [7, 7, 3, -1, 9, 2, 1, 0, -2, 4100, 11, 12]  # duplicate, unsorted, pad before valid
    want = 0
    for l in range(1, L + 1):
        want |= clean_indices(idx[l], N // 16**l)[1]
    assert want == llsa.DEV_BAD_INDEX | llsa.DEV_NONCANONICAL
    out, st = _gpu_transpose(B, H, N, L, 12, idx, topk_l=topk_l)
    _check(out, idx, N, L, want_flags=want, status=st)
