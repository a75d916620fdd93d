"""GPU parity of the whole LLSA path (through the C ABI) against the oracle.

Bar: pyramid, indices and key-major lists bit-exact; O, LSE, dQ, dK, dV within
max-abs 1e-4 (fp32 inputs) or 2e-2 * max(|ref|, rms(ref)) per element (bf16
inputs, against the fp64 oracle on the same bf16-rounded inputs).  Full-size
workloads run whole on the GPU and are checked on sampled heads, for which the
oracle runs on the head slice of the same draw (heads are independent).
"""

import numpy as np
import pytest

import hierarchical_top_sparse_llsa_b200 as llsa
from hierarchical_top_sparse_llsa_b200 import workloads
import oracle
from llsa_testlib import adjudicate_selection, assert_close, clean_indices, run_gpu, run_oracle, settle_indices

pytestmark = pytest.mark.gpu


def _compare(w, g, r, hs, bwd, x=None, topk=None, **run_kw):
    """Pyramid bit-exact; indices bit-exact or differing by near ties only
    (then O, LSE and the gradients are compared on a GPU run with the
    oracle's indices: pass the sliced inputs x); key-major lists bit-exact
    against the oracle's transpose of the same indices."""
    sl = (slice(None), hs)
    for l in range(1, w.L + 1):
        assert np.array_equal(g["pq"][l][sl], r["pq"][l]), f"Q pyramid level {l}"
        assert np.array_equal(g["pk"][l][sl], r["pk"][l]), f"K pyramid level {l}"
        if l >= 2:
            assert np.array_equal(g["pv"][l][sl], r["pv"][l]), f"V pyramid level {l}"
    gidx = {l: g["idx"][l][sl] for l in range(1, w.L + 1)}
    if not all(np.array_equal(gidx[l], r["idx"][l]) for l in gidx):
        near = adjudicate_selection(r["pq"], r["pk"], gidx, w.L, w.topk if topk is None else topk)
        print(f"{w.name}: {near} index rows differ by near ties only (adjudicated)")
        assert x is not None, "indices differ by near ties: the outputs need a run on the oracle's indices"
        # the same path on the oracle's indices, heads of the slice only
        B, H = x["q"].shape[:2]
        g = run_gpu(B, H, w.N, w.D, w.L, w.topk, w.dtype, x, ext_idx=r["idx"], bwd=bwd, **run_kw)
        sl = (slice(None), slice(None))
    for l in range(1, w.L + 1):
        if bwd:
            rp, col = oracle.index_transpose(g["idx"][l][sl], w.n_level(l))
            assert np.array_equal(g["row_ptr"][l][sl], rp), f"row_ptr level {l}"
            assert np.array_equal(g["col"][l][sl], col), f"col level {l}"
    assert_close(g["O"][sl], r["O"], w.dtype, "O")
    assert_close(g["LSE"][sl], r["LSE"], "f32" if w.dtype == "f32" else "bf16", "LSE")
    if bwd:
        for name in ("dQ", "dK", "dV"):
            assert_close(g[name][sl], r[name], w.dtype, name)


@pytest.mark.parametrize("name,heads", [
    ("tiny_32x32_f32", None),
    ("img64_bf16", None),
    ("img128_bf16", [0, 11]),
    ("img256_bf16", [0, 15]),
])
def test_workload_fwd_bwd(name, heads):
    w = workloads.WORKLOADS[name]
    x = workloads.make_inputs(w)
    g = run_gpu(w.B, w.H, w.N, w.D, w.L, w.topk, w.dtype, x)
    assert g["status"] == 0
    hs = slice(None) if heads is None else heads
    xs = x if heads is None else {k: np.ascontiguousarray(v[:, heads]) for k, v in x.items()}
    r = run_oracle(xs, w.L, w.topk)
    _compare(w, g, r, hs, True, x=xs)


@pytest.mark.parametrize("name", ["img512_k8_bf16", "img512_k32_bf16"])
def test_workload_fwd_only_scaling(name):
    w = workloads.WORKLOADS[name]
    x = workloads.make_inputs(w, with_dout=False)
    g = run_gpu(w.B, w.H, w.N, w.D, w.L, w.topk, w.dtype, x, bwd=False)
    assert g["status"] == 0
    heads = [5]
    xs = {k: np.ascontiguousarray(v[:, heads]) for k, v in x.items()}
    r = run_oracle(xs, w.L, w.topk, bwd=False)
    _compare(w, g, r, heads, False, x=xs)


def _small(seed, B, H, N, D, dtype="bf16"):
    rng = np.random.default_rng(seed)
    x = {k: rng.standard_normal((B, H, N, D)).astype(np.float32) for k in ("q", "k", "v", "do")}
    if dtype == "bf16":
        x = {k: workloads.round_to_bf16(v) for k, v in x.items()}
    return x


def test_paper_level_weights():
    w = workloads.WORKLOADS["img64_bf16"]
    x = workloads.make_inputs(w)
    lw = [0, 0] + [16.0**l for l in range(2, w.L + 1)]
    g = run_gpu(w.B, w.H, w.N, w.D, w.L, w.topk, w.dtype, x, level_w=lw)
    r = run_oracle(x, w.L, w.topk, level_w=lw)
    _compare(w, g, r, slice(None), True, x=x, level_w=lw)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_single_level_flat_topk(dtype):
    # L = 1: every query block scores every block (the single-level baseline)
    x = _small(21, 1, 3, 2048, 64, dtype)
    g = run_gpu(1, 3, 2048, 64, 1, 8, dtype, x)
    r = run_oracle(x, 1, 8)
    w = workloads.Workload("flat", 1, 3, 2048, 64, dtype, 1, 8, 0)
    _compare(w, g, r, slice(None), True, x=x)


def test_topk_above_candidates_pads():
    # K = 32 with one top-level token and 16 level-2 candidates: rows padded
    x = _small(22, 1, 2, 4096, 64)
    g = run_gpu(1, 2, 4096, 64, 3, 32, "bf16", x)
    r = run_oracle(x, 3, 32)
    w = workloads.Workload("k32", 1, 2, 4096, 64, "bf16", 3, 32, 0)
    _compare(w, g, r, slice(None), True, x=x)
    assert np.all(g["idx"][3][..., 1:] == -1) and np.all(g["idx"][2][..., 16:] == -1)


def test_head_dim_128_backward():
    x = _small(23, 2, 2, 4096, 128)
    g = run_gpu(2, 2, 4096, 128, 2, 8, "bf16", x)
    r = run_oracle(x, 2, 8)
    w = workloads.Workload("d128", 2, 2, 4096, 128, "bf16", 2, 8, 0)
    _compare(w, g, r, slice(None), True, x=x)


def test_external_indices_garbage_is_skipped_and_reported():
    B, H, N, D, L, K = 1, 2, 4096, 64, 3, 6
    x = _small(24, B, H, N, D)
    rng = np.random.default_rng(25)
    ext = {}
    for l in range(1, L + 1):
        n = N // 16**l
        I = rng.integers(-3, n + 3, size=(B, H, n, K)).astype(np.int32)
        I[..., 0, :] = -1  # an empty row
        ext[l] = I
    ext[1][0, 0, 7] = [5, 5, 9, 2, -1, 11]  # duplicate, unsorted, pad before valid
    clean = {}
    want_flags = 0
    for l in range(1, L + 1):
        clean[l], f = clean_indices(ext[l], N // 16**l)
        want_flags |= f
    g = run_gpu(B, H, N, D, L, K, "bf16", x, ext_idx=ext)
    r = run_oracle(x, L, K, idx=clean)
    assert g["status"] == want_flags and want_flags == (llsa.DEV_BAD_INDEX | llsa.DEV_NONCANONICAL)
    assert_close(g["O"], r["O"], "bf16", "O")
    assert_close(g["LSE"], r["LSE"], "bf16", "LSE")
    for l in range(1, L + 1):
        rp, col = r["csr"][l]
        assert np.array_equal(g["row_ptr"][l], rp) and np.array_equal(g["col"][l], col)
    for name in ("dQ", "dK", "dV"):
        assert_close(g[name], r[name], "bf16", name)


def test_empty_key_sets_give_zero_output():
    B, H, N, D, L, K = 1, 1, 1024, 64, 2, 4
    x = _small(26, B, H, N, D)
    ext = {1: np.full((B, H, 64, K), -1, np.int32), 2: np.full((B, H, 4, K), -1, np.int32)}
    ext[1][0, 0, 10:] = [0, 1, 2, 3]
    ext[2][0, 0, 1:] = [0, 1, 2, 3]
    g = run_gpu(B, H, N, D, L, K, "bf16", x, ext_idx=ext)
    r = run_oracle(x, L, K, idx=ext)
    assert g["status"] == 0
    assert np.all(g["O"][0, 0, :160] == 0) and np.all(np.isneginf(g["LSE"][0, 0, :160]))
    assert_close(g["O"], r["O"], "bf16", "O")
    for name in ("dQ", "dK", "dV"):
        assert_close(g[name], r[name], "bf16", name)


def test_runs_are_bitwise_deterministic():
    w = workloads.WORKLOADS["img64_bf16"]
    x = workloads.make_inputs(w)
    a = run_gpu(w.B, w.H, w.N, w.D, w.L, w.topk, w.dtype, x)
    b = run_gpu(w.B, w.H, w.N, w.D, w.L, w.topk, w.dtype, x)
    for key in ("O", "LSE", "dQ", "dK", "dV"):
        assert np.array_equal(a[key], b[key], equal_nan=True), key


@pytest.mark.parametrize("name,heads,flags", [
    ("img64_bf16", None, llsa.FLAG_FWD_TCGEN05),
    ("img128_bf16", [3], llsa.FLAG_FWD_TCGEN05),
    ("img256_bf16", [7], llsa.FLAG_FWD_TCGEN05),
    ("img512_k8_bf16", [2], llsa.FLAG_FWD_MMA_SYNC),
])
def test_forced_forward_kernel(name, heads, flags):
    # the default bf16 forward is tcgen05 at D = 128 and warp mma.sync at
    # D = 64 (every other test runs it); here the other kernel is forced
    w = workloads.WORKLOADS[name]
    x = workloads.make_inputs(w, with_dout=w.backward)
    g = run_gpu(w.B, w.H, w.N, w.D, w.L, w.topk, w.dtype, x, bwd=False, flags=flags)
    assert g["status"] == 0
    hs = slice(None) if heads is None else heads
    xs = x if heads is None else {k: np.ascontiguousarray(v[:, heads]) for k, v in x.items()}
    r = run_oracle(xs, w.L, w.topk, bwd=False)
    _compare(w, g, r, hs, False, x=xs, flags=flags)


@pytest.mark.parametrize("N,D", [(192, 64), (3 * 256 + 64, 128)])
def test_tcgen05_forward_partial_cta(N, D):
    # a CTA owns 8 query blocks; here the last one owns fewer (12 and 52
    # blocks), so its rows are stored by the threads rather than by TMA
    x = _small(41, 1, 2, N, D)
    g = run_gpu(1, 2, N, D, 1, 4, "bf16", x, bwd=False, resid=True, flags=llsa.FLAG_FWD_TCGEN05)
    r = run_oracle(x, 1, 4, bwd=False)
    assert g["status"] == 0
    assert_close(g["O"], r["O"], "bf16", "O")
    assert_close(g["LSE"], r["LSE"], "bf16", "LSE")
    # o + residual carries O to far below bf16 rounding
    err = np.abs(g["O"] + g["O_res"] - r["O"]).max()
    assert err < 2e-3 * np.abs(r["O"]).max(), err


@pytest.mark.parametrize("D", [64, 128])
def test_tcgen05_forward_rising_maximum(D):
    # keys whose magnitude grows with their block index, every block of the
    # single level kept (K = 32 of 32): each row's maximum rises chunk after
    # chunk by far more than the 2^8 the forward lets its reference lag, so
    # O and l are rescaled in tensor memory repeatedly
    B, H, N, L, K = 1, 2, 512, 1, 32
    x = _small(42, B, H, N, D)
    scale = np.repeat(np.linspace(0.2, 6.0, N // 16), 16).astype(np.float32)
    x["k"] = workloads.round_to_bf16(x["k"] * scale[None, None, :, None])
    g = run_gpu(B, H, N, D, L, K, "bf16", x, bwd=False, flags=llsa.FLAG_FWD_TCGEN05)
    r = run_oracle(x, L, K, bwd=False)
    assert g["status"] == 0
    assert np.all(g["idx"][1] >= 0)
    assert_close(g["O"], r["O"], "bf16", "O")
    assert_close(g["LSE"], r["LSE"], "bf16", "LSE")


@pytest.mark.parametrize("flags", [llsa.FLAG_FWD_TCGEN05, llsa.FLAG_FWD_MMA_SYNC])
def test_forward_external_indices_and_weights(flags):
    B, H, N, D, L, K = 1, 2, 4096, 64, 3, 6
    x = _small(27, B, H, N, D)
    rng = np.random.default_rng(28)
    ext = {}
    for l in range(1, L + 1):
        n = N // 16**l
        I = rng.integers(-3, n + 3, size=(B, H, n, K)).astype(np.int32)
        I[..., 0, :] = -1
        ext[l] = I
    clean = {}
    for l in range(1, L + 1):
        clean[l], _ = clean_indices(ext[l], N // 16**l)
    lw = [0, 0, 16.0**2, 16.0**3]
    g = run_gpu(B, H, N, D, L, K, "bf16", x, ext_idx=ext, bwd=False, level_w=lw, flags=flags)
    r = run_oracle(x, L, K, idx=clean, bwd=False, level_w=lw)
    assert_close(g["O"], r["O"], "bf16", "O")
    assert_close(g["LSE"], r["LSE"], "bf16", "LSE")


@pytest.mark.parametrize("name,heads", [
    ("img64_bf16", None),
    ("img128_bf16", [0, 11]),
    ("img256_bf16", [5]),
])
def test_tcgen05_backward(name, heads):
    # the tcgen05 key-major backward pass, selected by LLSA_FLAG_BWD_TCGEN05
    w = workloads.WORKLOADS[name]
    x = workloads.make_inputs(w)
    g = run_gpu(w.B, w.H, w.N, w.D, w.L, w.topk, w.dtype, x, flags=llsa.FLAG_BWD_TCGEN05)
    assert g["status"] == 0
    hs = slice(None) if heads is None else heads
    xs = x if heads is None else {k: np.ascontiguousarray(v[:, heads]) for k, v in x.items()}
    r = run_oracle(xs, w.L, w.topk)
    _compare(w, g, r, hs, True, x=xs, flags=llsa.FLAG_BWD_TCGEN05)


def test_tcgen05_backward_external_indices_and_long_rows():
    # caller indices with skipped entries, empty rows and one key block kept by
    # every query block (a key-major row of 256 query blocks: 32 groups)
    B, H, N, D, L, K = 1, 2, 4096, 64, 3, 6
    x = _small(29, B, H, N, D)
    rng = np.random.default_rng(30)
    ext = {}
    for l in range(1, L + 1):
        n = N // 16**l
        I = rng.integers(-3, n + 3, size=(B, H, n, K)).astype(np.int32)
        I[..., 0, :] = -1
        ext[l] = I
    ext[1][0, 1, :, 0] = 7
    ext[1][0, 1, :, 1:] = np.sort(rng.choice(np.arange(8, 256), size=(256, K - 1), replace=True), axis=1)
    clean = {}
    for l in range(1, L + 1):
        clean[l], _ = clean_indices(ext[l], N // 16**l)
    lw = [0, 0, 16.0**2, 16.0**3]
    g = run_gpu(B, H, N, D, L, K, "bf16", x, ext_idx=ext, level_w=lw, flags=llsa.FLAG_BWD_TCGEN05)
    r = run_oracle(x, L, K, idx=clean, level_w=lw)
    for name in ("dQ", "dK", "dV"):
        assert_close(g[name], r[name], "bf16", name)


@pytest.mark.parametrize("enrich,flags", [
    (-1, 0),
    (1, 0),
    (1, llsa.FLAG_FWD_TCGEN05 | llsa.FLAG_BWD_TCGEN05),
    (1, llsa.FLAG_FWD_MMA_SYNC),
    (2, llsa.FLAG_FWD_TCGEN05),
])
def test_enrichment_depth(enrich, flags):
    # L = 3 with the paper's level weights: depth 1 keeps the level-2 keys only,
    # -1 the fine keys only, 2 every level (the default).  Selection walks all
    # three levels either way; the key-major lists exist for levels 1..Lc.
    B, H, N, D, L, K = 1, 3, 8192, 64, 3, 8
    top = {-1: 1, 1: 2, 2: 3}[enrich]
    x = _small(31, B, H, N, D)
    lw = [0, 0] + [16.0**l for l in range(2, L + 1)]
    g = run_gpu(B, H, N, D, L, K, "bf16", x, level_w=lw, flags=flags, enrich=enrich)
    assert g["status"] == 0
    r = run_oracle(x, L, K, level_w=lw, enrich=enrich)
    g, _, _ = settle_indices(g, r, x, L, K, "bf16", level_w=lw, flags=flags, enrich=enrich)
    for l in range(1, top + 1):
        rp, col = r["csr"][l]
        assert np.array_equal(g["row_ptr"][l], rp), f"row_ptr level {l}"
        assert np.array_equal(g["col"][l], col), f"col level {l}"
    for name in ("O", "dQ", "dK", "dV"):
        assert_close(g[name], r[name], "bf16", name)
    assert_close(g["LSE"], r["LSE"], "bf16", "LSE")
    if enrich != 2:  # the depth changes the result
        full = run_oracle(x, L, K, level_w=lw, bwd=False)
        assert not np.allclose(full["O"], r["O"], rtol=1e-3, atol=1e-3)


@pytest.mark.parametrize("dtype,flags,kl", [
    ("bf16", 0, {1: 12, 2: 4, 3: 2}),
    ("bf16", 0, {1: 4, 2: 16, 3: 1}),
    ("bf16", 0, {1: 20, 2: 1, 3: 1}),   # 16 level-1 candidates: four pads per row
    ("bf16", llsa.FLAG_FWD_TCGEN05 | llsa.FLAG_BWD_TCGEN05, {1: 12, 2: 4, 3: 2}),
    ("bf16", llsa.FLAG_FWD_MMA_SYNC, {1: 12, 2: 4, 3: 2}),
    ("f32", 0, {1: 6, 2: 3, 3: 2}),
])
def test_topk_per_level(dtype, flags, kl):
    # K_l kept keys at level l: I(l) rows of width K_l, level l choosing among
    # the 16 * K_{l+1} children of its parent's keys; the paper weights make
    # the coarse keys count.
    B, H, N, D, L = 1, 3, 8192, 64, 3
    x = _small(32, B, H, N, D, dtype)
    lw = [0, 0] + [16.0**l for l in range(2, L + 1)]
    g = run_gpu(B, H, N, D, L, 8, dtype, x, level_w=lw, flags=flags, topk_l=[0] + [kl[l] for l in (1, 2, 3)])
    assert g["status"] == 0
    r = run_oracle(x, L, kl, level_w=lw)
    w = workloads.Workload("kl", B, H, N, D, dtype, L, 8, 0)
    for l in range(1, L + 1):
        assert g["idx"][l].shape[-1] == kl[l]
    _compare(w, g, r, slice(None), True, x=x, topk=kl, level_w=lw, flags=flags,
             topk_l=[0] + [kl[l] for l in (1, 2, 3)])
    if kl[1] > 16 * kl[2]:
        assert np.all((g["idx"][1] >= 0).sum(-1) == 16 * kl[2])
