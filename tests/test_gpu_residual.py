"""GPU parity of the residual forward/backward (llsa_attn_fwd_res,
llsa_attn_bwd_res: Delta from dO . (O + O_res), one walk of each key list)
against the oracle, on the same cases and bar as the plain calls."""

import numpy as np
import pytest

import hierarchical_top_sparse_llsa_b200 as llsa
from hierarchical_top_sparse_llsa_b200 import workloads
from llsa_testlib import assert_close, run_gpu, run_oracle, settle_indices

pytestmark = pytest.mark.gpu


def _small(seed, B, H, N, D, dtype="bf16"):
    rng = np.random.default_rng(seed)
    x = {k: rng.standard_normal((B, H, N, D)).astype(np.float32) for k in ("q", "k", "v", "do")}
    return {k: workloads.round_to_bf16(v) for k, v in x.items()} if dtype == "bf16" else x


def _check(g, r, L, dtype, hs=slice(None), x=None, topk=8, **run_kw):
    sl = (slice(None), hs)  # heads are axis 1
    g, sl, _ = settle_indices(g, r, x, L, topk, dtype, sl, resid=True, **run_kw)
    assert_close(g["O"][sl], r["O"], dtype, "O")
    assert_close(g["LSE"][sl], r["LSE"], "f32" if dtype == "f32" else "bf16", "LSE")
    for name in ("dQ", "dK", "dV"):
        assert_close(g[name][sl], r[name], dtype, name)


@pytest.mark.parametrize("name,heads", [
    ("img64_bf16", None),
    ("img128_bf16", [0, 11]),
    ("img256_bf16", [0, 15]),
])
def test_workloads(name, heads):
    w = workloads.WORKLOADS[name]
    x = workloads.make_inputs(w)
    g = run_gpu(w.B, w.H, w.N, w.D, w.L, w.topk, w.dtype, x, resid=True)
    assert g["status"] == 0
    hs = slice(None) if heads is None else heads
    xs = x if heads is None else {k: np.ascontiguousarray(v[:, heads]) for k, v in x.items()}
    r = run_oracle(xs, w.L, w.topk)
    _check(g, r, w.L, w.dtype, hs, x=xs)


@pytest.mark.parametrize("B,H,N,D,L,kw", [
    (1, 3, 8192, 64, 3, {"level_w": [0, 0, 256.0, 4096.0]}),
    (2, 2, 4096, 128, 2, {}),
    (1, 3, 8192, 64, 3, {"topk_l": [0, 12, 4, 2], "level_w": [0, 0, 256.0, 4096.0]}),
    (1, 2, 8192, 64, 3, {"enrich": -1}),
    (1, 2, 8192, 64, 3, {"flags": llsa.FLAG_BWD_TCGEN05}),
    (1, 3, 2048, 64, 1, {}),
])
def test_variants(B, H, N, D, L, kw):
    x = _small(71 + N + D, B, H, N, D)
    g = run_gpu(B, H, N, D, L, 8, "bf16", x, resid=True, **kw)
    assert g["status"] == 0
    topk = 8 if "topk_l" not in kw else {l: kw["topk_l"][l] or 8 for l in range(1, L + 1)}
    r = run_oracle(x, L, topk, level_w=kw.get("level_w"), enrich=kw.get("enrich") or None)
    _check(g, r, L, "bf16", x=x, topk=topk, **kw)


def test_forward_outputs_and_residual_bound():
    # O and LSE are those of the plain forward; the residual is below half a
    # bf16 step of O (plus its own rounding) and brings O closer to the oracle
    B, H, N, D, L = 1, 2, 8192, 64, 3
    x = _small(81, B, H, N, D)
    g = run_gpu(B, H, N, D, L, 8, "bf16", x, resid=True, bwd=False)
    p = run_gpu(B, H, N, D, L, 8, "bf16", x, bwd=False)
    assert np.array_equal(g["O"], p["O"]) and np.array_equal(g["LSE"], p["LSE"])
    O, R = g["O"], g["O_res"]
    assert np.all(np.isfinite(R))
    half_ulp = np.ldexp(1.0, np.frexp(np.abs(O))[1] - 9)  # half a bf16 step at |O|
    assert np.all(np.abs(R) <= half_ulp * (1 + 2.0**-7) + 1e-30)
    r = run_oracle(x, L, 8, bwd=False, idx=g["idx"])  # attention on the GPU's own indices
    err_plain = np.sqrt(np.mean((O - r["O"]) ** 2))
    err_res = np.sqrt(np.mean((O + R - r["O"]) ** 2))
    assert err_res < err_plain


def test_fp32_residual_calls_equal_the_plain_ones():
    x = _small(82, 1, 2, 4096, 64, "f32")
    g = run_gpu(1, 2, 4096, 64, 3, 8, "f32", x, resid=True)
    p = run_gpu(1, 2, 4096, 64, 3, 8, "f32", x)
    for name in ("O", "LSE", "dQ", "dK", "dV"):
        assert np.array_equal(g[name], p[name]), name
