"""GPU parity of llsa_select_attn_fwd (the forward with the level-1 selection
in its prologue): identical, bit for bit, to llsa_select followed by
llsa_attn_fwd, and within the bar of the oracle."""

import numpy as np
import pytest

import hierarchical_top_sparse_llsa_b200 as llsa
from hierarchical_top_sparse_llsa_b200 import workloads
from llsa_testlib import assert_close, run_oracle

pytestmark = pytest.mark.gpu


def _both(B, H, N, D, L, K, dtype, x, **kw):
    import torch

    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    t = {k: torch.from_numpy(np.ascontiguousarray(v)).to(device="cuda", dtype=tdt) for k, v in x.items()}
    desc = llsa.make_desc(B, H, N, D, L, K, llsa.BF16 if dtype == "bf16" else llsa.F32, **kw)
    res = []
    for fused in (False, True):
        bufs = llsa.LlsaBuffers(desc, "cuda", with_bwd=False)
        for l in bufs.idx:
            bufs.idx[l].fill_(12345)  # every entry must be written
        st = bufs.status.data_ptr()
        llsa.llsa_pool(desc, t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), bufs.pyramid)
        o = torch.empty_like(t["q"])
        lse = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
        args = (desc, t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), bufs.pyramid, bufs.indices,
                o.data_ptr(), lse.data_ptr(), st)
        if fused:
            llsa.llsa_select_attn_fwd(*args)
        else:
            llsa.llsa_select(desc, bufs.pyramid, bufs.indices)
            llsa.llsa_attn_fwd(*args)
        torch.cuda.synchronize()
        res.append({"idx": {l: bufs.idx[l].cpu().numpy() for l in bufs.idx},
                    "O": o.float().cpu().numpy(), "LSE": lse.cpu().numpy(),
                    "status": int(bufs.status.item())})
    return res


def _small(seed, B, H, N, D, dtype):
    rng = np.random.default_rng(seed)
    x = {k: rng.standard_normal((B, H, N, D)).astype(np.float32) for k in ("q", "k", "v")}
    return {k: workloads.round_to_bf16(v) for k, v in x.items()} if dtype == "bf16" else x


@pytest.mark.parametrize("B,H,N,D,L,K,dtype,kw", [
    (2, 3, 16384, 64, 3, 8, "bf16", {}),
    (1, 2, 8192, 128, 2, 8, "bf16", {}),
    (1, 3, 8192, 64, 3, 8, "bf16", {"topk_l": [0, 12, 4, 2], "level_w": [0, 0, 256.0, 4096.0]}),
    (1, 3, 8192, 64, 3, 8, "bf16", {"topk_l": [0, 20, 1, 1]}),
    (1, 2, 8192, 64, 3, 8, "bf16", {"enrich_levels": 1}),
    (1, 2, 2048, 64, 1, 8, "bf16", {}),          # L = 1: the fused prologue scores every block
    (1, 2, 8192, 64, 3, 8, "bf16", {"flags": 1}),  # tcgen05 forward: selection unfused
    (1, 2, 4096, 64, 3, 8, "f32", {}),             # fp32 forward: selection unfused
])
def test_fused_equals_separate_calls_and_oracle(B, H, N, D, L, K, dtype, kw):
    x = _small(61 + N + D + L, B, H, N, D, dtype)
    sep, fus = _both(B, H, N, D, L, K, dtype, x, **kw)
    assert sep["status"] == 0 and fus["status"] == 0
    for l in sep["idx"]:
        assert np.array_equal(sep["idx"][l], fus["idx"][l]), f"indices level {l}"
    assert np.array_equal(sep["O"], fus["O"])
    assert np.array_equal(sep["LSE"], fus["LSE"])
    topk = K if "topk_l" not in kw else {l: (kw["topk_l"][l] or K) for l in range(1, L + 1)}
    enrich = kw.get("enrich_levels") or None
    lw = kw.get("level_w")
    r = run_oracle(x, L, topk, level_w=lw, bwd=False, enrich=enrich)
    for l in range(1, L + 1):
        assert np.array_equal(fus["idx"][l], r["idx"][l]), f"oracle indices level {l}"
    assert_close(fus["O"], r["O"], dtype, "O")
    assert_close(fus["LSE"], r["LSE"], "f32" if dtype == "f32" else "bf16", "LSE")
