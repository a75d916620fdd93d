"""GPU raster <-> Z-order permutation against the oracle (a permutation:
compared bit for bit), both directions, both dtypes, both head dims."""

import numpy as np
import pytest

import oracle
import hierarchical_top_sparse_llsa_b200 as llsa

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("side,D,dtype", [(4, 64, "f32"), (32, 64, "bf16"), (64, 128, "bf16"), (256, 64, "bf16")])
@pytest.mark.parametrize("to_zorder", [True, False])
def test_reorder_matches_oracle(side, D, dtype, to_zorder):
    import torch

    B, H = 1, 3
    rng = np.random.default_rng(side + D)
    x = rng.standard_normal((B, H, side * side, D)).astype(np.float32)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    src = torch.from_numpy(x).to("cuda", dtype=tdt)
    dst = torch.full_like(src, float("nan"))
    llsa.llsa_reorder(B, H, side, side, D, llsa.BF16 if dtype == "bf16" else llsa.F32, src.data_ptr(),
                      dst.data_ptr(), to_zorder, torch.cuda.current_stream().cuda_stream)
    want = oracle.reorder(src.float().cpu().numpy(), side, side, to_zorder)
    assert np.array_equal(dst.float().cpu().numpy(), want)


def test_reorder_round_trip():
    import torch

    side, D = 128, 64
    x = torch.randn(2, 4, side * side, D, device="cuda", dtype=torch.bfloat16)
    z, back = torch.empty_like(x), torch.empty_like(x)
    s = torch.cuda.current_stream().cuda_stream
    llsa.llsa_reorder(2, 4, side, side, D, llsa.BF16, x.data_ptr(), z.data_ptr(), True, s)
    llsa.llsa_reorder(2, 4, side, side, D, llsa.BF16, z.data_ptr(), back.data_ptr(), False, s)
    assert torch.equal(back.view(torch.int16), x.view(torch.int16))
