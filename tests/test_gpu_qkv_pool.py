"""GPU parity of the QKV projection with the pooling epilogue (llsa_qkv_pool):
Q, K, V against the product X W^T of the same bf16 values in fp64 (within one
bf16 rounding plus fp32 accumulation error), and the pyramid bit for bit
against llsa_pool run on the call's own Q, K, V, and against the oracle's
pool of them."""

import numpy as np
import pytest
import torch

import hierarchical_top_sparse_llsa_b200 as llsa
from hierarchical_top_sparse_llsa_b200 import workloads
from oracle import llsa_oracle as oracle

pytestmark = pytest.mark.gpu


def _run(B, H, N, D, L, C, seed):
    rng = np.random.default_rng(seed)
    x = workloads.round_to_bf16(rng.standard_normal((B, N, C)).astype(np.float32))
    w = workloads.round_to_bf16((rng.standard_normal((3 * H * D, C)) / np.sqrt(C)).astype(np.float32))
    dev = "cuda"
    xt = torch.from_numpy(x).to(dev, torch.bfloat16)
    wt = torch.from_numpy(w).to(dev, torch.bfloat16)
    desc = llsa.make_desc(B, H, N, D, L, 8, llsa.BF16)
    fused = llsa.LlsaBuffers(desc, dev, with_bwd=False)
    plain = llsa.LlsaBuffers(desc, dev, with_bwd=False)
    qkv = [torch.full((B, H, N, D), float("nan"), dtype=torch.bfloat16, device=dev) for _ in range(3)]
    for t in (fused.pq, fused.pk, fused.pv):
        for a in t.values():
            a.fill_(float("nan"))  # every element must be written
    stream = torch.cuda.current_stream().cuda_stream
    llsa.llsa_qkv_pool(desc, xt.data_ptr(), wt.data_ptr(), C, qkv[0].data_ptr(), qkv[1].data_ptr(),
                       qkv[2].data_ptr(), fused.pyramid, fused.status.data_ptr(), stream)
    llsa.llsa_pool(desc, qkv[0].data_ptr(), qkv[1].data_ptr(), qkv[2].data_ptr(), plain.pyramid, stream)
    torch.cuda.synchronize()
    assert int(fused.status.item()) == 0
    return x, w, [a.float().cpu().numpy() for a in qkv], fused, plain


def _check_projection(x, w, qkv, B, H, N, D):
    ref = np.einsum("bnc,fc->bnf", x.astype(np.float64), w.astype(np.float64))
    mag = np.einsum("bnc,fc->bnf", np.abs(x).astype(np.float64), np.abs(w).astype(np.float64))
    got = np.concatenate([a.transpose(0, 2, 1, 3).reshape(B, N, H * D) for a in qkv], axis=-1)
    # one bf16 rounding (half a unit: 2^-9 relative) of an fp32 sum whose own
    # error is within C * 2^-24 of the sum of |x w|
    C = x.shape[-1]
    bound = 2.0**-8 * np.abs(ref) + C * 2.0**-23 * mag + 1e-30
    err = np.abs(got - ref)
    assert np.all(err <= bound), f"max excess {np.max(err / bound):.3g}"


@pytest.mark.parametrize("B,H,N,D,L,C", [
    (1, 4, 4096, 64, 3, 256),
    (2, 2, 1024, 128, 2, 128),
    (1, 2, 65536, 64, 4, 64),
    (2, 4, 256, 64, 1, 192),
])
def test_projection_and_pyramid(B, H, N, D, L, C):
    x, w, qkv, fused, plain = _run(B, H, N, D, L, C, seed=300 + N + C)
    _check_projection(x, w, qkv, B, H, N, D)
    for name, tf, tp in (("Q", fused.pq, plain.pq), ("K", fused.pk, plain.pk), ("V", fused.pv, plain.pv)):
        for l in tf:
            a, b = tf[l].cpu().numpy(), tp[l].cpu().numpy()
            assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), f"{name} level {l}"
    # and the oracle's pool of the same Q, K, V
    for name, t, X in (("Q", fused.pq, qkv[0]), ("K", fused.pk, qkv[1]), ("V", fused.pv, qkv[2])):
        ref = oracle.pool(X, L)
        for l in t:
            assert np.array_equal(t[l].cpu().numpy(), ref[l]), f"{name} level {l} vs oracle"


def test_headline_width_sampled():
    # 256x256 pixels, 16 heads of 64, model width 1024: the projection on
    # sampled tokens, the whole pyramid bit for bit against llsa_pool
    B, H, N, D, L, C = 1, 16, 65536, 64, 3, 1024
    x, w, qkv, fused, plain = _run(B, H, N, D, L, C, seed=9)
    rows = np.random.default_rng(5).choice(N, 512, replace=False)
    _check_projection(x[:, rows], w, [a[:, :, rows] for a in qkv], B, H, len(rows), D)
    for tf, tp in ((fused.pq, plain.pq), (fused.pk, plain.pk), (fused.pv, plain.pv)):
        for l in tf:
            assert torch.equal(tf[l].view(torch.int32), tp[l].view(torch.int32)), f"level {l}"
