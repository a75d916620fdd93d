"""The kernels' bounded waits end with a status, not a hung GPU.

Every mbarrier wait in the attention kernels gives up after a time limit and
reports LLSA_DEV_TIMEOUT through the caller's status word.  A correct launch
never reaches the limit, so llsa_selftest_wait_timeout runs the same wait
helper on a barrier nothing arrives on (no copy in flight, no fault).  The
test checks that the status arrives, that the wait took about its limit, and
that the same stream then runs the path's ordinary calls correctly."""

import time

import numpy as np
import pytest

import hierarchical_top_sparse_llsa_b200 as llsa
from hierarchical_top_sparse_llsa_b200 import workloads

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_stream_stays_usable():
    import torch

    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    llsa.llsa_selftest_wait_timeout(status.data_ptr(), 20000, s)  # 20 ms limit
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert int(status.item()) == llsa.DEV_TIMEOUT
    assert 0.015 <= waited < 2.0, waited

    # the context and the stream still work: the pool runs and is exact
    w = workloads.WORKLOADS["img64_bf16"]
    x = workloads.make_inputs(w, with_dout=False)
    t = {k: torch.from_numpy(v).to("cuda", dtype=torch.bfloat16) for k, v in x.items()}
    desc = llsa.make_desc(w.B, w.H, w.N, w.D, w.L, w.topk, llsa.BF16)
    bufs = llsa.LlsaBuffers(desc, "cuda", with_bwd=False)
    llsa.llsa_pool(desc, t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), bufs.pyramid, s)
    torch.cuda.synchronize()
    q1 = t["q"].float().reshape(w.B, w.H, w.N // 16, 16, w.D)
    # level 1 is the left-to-right fp32 sum of 16 rows times 1/16
    acc = q1[:, :, :, 0]
    for j in range(1, 16):
        acc = acc + q1[:, :, :, j]
    assert torch.equal(bufs.pq[1], acc * (1.0 / 16))
