"""llsa_attn_bwd_noalloc, the backward for callers that cannot allocate.

Callers such as a plugin host without an allocator, a runtime whose device
memory is fixed at start-up, or a latency-critical loop that must not call
cudaMalloc cannot hand the backward a scratch buffer; this entry point takes
its scratch from a fixed 16 MiB array inside the library instead.  The test
calls it through the C ABI twice in a row and checks each result against the
ordinary llsa_attn_bwd (caller-provided workspace) on the same inputs, with
the tolerance the parity tests use.  It lives in its own file, named to be
collected last, and passes alone in a fresh process as well as after the
other tests (its first call sets up the scratch address on the device).
"""

import numpy as np
import pytest

import hierarchical_top_sparse_llsa_b200 as llsa
from hierarchical_top_sparse_llsa_b200 import workloads
from llsa_testlib import assert_close

pytestmark = pytest.mark.gpu


def _problem(name):
    import torch

    w = workloads.WORKLOADS[name]
    x = workloads.make_inputs(w)
    t = {k: torch.from_numpy(v).to("cuda", dtype=torch.bfloat16) for k, v in x.items()}
    desc = llsa.make_desc(w.B, w.H, w.N, w.D, w.L, w.topk, llsa.BF16)
    bufs = llsa.LlsaBuffers(desc, "cuda")
    s = torch.cuda.current_stream().cuda_stream
    q, k, v = t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr()
    llsa.llsa_pool(desc, q, k, v, bufs.pyramid, s)
    llsa.llsa_select(desc, bufs.pyramid, bufs.indices, s)
    o = torch.empty_like(t["q"])
    lse = torch.empty(w.B, w.H, w.N, dtype=torch.float32, device="cuda")
    llsa.llsa_attn_fwd(desc, q, k, v, bufs.pyramid, bufs.indices, o.data_ptr(), lse.data_ptr(),
                       bufs.status.data_ptr(), s)
    llsa.llsa_index_transpose(desc, bufs.indices, bufs.csr, bufs.tr_ws.data_ptr(), bufs.tr_ws_bytes,
                              bufs.status.data_ptr(), s)
    return w, t, desc, bufs, o, lse, s


def test_noalloc_backward_matches_workspace_backward_twice():
    import torch

    w, t, desc, bufs, o, lse, s = _problem("img64_bf16")
    assert llsa.llsa_bwd_workspace_bytes(desc) <= llsa.NOALLOC_SCRATCH_BYTES
    args = (t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), bufs.pyramid, o.data_ptr(),
            lse.data_ptr(), t["do"].data_ptr(), bufs.indices, bufs.csr)
    ref = [torch.empty_like(o) for _ in range(3)]
    llsa.llsa_attn_bwd(desc, *args, *(g.data_ptr() for g in ref), bufs.ws.data_ptr(), bufs.ws_bytes,
                       bufs.status.data_ptr(), s)
    torch.cuda.synchronize()
    want = [g.float().cpu().numpy() for g in ref]
    for call in range(2):
        got = [torch.full_like(o, float("nan")) for _ in range(3)]
        llsa.llsa_attn_bwd_noalloc(desc, *args, *(g.data_ptr() for g in got),
                                   bufs.status.data_ptr(), s)
        torch.cuda.synchronize()
        for name, g, r in zip(("dQ", "dK", "dV"), got, want):
            assert_close(g.float().cpu().numpy(), r, "bf16", f"call {call}: {name}")
    assert int(bufs.status.item()) == 0


def test_noalloc_rejects_problems_above_its_scratch():
    w = workloads.WORKLOADS["img256_bf16"]
    desc = llsa.make_desc(w.B, w.H, w.N, w.D, w.L, w.topk, llsa.BF16)
    assert llsa.llsa_bwd_workspace_bytes(desc) > llsa.NOALLOC_SCRATCH_BYTES
    pyr, ind, csr = llsa.LlsaPyramid(), llsa.LlsaIndices(), llsa.LlsaCsr()
    fake = 256  # never dereferenced: the size check comes first
    st = llsa.llsa_attn_bwd_noalloc(desc, fake, fake, fake, pyr, fake, fake, fake, ind, csr,
                                    fake, fake, fake, check=False)
    assert st == llsa.ERR_WORKSPACE
