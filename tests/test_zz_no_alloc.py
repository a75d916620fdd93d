"""llsa_attn_bwd_noalloc, the backward for callers that cannot allocate.

Callers such as a plugin host without an allocator, a runtime whose device
memory is fixed at start-up, or a latency-critical loop that must not call
cudaMalloc cannot hand the backward a scratch buffer; this entry point takes
its scratch from a fixed 16 MiB array inside the library instead.  The test
first runs it on an unrelated problem, so the array holds other data, then
calls it through the C ABI twice in a row on the checked problem: both
results must equal the ordinary llsa_attn_bwd (caller-provided workspace)
bit for bit (the same deterministic kernels run), and the first is also
checked against the oracle on one head, with the tolerance the parity tests
use.  It lives in its own file, named to be collected last, and passes alone
in a fresh process as well as after the other tests (its first call sets up
the scratch address on the device).
"""

import numpy as np
import pytest

import hierarchical_top_sparse_llsa_b200 as llsa
from hierarchical_top_sparse_llsa_b200 import workloads
from llsa_testlib import assert_close, run_oracle

pytestmark = pytest.mark.gpu


def _problem(name, seed_shift=0, level_w=None):
    import torch

    w = workloads.WORKLOADS[name]
    if seed_shift:
        w = workloads.Workload(w.name, w.B, w.H, w.N, w.D, w.dtype, w.L, w.topk, w.seed + seed_shift)
    x = workloads.make_inputs(w)
    t = {k: torch.from_numpy(v).to("cuda", dtype=torch.bfloat16) for k, v in x.items()}
    desc = llsa.make_desc(w.B, w.H, w.N, w.D, w.L, w.topk, llsa.BF16, level_w=level_w)
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
    args = (t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), bufs.pyramid, o.data_ptr(),
            lse.data_ptr(), t["do"].data_ptr(), bufs.indices, bufs.csr)
    return w, x, t, desc, bufs, o, s, args


def test_noalloc_backward_matches_workspace_backward_twice():
    import torch

    # an unrelated problem first (other inputs, the paper's level weights):
    # the scratch array then holds its partial sums, not zeros
    w0, _, _, desc0, bufs0, o0, s, args0 = _problem("img64_bf16", seed_shift=77,
                                                     level_w=[0, 0, 256.0, 4096.0])
    junk = [torch.empty_like(o0) for _ in range(3)]
    llsa.llsa_attn_bwd_noalloc(desc0, *args0, *(g.data_ptr() for g in junk), bufs0.status.data_ptr(), s)
    torch.cuda.synchronize()
    assert int(bufs0.status.item()) == 0

    w, x, t, desc, bufs, o, s, args = _problem("img64_bf16")
    assert llsa.llsa_bwd_workspace_bytes(desc) <= llsa.NOALLOC_SCRATCH_BYTES
    ref = [torch.empty_like(o) for _ in range(3)]
    llsa.llsa_attn_bwd(desc, *args, *(g.data_ptr() for g in ref), bufs.ws.data_ptr(), bufs.ws_bytes,
                       bufs.status.data_ptr(), s)
    torch.cuda.synchronize()
    want = [g.float().cpu().numpy() for g in ref]
    for call in range(2):
        got = [torch.full_like(o, float("nan")) for _ in range(3)]
        llsa.llsa_attn_bwd_noalloc(desc, *args, *(g.data_ptr() for g in got), bufs.status.data_ptr(), s)
        torch.cuda.synchronize()
        for name, g, r in zip(("dQ", "dK", "dV"), got, want):
            assert np.array_equal(g.float().cpu().numpy(), r), f"call {call}: {name} differs from llsa_attn_bwd"
        if call == 0:  # and against the oracle, on one head
            heads = [3]
            xs = {k: np.ascontiguousarray(v[:, heads]) for k, v in x.items()}
            r = run_oracle(xs, w.L, w.topk)
            for name, g in zip(("dQ", "dK", "dV"), got):
                assert_close(g.float().cpu().numpy()[:, heads], r[name], "bf16", f"{name} vs the oracle")
    assert int(bufs.status.item()) == 0


@pytest.mark.parametrize("name", ["img128_bf16", "img256_bf16"])
def test_noalloc_rejects_problems_above_its_scratch(name):
    # the scratch holds llsa_bwd_workspace_bytes(desc) up to 16 MiB: the
    # 64x64-pixel workload fits (4.4 MiB); the 128x128 (26.3 MiB) and
    # 256x256 ones do not
    w = workloads.WORKLOADS[name]
    desc = llsa.make_desc(w.B, w.H, w.N, w.D, w.L, w.topk, llsa.BF16)
    assert llsa.llsa_bwd_workspace_bytes(desc) > llsa.NOALLOC_SCRATCH_BYTES
    pyr, ind, csr = llsa.LlsaPyramid(), llsa.LlsaIndices(), llsa.LlsaCsr()
    fake = 256  # never dereferenced: the size check comes first
    st = llsa.llsa_attn_bwd_noalloc(desc, fake, fake, fake, pyr, fake, fake, fake, ind, csr,
                                    fake, fake, fake, check=False)
    assert st == llsa.ERR_WORKSPACE
