"""The whole path (pool, select, forward, transpose, backward) captured in
one CUDA graph and replayed gives the same bits as direct calls: every
entry point only enqueues work on the stream it is given."""

import numpy as np
import pytest

import hierarchical_top_sparse_llsa_b200 as llsa
from hierarchical_top_sparse_llsa_b200 import workloads

pytestmark = pytest.mark.gpu


def test_cuda_graph_replay_matches_direct_calls():
    import torch

    w = workloads.WORKLOADS["img64_bf16"]
    x = workloads.make_inputs(w)
    dev = torch.device("cuda")
    t = {k: torch.from_numpy(v).to(dev, dtype=torch.bfloat16) for k, v in x.items()}
    desc = llsa.make_desc(w.B, w.H, w.N, w.D, w.L, w.topk, llsa.BF16)
    bufs = llsa.LlsaBuffers(desc, dev)
    o = torch.empty_like(t["q"])
    lse = torch.empty(w.B, w.H, w.N, dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty_like(o) for _ in range(3))
    st = bufs.status.data_ptr()

    def step(sh):
        q, k, v = t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr()
        llsa.llsa_pool(desc, q, k, v, bufs.pyramid, sh)
        llsa.llsa_select(desc, bufs.pyramid, bufs.indices, sh)
        llsa.llsa_attn_fwd(desc, q, k, v, bufs.pyramid, bufs.indices, o.data_ptr(), lse.data_ptr(), st, sh)
        llsa.llsa_index_transpose(desc, bufs.indices, bufs.csr, bufs.tr_ws.data_ptr(), bufs.tr_ws_bytes, st, sh)
        llsa.llsa_attn_bwd(desc, q, k, v, bufs.pyramid, o.data_ptr(), lse.data_ptr(), t["do"].data_ptr(),
                           bufs.indices, bufs.csr, dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                           bufs.ws.data_ptr(), bufs.ws_bytes, st, sh)

    outs = lambda: [a.clone() for a in (o, lse, dq, dk, dv)] + [bufs.idx[l].clone() for l in bufs.idx]
    step(torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    direct = outs()
    for a in (o, lse, dq, dk, dv):
        a.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream()
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=cs):
        step(cs.cuda_stream)
    torch.cuda.current_stream().wait_stream(cs)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert int(bufs.status.item()) == 0
    for a, b in zip(direct, outs()):
        assert torch.equal(a.view(torch.uint8) if a.dtype == torch.bfloat16 else a,
                           b.view(torch.uint8) if b.dtype == torch.bfloat16 else b)
