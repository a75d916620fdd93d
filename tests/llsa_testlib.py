"""Shared helpers of the tests: run the CUDA path through the C ABI on torch
buffers, run the oracle on the same inputs, and compare."""

from __future__ import annotations

import numpy as np

import oracle
import hierarchical_top_sparse_llsa_b200 as llsa
from hierarchical_top_sparse_llsa_b200 import workloads

BF16_REL = 2e-2  # bf16 inputs: |a - b| <= 2e-2 * max(|b|, rms(b)) elementwise
F32_ABS = 1e-4   # fp32 inputs: max-abs


def clean_indices(I: np.ndarray, n: int):
    """Apply the library's used-entry rule to index rows (entries used iff in
    [0, n) and above the last used one); returns rows in the canonical
    layout (ascending, -1 tail) and the status bits the kernels must report."""
    I = np.asarray(I)
    out = np.full(I.shape, -1, dtype=np.int32)
    flags = 0
    for pos in np.ndindex(*I.shape[:-1]):
        last, seen_pad, kept = -1, False, []
        for v in I[pos]:
            v = int(v)
            if v == -1:
                seen_pad = True
            elif v < -1 or v >= n:
                flags |= llsa.DEV_BAD_INDEX
            elif v <= last:
                flags |= llsa.DEV_NONCANONICAL
            else:
                if seen_pad:
                    flags |= llsa.DEV_NONCANONICAL
                last = v
                kept.append(v)
        out[pos][: len(kept)] = kept
    return out, flags


def assert_close(got, want, dtype: str, what: str):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    fin = np.isfinite(want)
    assert np.array_equal(np.isfinite(got), fin), f"{what}: non-finite pattern differs"
    err = np.abs(got[fin] - want[fin])
    if dtype == "f32":
        worst = err.max(initial=0.0)
        assert worst <= F32_ABS, f"{what}: max-abs {worst:.3g} > {F32_ABS}"
    else:
        rms = np.sqrt(np.mean(want[fin] ** 2)) if fin.any() else 0.0
        bound = BF16_REL * np.maximum(np.abs(want[fin]), rms)
        bad = err > bound
        assert not bad.any(), (
            f"{what}: {bad.sum()} of {bad.size} elements outside 2e-2*max(|ref|, rms); "
            f"worst excess {np.max(err - bound):.3g}, max-abs {err.max():.3g}, rms {rms:.3g}")


def run_gpu(B, H, N, D, L, topk, dtype, inputs, level_w=None, ext_idx=None, bwd=True,
            device="cuda", flags=0, enrich=0, topk_l=None, resid=False):
    """The whole path through the C ABI.  Returns numpy copies of everything.
    resid: run llsa_attn_fwd_res / llsa_attn_bwd_res (Delta from the O
    residual) instead of llsa_attn_fwd / llsa_attn_bwd."""
    import torch

    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    t = {k: torch.from_numpy(np.ascontiguousarray(v)).to(device=device, dtype=tdt) for k, v in inputs.items()}
    desc = llsa.make_desc(B, H, N, D, L, topk, llsa.BF16 if dtype == "bf16" else llsa.F32,
                          level_w=level_w, flags=flags, enrich_levels=enrich, topk_l=topk_l)
    bufs = llsa.LlsaBuffers(desc, device, with_bwd=bwd)
    stream = torch.cuda.current_stream().cuda_stream
    st = bufs.status.data_ptr()
    llsa.llsa_pool(desc, t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), bufs.pyramid, stream)
    llsa.llsa_select(desc, bufs.pyramid, bufs.indices, stream)
    torch.cuda.synchronize()
    out = {"pq": {l: bufs.pq[l].cpu().numpy() for l in bufs.pq},
           "pk": {l: bufs.pk[l].cpu().numpy() for l in bufs.pk},
           "pv": {l: bufs.pv[l].cpu().numpy() for l in bufs.pv},
           "sel": {l: bufs.idx[l].cpu().numpy() for l in bufs.idx}}
    if ext_idx is not None:
        for l, I in ext_idx.items():
            bufs.idx[l].copy_(torch.from_numpy(np.ascontiguousarray(I, dtype=np.int32)))
    o = torch.empty_like(t["q"])
    lse = torch.empty(B, H, N, dtype=torch.float32, device=device)
    o_res = torch.full_like(o, float("nan")) if resid and dtype == "bf16" else None
    if resid:
        llsa.llsa_attn_fwd_res(desc, t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), bufs.pyramid,
                               bufs.indices, o.data_ptr(), o_res.data_ptr() if o_res is not None else None,
                               lse.data_ptr(), st, stream)
    else:
        llsa.llsa_attn_fwd(desc, t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), bufs.pyramid,
                           bufs.indices, o.data_ptr(), lse.data_ptr(), st, stream)
    if bwd:
        llsa.llsa_index_transpose(desc, bufs.indices, bufs.csr, bufs.tr_ws.data_ptr(), bufs.tr_ws_bytes, st, stream)
        dq, dk, dv = torch.empty_like(o), torch.empty_like(o), torch.empty_like(o)
        if resid:
            llsa.llsa_attn_bwd_res(desc, t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), bufs.pyramid,
                                   o.data_ptr(), o_res.data_ptr() if o_res is not None else None,
                                   lse.data_ptr(), t["do"].data_ptr(), bufs.indices, bufs.csr,
                                   dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), bufs.ws.data_ptr(),
                                   bufs.ws_bytes, st, stream)
        else:
            llsa.llsa_attn_bwd(desc, t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), bufs.pyramid,
                               o.data_ptr(), lse.data_ptr(), t["do"].data_ptr(), bufs.indices, bufs.csr,
                               dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), bufs.ws.data_ptr(),
                               bufs.ws_bytes, st, stream)
    torch.cuda.synchronize()
    out["idx"] = {l: bufs.idx[l].cpu().numpy() for l in bufs.idx}
    out["O"] = o.float().cpu().numpy()
    if o_res is not None:
        out["O_res"] = o_res.float().cpu().numpy()
    out["LSE"] = lse.cpu().numpy()
    if bwd:
        out["row_ptr"] = {l: bufs.row_ptr[l].cpu().numpy() for l in bufs.row_ptr}
        out["col"] = {l: bufs.col[l].cpu().numpy() for l in bufs.col}
        out["dQ"] = dq.float().cpu().numpy()
        out["dK"] = dk.float().cpu().numpy()
        out["dV"] = dv.float().cpu().numpy()
    out["status"] = int(bufs.status.item())
    return out


def run_oracle(inputs, L, topk, level_w=None, idx=None, bwd=True, pyr=None, enrich=None):
    """The oracle on the same inputs.  ``idx`` replaces the selection;
    ``pyr`` (a dict with pq, pk, pv) replaces the pooling."""
    Q, K, V = inputs["q"], inputs["k"], inputs["v"]
    D = Q.shape[-1]
    scale = oracle.default_scale(D)
    if pyr is None:
        pyr = {"pq": oracle.pool(Q, L), "pk": oracle.pool(K, L), "pv": oracle.pool(V, L)}
    sel = oracle.select_all(pyr["pq"], pyr["pk"], L, topk) if idx is None else idx
    O, LSE = oracle.attn_fwd(Q, K, V, pyr["pk"], pyr["pv"], sel, L, scale, level_w, enrich=enrich)
    res = {"pq": pyr["pq"], "pk": pyr["pk"], "pv": pyr["pv"], "idx": sel, "O": O, "LSE": LSE}
    if bwd:
        res["csr"] = {l: oracle.index_transpose(sel[l], Q.shape[2] // 16**l) for l in sel}
        res["dQ"], res["dK"], res["dV"] = oracle.attn_bwd(
            Q, K, V, pyr["pk"], pyr["pv"], O, LSE, inputs["do"], sel, L, scale, level_w,
            enrich=enrich)
    return res


# ---------------------------------------------------------------- near ties
# North star's acceptance rule for selected indices: bit-exact, except that a
# near tie may go either way.  The reading taken (the near-tie adjudication of
# the build's reading list): compare level by level against the oracle's
# selection *given the GPU's parent row* (so one tie does not cascade), and
# accept a differing slot only if its fp32 score lies within the rounding
# bound of the K-th kept score.  A dot product of length D summed in any order
# in fp32 is within gamma_D * sum_d |q_d k_d| of the exact value,
# gamma_D = D u / (1 - D u), u = 2^-24 (Higham, recursive summation); two
# computed scores can cross when their exact values are within the sum of
# their two bounds.  Outputs are then compared on the oracle's indices.

def _gamma(D):
    u = 2.0 ** -24
    return D * u / (1.0 - D * u)


def adjudicate_selection(pq, pk, gpu_idx, L, topk):
    """Check the GPU's I(1..L) against the oracle level by level, conditional
    on the GPU's parents.  Returns the number of rows that differ only by near
    ties; raises AssertionError on any other difference.  pq, pk: the pooled
    queries and keys (the GPU's equal the oracle's bit for bit); topk: K or a
    {level: K_l} mapping."""
    from oracle.llsa_oracle import _scores_fp32, candidates_for_level

    kl = (lambda l: topk[l]) if isinstance(topk, dict) else (lambda l: topk)
    near = 0
    for l in range(L, 0, -1):
        parent = None if l == L else np.asarray(gpu_idx[l + 1])
        ref = oracle.select_level(pq[l], pk[l], parent, kl(l))
        got = np.asarray(gpu_idx[l])
        diff = np.argwhere((ref != got).any(-1))
        for b, h, q in diff:
            if parent is None:
                cand = np.arange(pq[l].shape[2])
            else:
                cand = candidates_for_level(parent[b:b + 1, h:h + 1], 16)[0, 0, q // 16]
                cand = cand[cand >= 0]
            qv = np.asarray(pq[l][b, h, q], dtype=np.float32)
            kv = np.asarray(pk[l][b, h][cand], dtype=np.float32)
            s = _scores_fp32(qv[None], kv[None])[0].astype(np.float64)
            bound = _gamma(qv.shape[-1]) * np.abs(qv.astype(np.float64)[None] * kv.astype(np.float64)).sum(-1)
            pos = {int(c): i for i, c in enumerate(cand)}
            kept_ref = [int(c) for c in ref[b, h, q] if c >= 0]
            kept_got = [int(c) for c in got[b, h, q] if c >= 0]
            assert len(kept_ref) == len(kept_got), (l, b, h, q, kept_ref, kept_got)
            kth = min(kept_ref, key=lambda c: (s[pos[c]], -c))  # the oracle's last kept key
            for c in set(kept_ref) ^ set(kept_got):
                assert c in pos, (l, b, h, q, c, "not a candidate")
                gap = abs(s[pos[c]] - s[pos[kth]])
                assert gap <= bound[pos[c]] + bound[pos[kth]], (
                    f"level {l} row {(int(b), int(h), int(q))}: key {c} differs by {gap:.3g}, "
                    f"beyond the rounding bound {bound[pos[c]] + bound[pos[kth]]:.3g}")
            near += 1
    return near


def settle_indices(g, r, x, L, topk, dtype, sl=(slice(None), slice(None)), bwd=True, **run_kw):
    """Indices of the GPU run ``g`` against the oracle's ``r``: equal, or
    differing by near ties only (adjudicated), in which case the path is run
    again on the GPU over the oracle's indices for the heads of ``x``.
    Returns (the run whose outputs to compare, its head slice, the number of
    adjudicated rows)."""
    gidx = {l: g["idx"][l][sl] for l in range(1, L + 1)}
    if all(np.array_equal(gidx[l], r["idx"][l]) for l in gidx):
        return g, sl, 0
    near = adjudicate_selection(r["pq"], r["pk"], gidx, L, topk)
    print(f"{near} index rows differ by near ties only (adjudicated)")
    B, H, N, D = x["q"].shape
    g2 = run_gpu(B, H, N, D, L, topk if not isinstance(topk, dict) else max(topk.values()), dtype, x,
                 ext_idx=r["idx"], bwd=bwd, **run_kw)
    return g2, (slice(None), slice(None)), near


def workload_inputs(name, heads=None):
    w = workloads.WORKLOADS[name]
    return w, workloads.make_inputs(w, heads=heads, with_dout=w.backward)
