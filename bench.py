#!/usr/bin/env python
"""Throughput of the LLSA hot path (pool -> select -> sparse attention forward
-> sparse index transpose -> sparse attention backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   (the CPU oracle, timed the same way)

One step is one pass of the whole path over one batch of seeded synthetic
input already resident in device memory, replayed as one CUDA graph; the
forward and backward go through the residual calls (llsa_attn_fwd_res /
llsa_attn_bwd_res) unless --no-residual.  Every GPU runs its own copy of
the workload (heads and batches are independent, so the path shards with no
collective): per-GPU work is fixed as N grows, i.e. weak scaling.  Rank 0
prints one JSON line: the step rate, per-stage times against their
rooflines, the end-to-end rate with host copies (pipelined over steps), the
oracle on the host cores, a dense-attention reference, the index transpose
timed back to back and the Z-order permutation's bandwidth.
"""

from __future__ import annotations

import argparse
import hashlib
import datetime
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from hierarchical_top_sparse_llsa_b200 import workloads  # noqa: E402

METRIC = "LLSA fwd+bwd ms & tokens/s at N=65536, % BF16 tensor peak, selection GB/s"
UNIT = "tokens/s"
STAGES = ("pool", "select", "fwd", "transpose", "bwd")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
SMS = 148
FP32_LANES_PER_SM = 128


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    p = dict(FALLBACK_PEAKS)
    p["source"] = "fallback"
    return p


def algorithmic_work(w: workloads.Workload, resid: bool = False) -> dict:
    """Algorithmic bytes and FLOPs of one pass of each stage (no re-reads,
    no gathers counted).  es = bytes per element of Q/K/V/O/dO/dQ/dK/dV.
    resid: the forward also writes the bf16 residual of O and the backward
    reads it (llsa_attn_fwd_res / llsa_attn_bwd_res); those bytes go to
    `resid_bytes`, not to `bytes`."""
    es = 2 if w.dtype == "bf16" else 4
    BH, N, D, K, L = w.B * w.H, w.N, w.D, w.topk, w.L
    fine = BH * N * D * es
    nl = [w.n_level(l) for l in range(L + 1)]
    keff = w.k_eff()
    pyr_qk = sum(BH * nl[l] * D * 4 for l in range(1, L + 1))
    pyr_v = sum(BH * nl[l] * D * 4 for l in range(2, L + 1))
    idx_bytes = sum(BH * nl[l] * K * 4 for l in range(1, L + 1))
    pairs = BH * N * w.keys_per_query()
    cand = [0] * (L + 1)
    cand[L] = nl[L]
    for l in range(L - 1, 0, -1):
        cand[l] = 16 * keff[l + 1]
    work = {
        "pool": {"bytes": 3 * fine + 2 * pyr_qk + pyr_v, "flops": 0, "bound": "hbm"},
        # read Q(l), K(l) and the parent rows, write I(l); fp32 multiply + add per candidate channel
        "select": {"bytes": 2 * pyr_qk + 2 * idx_bytes,
                   "flops": sum(2 * D * BH * nl[l] * cand[l] for l in range(1, L + 1)),
                   "bound": "alu"},
        "fwd": {"bytes": 4 * fine + BH * N * 4, "flops": 4 * D * pairs, "bound": "hbm"},
        "transpose": {"bytes": idx_bytes + idx_bytes + sum(BH * (nl[l] + 1) * 4 for l in range(1, L + 1)),
                      "flops": 0, "bound": "hbm"},
        "bwd": {"bytes": 8 * fine + 2 * BH * N * 4, "flops": 10 * D * pairs, "bound": "hbm"},
    }
    # The residual calls (llsa_attn_fwd_res / llsa_attn_bwd_res) also move the
    # bf16 residual of O: a speed option of this library, not work the method
    # needs, so it is reported beside the method's bytes and never counted in
    # a roofline fraction.
    extra = fine if (resid and w.dtype == "bf16") else 0
    for n in work:
        work[n]["resid_bytes"] = extra if n in ("fwd", "bwd") else 0
    return work


def sources_digest() -> str:
    """sha1 over the library's CUDA sources: ties a committed ncu traffic
    figure to the kernels it was measured on."""
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "hierarchical_top_sparse_llsa_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh")):
            h.update(name.encode())
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(f.read())
    with open(os.path.join(ROOT, "include", "llsa.h"), "rb") as f:
        h.update(f.read())
    return h.hexdigest()


def committed_traffic(workload: str, stage: str):
    """DRAM bytes per call of `stage` from the committed ncu summary of this
    workload, or None when there is none or the sources changed since."""
    path = os.path.join(ROOT, "profiles", f"dram_traffic_{workload}.md")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        text = f.read()
    m = re.search(r"```json\n(.*?)\n```", text, re.S)
    if m is None:
        return None
    try:
        rec = json.loads(m.group(1))
    except ValueError:
        return None
    if rec.get("sources_sha1") != sources_digest():
        return None
    st = rec.get("stages", {}).get(stage)
    return None if st is None else st.get("dram_bytes_per_call")


def dense_reference(torch, w, dev, iters=3):
    """Dense attention at the same B, H, N, D through torch's
    scaled_dot_product_attention (library kernels, bf16), forward and
    forward + backward: the comparison point for the sparse path.  Not part
    of the LLSA path or of its timed region."""
    import torch.nn.functional as F

    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    gen = torch.Generator(device=dev)
    gen.manual_seed(4242)
    shape = (w.B, w.H, w.N, w.D)
    q, k, v = (torch.randn(shape, device=dev, dtype=dt, generator=gen).requires_grad_() for _ in range(3))
    do = torch.randn(shape, device=dev, dtype=dt, generator=gen)

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(iters):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / iters

    with torch.no_grad():
        fwd_ms = timed(lambda: F.scaled_dot_product_attention(q, k, v))

    def fwd_bwd():
        q.grad = k.grad = v.grad = None
        F.scaled_dot_product_attention(q, k, v).backward(do)

    fb_ms = timed(fwd_bwd)
    del q, k, v, do
    torch.cuda.empty_cache()
    return {"impl": "torch.nn.functional.scaled_dot_product_attention (bf16, library kernels)",
            "fwd_ms": round(fwd_ms, 3), "fwd_bwd_ms": round(fb_ms, 3), "iters": iters}


def qkv_projection(torch, llsa, w, dev, pool_ms, step_ms, tens, iters=10):
    """The step before the path: the QKV projection of a model of width
    C = H * D, fused with the pool (llsa_qkv_pool: tcgen05 GEMM whose epilogue
    writes Q, K, V head-major and the pyramid) against the unfused sequence
    (cuBLAS GEMM through torch.matmul, the head-major relayout, llsa_pool).
    Reports both and the step time with each in front of it.  Not part of the
    timed step."""
    C = w.H * w.D
    if w.dtype != "bf16" or C % 128 != 0 or w.N % 256 != 0:
        return None
    gen = torch.Generator(device=dev)
    gen.manual_seed(777)
    x = torch.randn(w.B, w.N, C, device=dev, dtype=torch.bfloat16, generator=gen)
    wt = (torch.randn(3 * C, C, device=dev, generator=gen) / C ** 0.5).to(torch.bfloat16)
    desc = llsa.make_desc(w.B, w.H, w.N, w.D, w.L, w.topk, llsa.BF16)
    fused = llsa.LlsaBuffers(desc, dev, with_bwd=False)
    plain = llsa.LlsaBuffers(desc, dev, with_bwd=False)
    qkv = [torch.empty(w.B, w.H, w.N, w.D, device=dev, dtype=torch.bfloat16) for _ in range(3)]
    sh = torch.cuda.current_stream(dev).cuda_stream
    holder = {}

    def fused_call():
        llsa.llsa_qkv_pool(desc, x.data_ptr(), wt.data_ptr(), C, qkv[0].data_ptr(), qkv[1].data_ptr(),
                           qkv[2].data_ptr(), fused.pyramid, fused.status.data_ptr(), sh)

    def gemm():
        holder["y"] = torch.matmul(x.view(-1, C), wt.t())

    def relayout():
        holder["t"] = holder["y"].view(w.B, w.N, 3, w.H, w.D).permute(2, 0, 3, 1, 4).contiguous()

    def pool():
        t = holder["t"]
        llsa.llsa_pool(desc, t[0].data_ptr(), t[1].data_ptr(), t[2].data_ptr(), plain.pyramid, sh)

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(iters):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / iters

    f_ms = timed(fused_call)
    g_ms = timed(gemm)
    r_ms = timed(relayout)
    p_ms = timed(pool)
    if int(fused.status.item()) != 0:
        raise RuntimeError(f"llsa_qkv_pool device status {int(fused.status.item())}")
    flops = 2.0 * w.B * w.N * C * 3 * C
    unfused = g_ms + r_ms + p_ms
    out = {"C": C, "flops": flops, "iters": iters, "l2": "X larger than L2" if x.numel() * 2 > L2_BYTES else "X in L2",
           "fused_ms": round(f_ms, 4), "fused_TFLOPs": round(flops / (f_ms * 1e-3) / 1e12, 1),
           "fused_frac_bf16_tensor": round(flops / (f_ms * 1e-3) / 1e12 / tens, 4),
           "cublas_gemm_ms": round(g_ms, 4), "cublas_TFLOPs": round(flops / (g_ms * 1e-3) / 1e12, 1),
           "relayout_ms": round(r_ms, 4), "pool_ms": round(p_ms, 4), "unfused_ms": round(unfused, 4),
           "step_ms_with_projection": {"fused": round(step_ms - pool_ms + f_ms, 4),
                                       "unfused": round(step_ms - pool_ms + unfused, 4)}}
    del x, wt, fused, plain, qkv, holder
    torch.cuda.empty_cache()
    return out


def max_over_ranks(torch, dist, values, device) -> list:
    """Element-wise maximum of per-rank timings (one all_reduce): the job's
    time is its slowest rank's."""
    t = torch.tensor([float(v) for v in values], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def reorder_rate(torch, llsa, w, dev, src, hbm_gbs, iters=10):
    """Raster -> Z-order permutation of one [B, H, N, D] tensor (llsa_reorder,
    for callers that hold raster-order tokens): ms per call and GB/s of its
    compulsory traffic (read + write once).  Not part of the step."""
    side = int(round(w.N ** 0.5))
    if side * side != w.N:
        return None
    dst = torch.empty_like(src)
    sh = torch.cuda.current_stream(dev).cuda_stream
    dt = llsa.BF16 if src.dtype == torch.bfloat16 else llsa.F32
    call = lambda: llsa.llsa_reorder(w.B, w.H, side, side, w.D, dt, src.data_ptr(), dst.data_ptr(), True, sh)
    call()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(iters):
        call()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / iters
    gbs = 2 * src.numel() * src.element_size() / (ms * 1e-3) / 1e9
    return {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm_gbs, 4),
            "tensor": f"[{w.B}, {w.H}, {w.N}, {w.D}] {str(src.dtype).replace('torch.', '')}"}


def gathered_select_bytes(w: workloads.Workload) -> int:
    """Candidate K(l) rows the selection loads (fp32), once per group of 16
    sibling queries (they share one candidate list), plus the Q(l) rows."""
    BH, D, L = w.B * w.H, w.D, w.L
    keff = w.k_eff()
    total = 0
    for l in range(1, L + 1):
        n = w.n_level(l)
        groups = -(-n // 16)
        cand = n if l == L else 16 * keff[l + 1]
        total += BH * (groups * cand + n) * D * 4
    return total


def transpose_graph_rate(torch, llsa, desc, bufs, dev, hbm_gbs, compulsory, repeats=20):
    """The index transpose as `repeats` back-to-back calls in one CUDA graph
    (launch gaps removed): ms per call and GB/s of its compulsory bytes."""
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    g = torch.cuda.CUDAGraph()
    call = lambda: llsa.llsa_index_transpose(desc, bufs.indices, bufs.csr, bufs.tr_ws.data_ptr(), bufs.tr_ws_bytes,
                                             None, s.cuda_stream)
    with torch.cuda.stream(s):
        call()
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=s):
        for _ in range(repeats):
            call()
    g.replay()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    g.replay()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / repeats
    gbs = compulsory / (ms * 1e-3) / 1e9
    del g
    return {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm_gbs, 4),
            "repeats_in_graph": repeats}


def transpose_512_k32(torch, llsa, dev, hbm_gbs):
    """The index transpose at the 512x512-pixel, K = 32 shape (B = 1, H = 8,
    N = 262144, D = 128, L = 4: 36 MB of lists), where its compulsory bytes
    are large enough to measure bandwidth.  Its indices come from the path's
    own pool and selection on device-drawn N(0, 1) inputs (only the index
    pattern matters here)."""
    w = workloads.WORKLOADS["img512_k32_bf16"]
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed)
    x = [torch.randn(w.B, w.H, w.N, w.D, device=dev, dtype=torch.bfloat16, generator=g) for _ in range(3)]
    desc = llsa.make_desc(w.B, w.H, w.N, w.D, w.L, w.topk, llsa.BF16)
    bufs = llsa.LlsaBuffers(desc, dev, with_bwd=True)
    sh = torch.cuda.current_stream(dev).cuda_stream
    llsa.llsa_pool(desc, x[0].data_ptr(), x[1].data_ptr(), x[2].data_ptr(), bufs.pyramid, sh)
    llsa.llsa_select(desc, bufs.pyramid, bufs.indices, sh)
    torch.cuda.synchronize()
    del x
    work = algorithmic_work(w)["transpose"]["bytes"]
    rec = transpose_graph_rate(torch, llsa, desc, bufs, dev, hbm_gbs, work)
    rec["workload"] = f"{w.name}: N={w.N}, B={w.B}, H={w.H}, L={w.L}, K={w.topk}"
    del bufs
    torch.cuda.empty_cache()
    return rec


def select_scaling(args):
    """Selection cost against N: hierarchical (the levels of the path's
    workloads: L = 3 up to 256x256 pixels, 4 at 512x512) and single-level (L = 1: every query block scores every
    key block, the prior-art baseline the pages compare with), on the same
    kernels, B = 1, H = 8, D = 64, K = 8, bf16 inputs of the synthetic
    image-like recipe.  Prints one JSON line; not part of the step."""
    import torch

    import hierarchical_top_sparse_llsa_b200 as llsa

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    out = []
    for side in (64, 128, 256, 512):
        N = side * side
        Lh = {64: 3, 128: 3, 256: 3, 512: 4}[side]
        w = workloads.Workload(f"sel{side}", 1, 8, N, 64, "bf16", Lh, 8, 2000 + side, backward=False)
        x = workloads.make_inputs(w, with_dout=False)
        q, k, v = (torch.from_numpy(x[n]).to(dev, dtype=torch.bfloat16) for n in ("q", "k", "v"))
        rec = {"side": side, "N": N}
        for L in (Lh, 1):
            desc = llsa.make_desc(w.B, w.H, N, 64, L, 8, llsa.BF16)
            bufs = llsa.LlsaBuffers(desc, dev, with_bwd=False)
            sh = torch.cuda.current_stream(dev).cuda_stream
            llsa.llsa_pool(desc, q.data_ptr(), k.data_ptr(), v.data_ptr(), bufs.pyramid, sh)
            llsa.llsa_select(desc, bufs.pyramid, bufs.indices, sh)
            torch.cuda.synchronize()
            iters = 5 if L == 1 and side >= 512 else 20
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(iters):
                llsa.llsa_select(desc, bufs.pyramid, bufs.indices, sh)
            b.record()
            torch.cuda.synchronize()
            rec["hierarchical_ms" if L == Lh else "flat_ms"] = round(a.elapsed_time(b) / iters, 4)
            if L == Lh:
                rec["levels"] = Lh
            del bufs
        rec["flat_over_hierarchical"] = round(rec["flat_ms"] / rec["hierarchical_ms"], 2)
        out.append(rec)
        del q, k, v
        torch.cuda.empty_cache()
    print(json.dumps({"select_scaling": out, "B": 1, "H": 8, "D": 64, "topk": 8, "dtype": "bf16",
                      "data": "synthetic image-like"}), flush=True)


def launches_per_step(L: int) -> dict:
    """Kernels each entry point launches (matches the C library's dispatch)."""
    return {"pool": 1 + max(0, L - 2), "select": L, "fwd": 1, "transpose": 4,
            "bwd": 2 + max(0, L - 1) + max(0, L - 2)}


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 7:
                continue
            try:
                sm.append(float(f[0]))
                smax = float(f[1])
            except ValueError:
                continue
            for n, v in zip(names, f[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_selector(torch, dev):
    try:
        p = torch.cuda.get_device_properties(dev)
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        return vis.split(",")[dev] if vis else str(dev)


# ------------------------------------------------------------- CPU oracle
def oracle_sample(w, x_head, stages=None):
    """The oracle's whole path on a head slice (a bounded sample of the
    workload); returns the seconds it took and, in ``stages`` if given, the
    seconds of each stage."""
    import oracle

    L, K = w.L, w.topk
    scale = oracle.default_scale(w.D)
    st = {} if stages is None else stages
    t0 = time.perf_counter()
    pq, pk, pv = oracle.pool(x_head["q"], L), oracle.pool(x_head["k"], L), oracle.pool(x_head["v"], L)
    t1 = time.perf_counter()
    idx = oracle.select_all(pq, pk, L, K)
    t2 = time.perf_counter()
    O, LSE = oracle.attn_fwd(x_head["q"], x_head["k"], x_head["v"], pk, pv, idx, L, scale)
    t3 = time.perf_counter()
    st.update(pool=t1 - t0, select=t2 - t1, fwd=t3 - t2)
    if w.backward:
        for l in range(1, L + 1):
            oracle.index_transpose(idx[l], w.n_level(l))
        t4 = time.perf_counter()
        oracle.attn_bwd(x_head["q"], x_head["k"], x_head["v"], pk, pv, O, LSE, x_head["do"], idx, L, scale)
        t5 = time.perf_counter()
        st.update(transpose=t4 - t3, bwd=t5 - t4)
    return time.perf_counter() - t0


def oracle_one_thread(name="img64_bf16"):
    """The oracle on one head of a small workload with one BLAS thread: the
    single-core figure of the CPU baseline (seconds and tokens/s)."""
    w = workloads.WORKLOADS[name]
    x = workloads.make_inputs(w, heads=[0], with_dout=w.backward)
    try:
        from threadpoolctl import threadpool_limits
    except Exception:  # threadpoolctl missing: report the default threads
        threadpool_limits = None
    if threadpool_limits is not None:
        with threadpool_limits(limits=1):
            t = oracle_sample(w, x)
    else:
        t = oracle_sample(w, x)
    return {"workload": name, "sample": "head 0 (B*N/H tokens)", "threads": 1 if threadpool_limits else None,
            "seconds": round(t, 3), "tokens/s": round(w.B * w.N / w.H / t, 1)}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def cpu_sample_inputs(w):
    x = workloads.make_inputs(w, heads=[0], with_dout=w.backward)
    return x


L2_BYTES = 126 * 2**20  # B200


def config_of(w, world):
    es = 2 if w.dtype == "bf16" else 4
    inputs = (4 if w.backward else 3) * w.B * w.H * w.N * w.D * es
    l2 = ("inputs larger than L2 (no flush needed)" if inputs > L2_BYTES else
          f"inputs {inputs / 2**20:.1f} MiB fit in L2: warm-cache timing (a small parity workload)")
    return {"workload": f"{w.name}: {w.side}x{w.side} pixels, N={w.N}, B={w.B}, H={w.H}, D={w.D}, "
                        f"L={w.L}, K={w.topk}, {'fwd+bwd' if w.backward else 'fwd only'}",
            "B": w.B, "H": w.H, "N": w.N, "D": w.D, "L": w.L, "topk": w.topk,
            "l2": l2,
            "parallelism": f"replicas x{world} (no collective)"}


# --------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    w = workloads.WORKLOADS[args.workload]
    if rank != 0:
        return
    x = cpu_sample_inputs(w)
    for _ in range(args.warmup):
        oracle_sample(w, x)
    times = [oracle_sample(w, x) for _ in range(args.steps)]
    t = sum(times) / len(times)
    value = w.B * w.N / w.H / t  # one head of B*N tokens out of H
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(w, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"whole path on head 0 of {w.H} (B*N/H tokens per step)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import hierarchical_top_sparse_llsa_b200 as llsa

    w = workloads.WORKLOADS[args.workload]
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    peaks = load_peaks()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        nh = min(4, w.H)
        xc = workloads.make_inputs(w, heads=slice(0, nh), with_dout=w.backward)
        stage_s = {}
        t = oracle_sample(w, xc, stage_s)
        cpu = {"value": w.B * w.N * nh / w.H / t, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"oracle whole path on heads 0..{nh - 1} of {w.H} ({t:.1f} s)",
               "stage_seconds": {k: round(v, 3) for k, v in stage_s.items()},
               "one_thread": oracle_one_thread()}

    x = workloads.make_inputs(w, with_dout=w.backward)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    t_in = {k: torch.from_numpy(v).to(dev, dtype=tdt) for k, v in x.items()}
    host = {k: torch.from_numpy(v).to(dtype=tdt).pin_memory() for k, v in x.items()}
    del x
    desc = llsa.make_desc(w.B, w.H, w.N, w.D, w.L, w.topk, llsa.BF16 if w.dtype == "bf16" else llsa.F32,
                          flags=(llsa.FLAG_FWD_MMA_SYNC if args.fwd_mma_sync else 0)
                          | (llsa.FLAG_FWD_TCGEN05 if args.fwd_tcgen05 else 0)
                          | (llsa.FLAG_BWD_TCGEN05 if args.bwd_tcgen05 else 0))
    bufs = llsa.LlsaBuffers(desc, dev, with_bwd=w.backward)
    o = torch.empty_like(t_in["q"])
    lse = torch.empty(w.B, w.H, w.N, dtype=torch.float32, device=dev)
    grads = [torch.empty_like(o) for _ in range(3)] if w.backward else []
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    st = bufs.status.data_ptr()

    fuse = args.fuse_select
    resid = not args.no_residual and w.dtype == "bf16" and not fuse
    o_res = torch.empty_like(o) if resid else None

    def step(tin, ev=None, sh=sh):
        # ev given: the stages as separate calls with events between them;
        # otherwise the step as timed (with --fuse-select, the level-1
        # selection inside the forward)
        q, k, v = tin["q"].data_ptr(), tin["k"].data_ptr(), tin["v"].data_ptr()
        if ev is not None:
            ev[0].record(stream)
        llsa.llsa_pool(desc, q, k, v, bufs.pyramid, sh)
        if ev is not None:
            ev[1].record(stream)
        if fuse and ev is None:
            llsa.llsa_select_attn_fwd(desc, q, k, v, bufs.pyramid, bufs.indices, o.data_ptr(), lse.data_ptr(),
                                      st, sh)
        else:
            llsa.llsa_select(desc, bufs.pyramid, bufs.indices, sh)
            if ev is not None:
                ev[2].record(stream)
            if resid:
                llsa.llsa_attn_fwd_res(desc, q, k, v, bufs.pyramid, bufs.indices, o.data_ptr(), o_res.data_ptr(),
                                       lse.data_ptr(), st, sh)
            else:
                llsa.llsa_attn_fwd(desc, q, k, v, bufs.pyramid, bufs.indices, o.data_ptr(), lse.data_ptr(), st,
                                   sh)
        if ev is not None:
            ev[3].record(stream)
        if w.backward:
            llsa.llsa_index_transpose(desc, bufs.indices, bufs.csr, bufs.tr_ws.data_ptr(), bufs.tr_ws_bytes, st, sh)
            if ev is not None:
                ev[4].record(stream)
            dq, dk, dv = grads
            if resid:
                llsa.llsa_attn_bwd_res(desc, q, k, v, bufs.pyramid, o.data_ptr(), o_res.data_ptr(), lse.data_ptr(),
                                       tin["do"].data_ptr(), bufs.indices, bufs.csr, dq.data_ptr(),
                                       dk.data_ptr(), dv.data_ptr(), bufs.ws.data_ptr(), bufs.ws_bytes, st, sh)
            else:
                llsa.llsa_attn_bwd(desc, q, k, v, bufs.pyramid, o.data_ptr(), lse.data_ptr(),
                                   tin["do"].data_ptr(), bufs.indices, bufs.csr, dq.data_ptr(),
                                   dk.data_ptr(), dv.data_ptr(), bufs.ws.data_ptr(), bufs.ws_bytes, st, sh)
            if ev is not None:
                ev[5].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step(t_in)
    torch.cuda.synchronize()
    if int(bufs.status.item()) != 0:
        raise RuntimeError(f"device status {int(bufs.status.item())} during warm-up")

    # the whole step as one CUDA graph (its 15 launches replayed without host
    # round trips or launch gaps); the per-stage breakdown below comes from
    # a separate loop of direct calls with events between the stages
    graph, graph_note = None, "disabled (--no-graph)"
    if not args.no_graph:
        try:
            g = torch.cuda.CUDAGraph()
            cs = torch.cuda.Stream(dev)
            cs.wait_stream(stream)
            with torch.cuda.graph(g, stream=cs):
                step(t_in, None, cs.cuda_stream)
            stream.wait_stream(cs)
            g.replay()
            torch.cuda.synchronize()
            graph, graph_note = g, "captured"
        except RuntimeError as exc:  # capture refused: time direct calls instead
            torch.cuda.synchronize()
            graph_note = f"not captured ({str(exc).splitlines()[0][:120]})"

    nst = 6 if w.backward else 4
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nst)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(gpu_selector(torch, local_rank)) if rank == 0 else None
    if sampler:
        sampler.__enter__()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for s in range(args.steps):
        if graph is not None:
            graph.replay()
        else:
            step(t_in)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    if sampler:
        sampler.__exit__()
    ms = t_start.elapsed_time(t_end) / args.steps
    for s in range(args.steps):  # stage breakdown from separate direct calls
        step(t_in, evs[s])
    torch.cuda.synchronize()
    stage_ms = {}
    names = STAGES if w.backward else STAGES[:3]
    for i, name in enumerate(names):
        stage_ms[name] = statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs)

    # end to end: pinned host inputs -> device -> path -> results back to pinned host
    e2e_steps = max(1, min(args.steps, 8))
    h_out = {"o": torch.empty(o.shape, dtype=o.dtype).pin_memory(),
             "lse": torch.empty(lse.shape, dtype=lse.dtype).pin_memory()}
    if w.backward:
        for n in ("dq", "dk", "dv"):
            h_out[n] = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    d_out = {"o": o, "lse": lse}
    if w.backward:
        d_out.update(dq=grads[0], dk=grads[1], dv=grads[2])
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in h_out.values())
    # Pipelined as a training loop would run it: step k+1's inputs go up on
    # one copy stream and step k-1's results come down on another while step
    # k computes (two device input sets; the results are staged by a
    # device-to-device copy so the next step may overwrite them).  Every
    # step's copies are inside the timed region, the first upload and the
    # last download included.
    sets = [t_in, {k_: torch.empty_like(t_) for k_, t_ in t_in.items()}]
    staged = {k_: torch.empty_like(t_) for k_, t_ in d_out.items()}
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in_ready = [torch.cuda.Event(), torch.cuda.Event()]
    ev_in_free = [torch.cuda.Event(), torch.cuda.Event()]
    ev_out_ready, ev_out_free = torch.cuda.Event(), torch.cuda.Event()

    def upload(k):
        with torch.cuda.stream(s_up):
            for k_, t_ in host.items():
                sets[k % 2][k_].copy_(t_, non_blocking=True)
        ev_in_ready[k % 2].record(s_up)

    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_up.wait_stream(stream)
    s_down.wait_stream(stream)
    upload(0)
    for k in range(e2e_steps):
        if k + 1 < e2e_steps:
            if k >= 1:  # the set step k+1 uploads into was step k-1's
                s_up.wait_event(ev_in_free[(k + 1) % 2])
            upload(k + 1)
        stream.wait_event(ev_in_ready[k % 2])
        step(sets[k % 2])
        ev_in_free[k % 2].record(stream)
        if k >= 1:  # the staging buffers still hold step k-1's results
            stream.wait_event(ev_out_free)
        for k_, t_ in d_out.items():
            staged[k_].copy_(t_, non_blocking=True)
        ev_out_ready.record(stream)
        s_down.wait_event(ev_out_ready)
        with torch.cuda.stream(s_down):
            for k_, t_ in staged.items():
                h_out[k_].copy_(t_, non_blocking=True)
        ev_out_free.record(s_down)
    stream.wait_stream(s_up)
    stream.wait_stream(s_down)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps

    if world > 1:
        ms, e2e_ms = max_over_ranks(torch, dist, [ms, e2e_ms], dev)
    if int(bufs.status.item()) != 0:
        raise RuntimeError(f"device status {int(bufs.status.item())}")
    if rank != 0:
        return

    tokens = w.B * w.N
    work = algorithmic_work(w, resid)
    hbm = peaks["hbm_gbs"]
    # the step is timed as a short burst (tens of ms), so the burst GEMM
    # figure is the denominator; the sustained one is reported beside it
    tens = peaks["bf16_tflops"]
    tens_sus = peaks["bf16_tflops_sustained"]
    alu_peak = SMS * FP32_LANES_PER_SM * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12  # TFLOP/s, one op per lane-cycle
    stages = {}
    for n, t_ms in stage_ms.items():
        wk = work[n]
        gbs = wk["bytes"] / (t_ms * 1e-3) / 1e9
        tfl = wk["flops"] / (t_ms * 1e-3) / 1e12
        stages[n] = {"ms": round(t_ms, 4), "tokens/s": round(tokens / (t_ms * 1e-3)), "GB/s": round(gbs, 1),
                     "TFLOP/s": round(tfl, 2), "frac_hbm": round(gbs / hbm, 4),
                     "frac_bf16_tensor": round(tfl / tens, 4)}
        if wk.get("resid_bytes"):
            stages[n]["resid_bytes"] = wk["resid_bytes"]
        if wk["bound"] == "alu":
            stages[n]["frac_fp32_alu"] = round(tfl / alu_peak, 4)
        # the binding roofline: the slower of its memory and its arithmetic floor
        t_floor = max(wk["bytes"] / (hbm * 1e9), wk["flops"] / ((alu_peak if wk["bound"] == "alu" else tens) * 1e12))
        stages[n]["frac_binding"] = round(t_floor / (t_ms * 1e-3), 4)
    dom = max(stage_ms, key=stage_ms.get)
    wk = work[dom]
    if wk["bound"] == "alu":
        achieved = wk["flops"] / (stage_ms[dom] * 1e-3) / 1e12
        roof = {"bound": "alu", "achieved": achieved, "peak": alu_peak, "unit": "TFLOP/s"}
    else:
        achieved = wk["bytes"] / (stage_ms[dom] * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = committed_traffic(args.workload, dom)
    roof["traffic_source"] = (f"profiles/dram_traffic_{args.workload}.md (ncu dram__bytes_read.sum + "
                              "dram__bytes_write.sum, summed over the call's launches)"
                              if roof["traffic"] is not None else
                              "null: no ncu capture of the current sources")
    roof["kernel"] = f"llsa_{'attn_' if dom in ('fwd', 'bwd') else ''}{dom} ({launches_per_step(w.L)[dom]} launches)"
    roof["peak_source"] = f"{peaks['source']} (MEASURED_PEAKS.json)" if peaks["source"] == "measured" else "fallback"
    reorder = reorder_rate(torch, llsa, w, dev, t_in["q"], peaks["hbm_gbs"])
    proj = None if args.no_projection else qkv_projection(torch, llsa, w, dev, stage_ms["pool"], ms, tens)
    tr_graph = None
    if w.backward and not args.no_transpose_graph:
        tr_graph = {"headline": transpose_graph_rate(torch, llsa, desc, bufs, dev, hbm, work["transpose"]["bytes"])}
        tr_graph["img512_k32"] = transpose_512_k32(torch, llsa, dev, hbm)
    dense = None
    if w.backward and not args.no_dense:
        dense = dense_reference(torch, w, dev)
        dense["llsa_fwd_ms"] = round(stage_ms["fwd"], 4)
        dense["llsa_fwd_bwd_ms"] = round(stage_ms["fwd"] + stage_ms["bwd"], 4)
        dense["speedup_fwd"] = round(dense["fwd_ms"] / stage_ms["fwd"], 2)
        dense["speedup_fwd_bwd"] = round(dense["fwd_bwd_ms"] / dense["llsa_fwd_bwd_ms"], 2)
        # (query, key) pairs per second through each: dense attention scores all
        # N^2 pairs of a head, the sparse path B*H*N*keys-per-query; the
        # kernels' own dense form (every block selected, L = 1) would need rows
        # of N/16 keys, beyond the K <= 32 their selection rows hold
        dense_pairs = w.B * w.H * float(w.N) ** 2
        sparse_pairs = w.B * w.H * float(w.N) * w.keys_per_query()
        dense["pairs_per_s"] = {
            "dense_fwd": dense_pairs / (dense["fwd_ms"] * 1e-3),
            "llsa_fwd": sparse_pairs / (stage_ms["fwd"] * 1e-3),
            "dense_fwd_bwd": dense_pairs / (dense["fwd_bwd_ms"] * 1e-3),
            "llsa_fwd_bwd": sparse_pairs / (dense["llsa_fwd_bwd_ms"] * 1e-3),
            "keys_per_query": w.keys_per_query(),
        }
    attn_ms = stage_ms["fwd"] + stage_ms.get("bwd", 0.0)
    attn_flops = work["fwd"]["flops"] + (work["bwd"]["flops"] if w.backward else 0)
    sel_ms = stage_ms["pool"] + stage_ms["select"]
    # the fused call saves the level-1 selection launch on the bf16 warp-MMA forward
    fwd_is_mma = args.fwd_mma_sync or (w.D == 64 and not args.fwd_tcgen05)
    fused_saves = fuse and w.dtype == "bf16" and fwd_is_mma
    nlaunch = sum(launches_per_step(w.L)[n] for n in names) - (1 if fused_saves else 0)
    line = {
        "metric": METRIC, "value": world * tokens / (ms * 1e-3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": config_of(w, world),
        "stages": stages,
        "fwd_bwd_ms": attn_ms,
        "fwd_bwd_frac_bf16_tensor": attn_flops / (attn_ms * 1e-3) / 1e12 / tens,
        "fwd_bwd_frac_bf16_tensor_sustained": attn_flops / (attn_ms * 1e-3) / 1e12 / tens_sus,
        "tensor_peak_source": "bf16_tflops (burst) of MEASURED_PEAKS.json; _sustained: bf16_tflops_sustained",
        "selection_GBps": (work["pool"]["bytes"] + work["select"]["bytes"]) / (sel_ms * 1e-3) / 1e9,
        "select_gathered_GBps": gathered_select_bytes(w) / (stage_ms["select"] * 1e-3) / 1e9,
        "transpose_graph": tr_graph,
        "roofline": roof,
        "cpu_baseline": cpu,
        "dense_reference": dense,
        "reorder": reorder,
        "qkv_projection": proj,
        "e2e": {"value": world * tokens / (e2e_ms * 1e-3), "unit": UNIT, "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "pipelined": "uploads of step k+1 and downloads of step k-1 overlap step k"},
        "gpu_launches": nlaunch * args.steps,
        "cuda_graph": graph_note,
        "select_in_fwd": fuse,
        "o_residual": resid,
        "clocks": sampler.summary() if sampler else None,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=workloads.HEADLINE, choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--select-scaling", action="store_true",
                    help="time hierarchical vs single-level selection against N (separate report)")
    ap.add_argument("--no-graph", action="store_true",
                    help="time direct calls instead of a CUDA graph of the step")
    ap.add_argument("--no-dense", action="store_true",
                    help="skip the dense scaled_dot_product_attention comparison")
    ap.add_argument("--bwd-tcgen05", action="store_true",
                    help="run the key-major backward pass on the tcgen05 kernel (bf16, D=64)")
    ap.add_argument("--fwd-mma-sync", action="store_true",
                    help="force the forward onto the warp-level mma.sync kernel (bf16; the D=64 default)")
    ap.add_argument("--fwd-tcgen05", action="store_true",
                    help="force the forward onto the tcgen05 kernel (bf16; the D=128 default)")
    ap.add_argument("--no-transpose-graph", action="store_true",
                    help="skip the index transpose timed as back-to-back calls in a CUDA graph")
    ap.add_argument("--no-residual", action="store_true",
                    help="time llsa_attn_fwd + llsa_attn_bwd (two walks of each key list) instead of the "
                         "_res calls (Delta from the bf16 residual of O)")
    ap.add_argument("--no-projection", action="store_true",
                    help="skip the QKV-projection comparison (llsa_qkv_pool against cuBLAS + llsa_pool)")
    ap.add_argument("--fuse-select", action="store_true",
                    help="time llsa_select_attn_fwd (level-1 selection in the forward's prologue) "
                         "instead of llsa_select + llsa_attn_fwd")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be at least 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    if args.select_scaling:
        select_scaling(args)
        return
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
