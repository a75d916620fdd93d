"""Host-side logic of bench.py: the algorithmic work behind the roofline
fractions, the launch count, the committed-traffic lookup and the
max-over-ranks timing of multi-process runs (gloo, two ranks, CPU)."""

import os
import socket

import pytest
import torch.multiprocessing as mp

import bench
from hierarchical_top_sparse_llsa_b200 import workloads


def test_algorithmic_work_headline():
    # 256x256 pixels: B=1, H=16, N=65536, D=64, L=3, K=8 (144 keys per query)
    w = workloads.WORKLOADS["img256_bf16"]
    assert w.keys_per_query() == 144
    work = bench.algorithmic_work(w)
    pairs = 16 * 65536 * 144
    assert work["fwd"]["flops"] == 4 * 64 * pairs and abs(work["fwd"]["flops"] - 3.87e10) < 0.01e10
    assert work["bwd"]["flops"] == 10 * 64 * pairs
    fine = 16 * 65536 * 64 * 2
    assert work["fwd"]["bytes"] == 4 * fine + 16 * 65536 * 4
    assert abs(work["pool"]["bytes"] - 440e6) < 10e6
    assert abs(work["transpose"]["bytes"] - 4.8e6) < 0.2e6


def test_residual_is_reported_beside_the_method_bytes():
    # the residual calls move one more bf16 tensor each way (the forward
    # writes the residual of O, the backward reads it); that is this
    # library's speed option, so it goes to resid_bytes and the method's
    # bytes, the roofline numerator, stay the same
    w = workloads.WORKLOADS["img256_bf16"]
    fine = 16 * 65536 * 64 * 2
    plain, res = bench.algorithmic_work(w), bench.algorithmic_work(w, True)
    for n in plain:
        assert res[n]["bytes"] == plain[n]["bytes"]
        assert res[n]["flops"] == plain[n]["flops"]
    assert res["fwd"]["resid_bytes"] == fine and res["bwd"]["resid_bytes"] == fine
    assert plain["fwd"]["resid_bytes"] == 0 and res["pool"]["resid_bytes"] == 0
    assert plain["bwd"]["bytes"] == 8 * fine + 2 * 16 * 65536 * 4
    f32 = workloads.WORKLOADS["tiny_32x32_f32"]
    assert bench.algorithmic_work(f32, True) == bench.algorithmic_work(f32)  # no residual in fp32


def test_gathered_selection_bytes_headline():
    # per (b, h): level 3 one group of 16 queries scoring all 16 tokens; level 2
    # 16 groups of 16 queries x 16 * 8 candidates; level 1 256 groups x 128;
    # plus the Q(l) rows; fp32, D = 64, 16 heads
    w = workloads.WORKLOADS["img256_bf16"]
    rows = (1 * 16 + 16) + (16 * 128 + 256) + (256 * 128 + 4096)
    assert bench.gathered_select_bytes(w) == 16 * rows * 64 * 4


def test_launch_count_per_step():
    assert bench.launches_per_step(3) == {"pool": 2, "select": 3, "fwd": 1, "transpose": 4, "bwd": 5}
    assert sum(bench.launches_per_step(2).values()) == 1 + 2 + 1 + 4 + 3


def _fake_tree(root, src):
    os.makedirs(os.path.join(root, "hierarchical_top_sparse_llsa_b200", "csrc"))
    os.makedirs(os.path.join(root, "include"))
    os.makedirs(os.path.join(root, "profiles"))
    with open(os.path.join(root, "hierarchical_top_sparse_llsa_b200", "csrc", "k.cu"), "w") as f:
        f.write(src)
    with open(os.path.join(root, "include", "llsa.h"), "w") as f:
        f.write("/* header */\n")


def test_committed_traffic_is_dropped_when_sources_change(tmp_path, monkeypatch):
    root = str(tmp_path)
    _fake_tree(root, "__global__ void k() {}\n")
    monkeypatch.setattr(bench, "ROOT", root)
    digest = bench.sources_digest()
    with open(os.path.join(root, "profiles", "dram_traffic_wl.md"), "w") as f:
        f.write("# summary\n\n```json\n"
                '{"sources_sha1": "%s", "stages": {"bwd": {"dram_bytes_per_call": 12345}}}\n'
                "```\n" % digest)
    assert bench.committed_traffic("wl", "bwd") == 12345
    assert bench.committed_traffic("wl", "fwd") is None
    assert bench.committed_traffic("other", "bwd") is None
    with open(os.path.join(root, "hierarchical_top_sparse_llsa_b200", "csrc", "k.cu"), "a") as f:
        f.write("// changed\n")
    assert bench.committed_traffic("wl", "bwd") is None


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch
    import torch.distributed as dist

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        # rank r is slow on the first timing and fast on the second
        got = bench.max_over_ranks(torch, dist, [1.0 + rank, 10.0 - rank], "cpu")
        out[rank] = got
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(100)
        assert all(p.exitcode == 0 for p in procs)
        assert out[0] == [2.0, 10.0] and out[1] == [2.0, 10.0]


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_under_two_ranks(rank):
    # launched as one of two ranks: rank 0 alone times the oracle and prints
    # the line; the other rank exits 0 without work
    import json
    import subprocess
    import sys

    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    out = subprocess.run([sys.executable, os.path.join(os.path.dirname(bench.__file__), "bench.py"),
                          "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
                          "--workload", "tiny_32x32_f32"], env=env, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    if rank == 0:
        rec = json.loads(lines[-1])
        assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
        assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
    else:
        assert lines == []
