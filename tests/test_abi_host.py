"""CPU-only checks of the C ABI: the library loads, exports every entry point
that include/llsa.h declares, and its host-side argument checks reject bad
calls before any launch (no GPU is touched: no call here reaches a kernel)."""

import ctypes
import os
import re

import pytest

import hierarchical_top_sparse_llsa_b200 as llsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"LLSA_API\s+[\w\s\*]*?\b(llsa_\w+)\s*\(", text))
    return names


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(llsa.LIB_PATH):
        from hierarchical_top_sparse_llsa_b200 import build
        build.build()
    return llsa.lib()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert names == set(llsa.EXPORTED), names
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_status_strings(lib):
    assert llsa.version() == llsa.ABI_VERSION == 200
    assert llsa.status_string(llsa.OK) == "ok"
    assert "workspace" in llsa.status_string(llsa.ERR_WORKSPACE)


def _desc(**kw):
    base = dict(B=1, H=2, N=4096, D=64, L=3, topk=8, dtype=llsa.BF16)
    base.update(kw)
    return llsa.make_desc(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(D=96), llsa.ERR_UNSUPPORTED),
    (dict(topk=33), llsa.ERR_UNSUPPORTED),
    (dict(L=7, N=16**7), llsa.ERR_UNSUPPORTED),
    (dict(N=4096 + 16), llsa.ERR_INVALID_ARG),  # not a multiple of 16^L
    (dict(topk=0), llsa.ERR_INVALID_ARG),
    (dict(dtype=5), llsa.ERR_INVALID_ARG),
    (dict(B=0), llsa.ERR_INVALID_ARG),
    (dict(flags=8), llsa.ERR_INVALID_ARG),  # an unknown flag bit
    (dict(flags=llsa.FLAG_FWD_TCGEN05 | llsa.FLAG_FWD_MMA_SYNC), llsa.ERR_INVALID_ARG),  # two forwards
])
def test_bad_descriptors_are_rejected_before_launch(lib, kw, status):
    d = _desc(**kw)
    pyr, ind, csr = llsa.LlsaPyramid(), llsa.LlsaIndices(), llsa.LlsaCsr()
    fake = 256  # never dereferenced: the check fails first
    assert llsa.llsa_pool(d, fake, fake, fake, pyr, check=False) == status
    assert llsa.llsa_select(d, pyr, ind, check=False) == status
    assert llsa.llsa_index_transpose(d, ind, csr, 256, 1 << 40, check=False) == status
    assert llsa.llsa_transpose_workspace_bytes(d) == 0
    assert llsa.llsa_bwd_workspace_bytes(d) == 0


def test_null_buffers_are_rejected(lib):
    d = _desc()
    pyr, ind, csr = llsa.LlsaPyramid(), llsa.LlsaIndices(), llsa.LlsaCsr()
    assert llsa.llsa_pool(d, None, None, None, pyr, check=False) == llsa.ERR_INVALID_ARG
    assert llsa.llsa_pool(d, 256, 256, 256, pyr, check=False) == llsa.ERR_INVALID_ARG
    assert llsa.llsa_select(d, pyr, ind, check=False) == llsa.ERR_INVALID_ARG
    assert llsa.llsa_attn_fwd(d, 256, 256, 256, pyr, ind, 256, 256, check=False) == llsa.ERR_INVALID_ARG
    assert llsa.llsa_index_transpose(d, ind, csr, 256, 1 << 40, check=False) == llsa.ERR_INVALID_ARG
    assert llsa.llsa_select_attn_fwd(d, 256, 256, 256, pyr, ind, 256, 256, check=False) == llsa.ERR_INVALID_ARG
    with pytest.raises(llsa.LlsaError):
        llsa.llsa_select(d, pyr, ind)


def test_select_attn_fwd_checks_both_halves_before_launch(lib):
    d = _desc()
    pyr, ind = llsa.LlsaPyramid(), llsa.LlsaIndices()
    for l in range(1, 4):
        pyr.q[l] = pyr.k[l] = ind.idx[l] = 256
        if l >= 2:
            pyr.v[l] = 256
    # the selection needs Q(1): missing, it is an argument error
    pyr.q[1] = 0
    assert llsa.llsa_select_attn_fwd(d, 256, 256, 256, pyr, ind, 256, 256, check=False) == llsa.ERR_INVALID_ARG
    pyr.q[1] = 256
    # the forward needs V(2): missing, it is an argument error
    pyr.v[2] = 0
    assert llsa.llsa_select_attn_fwd(d, 256, 256, 256, pyr, ind, 256, 256, check=False) == llsa.ERR_INVALID_ARG
    pyr.v[2] = 256
    # bf16 output not 16-byte aligned
    assert llsa.llsa_select_attn_fwd(d, 256, 256, 256, pyr, ind, 264, 256, check=False) == llsa.ERR_INVALID_ARG
    # I(3) is needed by the selection even when the depth leaves level 3 out
    d.enrich_levels = 1
    ind.idx[3] = 0
    assert llsa.llsa_select_attn_fwd(d, 256, 256, 256, pyr, ind, 264, 256, check=False) == llsa.ERR_INVALID_ARG


def test_workspace_size_and_checks(lib):
    d = _desc()
    B, H, N, D, L, K = 1, 2, 4096, 64, 3, 8
    r256 = lambda x: (x + 255) // 256 * 256
    want = r256(B * H * N * 4)
    want += sum(r256(B * H * (N // 128) * K * 2 * D * 4) for _ in range(2, L + 1))
    want += sum(r256(B * H * (N // 16**l) * 2 * D * 4) for l in range(2, L + 1))
    want += 256  # the key-major pass's work counter
    assert llsa.llsa_bwd_workspace_bytes(d) == want
    # fill every pointer with a fake non-null value: the size check fails first
    pyr, ind, csr = llsa.LlsaPyramid(), llsa.LlsaIndices(), llsa.LlsaCsr()
    for l in range(1, L + 1):
        pyr.q[l] = pyr.k[l] = pyr.v[l] = ind.idx[l] = csr.row_ptr[l] = csr.col[l] = 256
    st = llsa.llsa_attn_bwd(d, 256, 256, 256, pyr, 256, 256, 256, ind, csr, 256, 256, 256,
                            256, want - 1, check=False)
    assert st == llsa.ERR_WORKSPACE
    st = llsa.llsa_attn_bwd(d, 256, 256, 256, pyr, 256, 256, 256, ind, csr, 256, 256, 256,
                            260, want, check=False)
    assert st == llsa.ERR_INVALID_ARG  # workspace not 256-byte aligned


def _transpose_ws_bytes(B, H, N, L):
    # per level: nchunk row chunks (128 rows each, at most 128 chunks), one
    # int32 count per (b, h, chunk, key), each level 256-byte aligned
    total = 0
    for l in range(1, L + 1):
        n = N // 16**l
        c = min(128, max(1, (n + 127) // 128))
        rows = (n + c - 1) // c
        c = (n + rows - 1) // rows
        total += (B * H * c * n * 4 + 255) // 256 * 256
    return total


@pytest.mark.parametrize("shape", [(1, 2, 4096, 3), (2, 3, 1024, 2), (1, 1, 65536, 4), (1, 2, 256, 2)])
def test_transpose_workspace_size_and_checks(lib, shape):
    B, H, N, L = shape
    d = _desc(B=B, H=H, N=N, L=L)
    want = _transpose_ws_bytes(B, H, N, L)
    assert llsa.llsa_transpose_workspace_bytes(d) == want
    ind, csr = llsa.LlsaIndices(), llsa.LlsaCsr()
    for l in range(1, L + 1):
        ind.idx[l] = csr.row_ptr[l] = csr.col[l] = 256
    assert llsa.llsa_index_transpose(d, ind, csr, 256, want - 1, check=False) == llsa.ERR_WORKSPACE
    assert llsa.llsa_index_transpose(d, ind, csr, 260, want, check=False) == llsa.ERR_INVALID_ARG
    assert llsa.llsa_index_transpose(d, ind, csr, None, want, check=False) == llsa.ERR_INVALID_ARG


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(llsa, "LIB_PATH", str(tmp_path / "nope.so"))
    monkeypatch.setattr(llsa, "_lib", None)
    with pytest.raises(llsa.LlsaError):
        llsa.lib()


@pytest.mark.parametrize("args,status", [
    (dict(img_h=8, img_w=16), llsa.ERR_UNSUPPORTED),   # not square
    (dict(img_h=12, img_w=12), llsa.ERR_UNSUPPORTED),  # not a power of two
    (dict(img_h=2, img_w=2), llsa.ERR_UNSUPPORTED),    # smaller than a 4x4 tile
    (dict(D=96), llsa.ERR_UNSUPPORTED),
    (dict(dtype=7), llsa.ERR_INVALID_ARG),
    (dict(B=0), llsa.ERR_INVALID_ARG),
    (dict(src=None), llsa.ERR_INVALID_ARG),
    (dict(src=1 << 20, dst=(1 << 20) + 1024), llsa.ERR_INVALID_ARG),  # overlapping
    (dict(src=(1 << 20) + 8), llsa.ERR_INVALID_ARG),                  # not 16-byte aligned
])
def test_reorder_argument_checks(lib, args, status):
    a = dict(B=1, H=2, img_h=16, img_w=16, D=64, dtype=llsa.BF16, src=1 << 20, dst=1 << 30)
    a.update(args)
    assert llsa.llsa_reorder(a["B"], a["H"], a["img_h"], a["img_w"], a["D"], a["dtype"], a["src"], a["dst"],
                             True, check=False) == status


@pytest.mark.parametrize("enrich,top", [(0, 3), (1, 2), (2, 3), (5, 3), (-1, 1), (-4, 1)])
def test_enrichment_depth_sizes_and_required_levels(lib, enrich, top):
    # the attention-side workspaces cover levels 1..Lc only, Lc = min(L, 1 + depth)
    B, H, N, D, L, K = 1, 2, 4096, 64, 3, 8
    d = _desc(B=B, H=H, N=N, L=L)
    d.enrich_levels = enrich
    r256 = lambda x: (x + 255) // 256 * 256
    want = r256(B * H * N * 4)
    want += sum(r256(B * H * (N // 128) * K * 2 * D * 4) for _ in range(2, top + 1))
    want += sum(r256(B * H * (N // 16**l) * 2 * D * 4) for l in range(2, top + 1))
    want += 256
    assert llsa.llsa_bwd_workspace_bytes(d) == want
    assert llsa.llsa_transpose_workspace_bytes(d) == _transpose_ws_bytes(B, H, N, top)
    # entries above Lc may be NULL: the workspace size check is what fails
    ind, csr = llsa.LlsaIndices(), llsa.LlsaCsr()
    for l in range(1, top + 1):
        ind.idx[l] = csr.row_ptr[l] = csr.col[l] = 256
    tw = llsa.llsa_transpose_workspace_bytes(d)
    assert llsa.llsa_index_transpose(d, ind, csr, 256, tw - 1, check=False) == llsa.ERR_WORKSPACE
    ind.idx[top] = 0  # a missing entry at or below Lc is an argument error
    assert llsa.llsa_index_transpose(d, ind, csr, 256, tw, check=False) == llsa.ERR_INVALID_ARG


def test_topk_per_level_sizes_and_checks(lib):
    B, H, N, D, L = 1, 2, 4096, 64, 3
    kl = {1: 12, 2: 4, 3: 2}
    d = llsa.make_desc(B, H, N, D, L, 8, llsa.BF16, topk_l=[0, 12, 4, 2])
    r256 = lambda x: (x + 255) // 256 * 256
    want = r256(B * H * N * 4)
    want += sum(r256(B * H * (N // 128) * kl[l] * 2 * D * 4) for l in range(2, L + 1))
    want += sum(r256(B * H * (N // 16**l) * 2 * D * 4) for l in range(2, L + 1))
    want += 256
    assert llsa.llsa_bwd_workspace_bytes(d) == want
    assert llsa.level_topk(d, 1) == 12 and llsa.level_topk(d, 3) == 2
    d0 = llsa.make_desc(B, H, N, D, L, 8, llsa.BF16, topk_l=[0, 0, 5, 0])
    assert [llsa.level_topk(d0, l) for l in (1, 2, 3)] == [8, 5, 8]
    bad = llsa.make_desc(B, H, N, D, L, 8, llsa.BF16, topk_l=[0, 33, 0, 0])
    assert llsa.llsa_bwd_workspace_bytes(bad) == 0
    bad = llsa.make_desc(B, H, N, D, L, 8, llsa.BF16, topk_l=[0, 0, -1, 0])
    assert llsa.llsa_bwd_workspace_bytes(bad) == 0
    pyr, ind = llsa.LlsaPyramid(), llsa.LlsaIndices()
    assert llsa.llsa_select(bad, pyr, ind, check=False) == llsa.ERR_INVALID_ARG
    bad.topk_l[2] = 40
    assert llsa.llsa_select(bad, pyr, ind, check=False) == llsa.ERR_UNSUPPORTED


def test_residual_calls_check_arguments(lib):
    d = _desc()
    pyr, ind, csr = llsa.LlsaPyramid(), llsa.LlsaIndices(), llsa.LlsaCsr()
    for l in range(1, 4):
        pyr.q[l] = pyr.k[l] = ind.idx[l] = csr.row_ptr[l] = csr.col[l] = 256
        if l >= 2:
            pyr.v[l] = 256
    # bf16 without a residual buffer, or a misaligned one
    assert llsa.llsa_attn_bwd_res(d, 256, 256, 256, pyr, 256, None, 256, 256, ind, csr, 256, 256, 256,
                                  256, 1 << 40, check=False) == llsa.ERR_INVALID_ARG
    assert llsa.llsa_attn_fwd_res(d, 256, 256, 256, pyr, ind, 256, None, 256, check=False) == llsa.ERR_INVALID_ARG
    assert llsa.llsa_attn_fwd_res(d, 256, 256, 256, pyr, ind, 264, 256, 256, check=False) == llsa.ERR_INVALID_ARG
    ws = llsa.llsa_bwd_workspace_bytes(d)
    assert llsa.llsa_attn_bwd_res(d, 256, 256, 256, pyr, 256, 264, 256, 256, ind, csr, 256, 256, 256,
                                  256, ws - 1, check=False) == llsa.ERR_WORKSPACE


def test_wait_timeout_selftest_checks_arguments(lib):
    # host checks come before any launch: nothing reaches a device here
    assert llsa.llsa_selftest_wait_timeout(None, 10, check=False) == llsa.ERR_INVALID_ARG
    assert llsa.llsa_selftest_wait_timeout(256, 0, check=False) == llsa.ERR_INVALID_ARG
    assert llsa.llsa_selftest_wait_timeout(256, 2000001, check=False) == llsa.ERR_INVALID_ARG


def test_qkv_pool_checks_arguments(lib):
    # every check below comes before the tensor maps are encoded or anything
    # is launched: nothing reaches a device here
    def pyramid(L):
        pyr = llsa.LlsaPyramid()
        for l in range(1, L + 1):
            pyr.q[l] = pyr.k[l] = 256
            if l >= 2:
                pyr.v[l] = 256
        return pyr

    def call(d, x=256, w=256, C=128, q=256, k=256, v=256, pyr=None):
        return llsa.llsa_qkv_pool(d, x, w, C, q, k, v, pyramid(d.L) if pyr is None else pyr, None, 0,
                                  check=False)

    d = llsa.make_desc(1, 2, 4096, 64, 3, 8, llsa.BF16)
    assert call(d, x=None) == llsa.ERR_INVALID_ARG
    assert call(d, v=None) == llsa.ERR_INVALID_ARG
    assert call(d, C=0) == llsa.ERR_INVALID_ARG
    assert call(d, C=96) == llsa.ERR_INVALID_ARG            # not a multiple of 64
    assert call(d, w=264) == llsa.ERR_INVALID_ARG           # not 16-byte aligned
    assert call(d, pyr=llsa.LlsaPyramid()) == llsa.ERR_INVALID_ARG  # pyramid levels missing
    assert call(llsa.make_desc(1, 2, 4096, 64, 3, 8, llsa.F32)) == llsa.ERR_UNSUPPORTED
    assert call(llsa.make_desc(1, 3, 4096, 64, 3, 8, llsa.BF16)) == llsa.ERR_UNSUPPORTED  # H*D = 192
    assert call(llsa.make_desc(1, 2, 16, 64, 1, 8, llsa.BF16)) == llsa.ERR_UNSUPPORTED    # N = 16 < 256
