"""Python binding of the LLSA C ABI (include/llsa.h) over libllsa.so.

Argument marshalling only: every step of the path runs in the CUDA library.
The functions take the same names and arguments as the C entry points, with
device pointers as Python ints and the stream as a cudaStream_t handle (int).
``LlsaBuffers`` is plumbing for callers that hold torch tensors: it allocates
the pyramid, index, key-major and workspace buffers with torch on a device and
fills the C structs with their pointers.

Importing the package does not load the library; the first call does, and it
raises if ``libllsa.so`` is missing (build it with
``python -m hierarchical_top_sparse_llsa_b200.build``).  There is no fallback.
"""

from __future__ import annotations

import ctypes
import math
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libllsa.so")

MAX_LEVELS = 6
MAX_TOPK = 32
BLOCK = 16
F32, BF16 = 0, 1
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_LAUNCH, ERR_WORKSPACE = 0, 1, 2, 3, 4
DEV_BAD_INDEX, DEV_NONCANONICAL, DEV_TIMEOUT = 1, 2, 4
FLAG_FWD_TCGEN05 = 1
FLAG_BWD_TCGEN05 = 2
FLAG_FWD_MMA_SYNC = 4
NOALLOC_SCRATCH_BYTES = 16 << 20

EXPORTED = (
    "llsa_pool",
    "llsa_qkv_pool",
    "llsa_select",
    "llsa_attn_fwd",
    "llsa_select_attn_fwd",
    "llsa_attn_fwd_res",
    "llsa_attn_bwd_res",
    "llsa_transpose_workspace_bytes",
    "llsa_index_transpose",
    "llsa_bwd_workspace_bytes",
    "llsa_attn_bwd",
    "llsa_attn_bwd_noalloc",
    "llsa_reorder",
    "llsa_selftest_wait_timeout",
    "llsa_status_string",
    "llsa_version",
)


class LlsaDesc(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int), ("D", ctypes.c_int),
        ("L", ctypes.c_int), ("topk", ctypes.c_int), ("dtype", ctypes.c_int), ("flags", ctypes.c_int),
        ("sm_scale", ctypes.c_float), ("level_w", ctypes.c_float * (MAX_LEVELS + 1)),
        ("enrich_levels", ctypes.c_int),
        ("topk_l", ctypes.c_int * (MAX_LEVELS + 1)),
    ]


_PtrArr = ctypes.c_void_p * (MAX_LEVELS + 1)


class LlsaPyramid(ctypes.Structure):
    _fields_ = [("q", _PtrArr), ("k", _PtrArr), ("v", _PtrArr)]


class LlsaIndices(ctypes.Structure):
    _fields_ = [("idx", _PtrArr)]


class LlsaCsr(ctypes.Structure):
    _fields_ = [("row_ptr", _PtrArr), ("col", _PtrArr)]


# llsa_version() of the library whose struct layouts (llsa_desc above) this
# binding mirrors
ABI_VERSION = 200


class LlsaError(RuntimeError):
    """A host status other than LLSA_OK."""


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libllsa.so (loaded on first use; raises if missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise LlsaError(f"{LIB_PATH} is missing: build the CUDA library first "
                            "(python -m hierarchical_top_sparse_llsa_b200.build)")
        L = ctypes.CDLL(LIB_PATH)
        vp, P = ctypes.c_void_p, ctypes.POINTER
        sig = {
            "llsa_pool": (ctypes.c_int, [P(LlsaDesc), vp, vp, vp, P(LlsaPyramid), vp]),
            "llsa_qkv_pool": (ctypes.c_int, [P(LlsaDesc), vp, vp, ctypes.c_int, vp, vp, vp, P(LlsaPyramid), vp, vp]),
            "llsa_select": (ctypes.c_int, [P(LlsaDesc), P(LlsaPyramid), P(LlsaIndices), vp]),
            "llsa_attn_fwd": (ctypes.c_int, [P(LlsaDesc), vp, vp, vp, P(LlsaPyramid), P(LlsaIndices),
                                             vp, vp, vp, vp]),
            "llsa_select_attn_fwd": (ctypes.c_int, [P(LlsaDesc), vp, vp, vp, P(LlsaPyramid), P(LlsaIndices),
                                                    vp, vp, vp, vp]),
            "llsa_transpose_workspace_bytes": (ctypes.c_size_t, [P(LlsaDesc)]),
            "llsa_index_transpose": (ctypes.c_int, [P(LlsaDesc), P(LlsaIndices), P(LlsaCsr), vp,
                                                    ctypes.c_size_t, vp, vp]),
            "llsa_bwd_workspace_bytes": (ctypes.c_size_t, [P(LlsaDesc)]),
            "llsa_attn_bwd": (ctypes.c_int, [P(LlsaDesc), vp, vp, vp, P(LlsaPyramid), vp, vp, vp,
                                             P(LlsaIndices), P(LlsaCsr), vp, vp, vp, vp, ctypes.c_size_t,
                                             vp, vp]),
            "llsa_attn_fwd_res": (ctypes.c_int, [P(LlsaDesc), vp, vp, vp, P(LlsaPyramid), P(LlsaIndices),
                                                 vp, vp, vp, vp, vp]),
            "llsa_attn_bwd_res": (ctypes.c_int, [P(LlsaDesc), vp, vp, vp, P(LlsaPyramid), vp, vp, vp, vp,
                                                 P(LlsaIndices), P(LlsaCsr), vp, vp, vp, vp, ctypes.c_size_t,
                                                 vp, vp]),
            "llsa_attn_bwd_noalloc": (ctypes.c_int, [P(LlsaDesc), vp, vp, vp, P(LlsaPyramid), vp, vp, vp,
                                                     P(LlsaIndices), P(LlsaCsr), vp, vp, vp, vp, vp]),
            "llsa_reorder": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, vp, vp, ctypes.c_int, vp]),
            "llsa_selftest_wait_timeout": (ctypes.c_int, [vp, ctypes.c_uint, vp]),
            "llsa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
            "llsa_version": (ctypes.c_int, []),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        if L.llsa_version() != ABI_VERSION:  # the structs above would not match its layout
            raise LlsaError(f"{LIB_PATH} is version {L.llsa_version()}, this binding expects {ABI_VERSION}: "
                            "rebuild the CUDA library")
        _lib = L
    return _lib


def _check(status: int) -> int:
    if status != OK:
        raise LlsaError(f"LLSA error {status}: {status_string(status)}")
    return status


def make_desc(B, H, N, D, L, topk, dtype, sm_scale=0.0, level_w=None, flags=0,
              enrich_levels=0, topk_l=None) -> LlsaDesc:
    """Fill an llsa_desc; level_w is None (every weight 1) or indexable by level.

    enrich_levels is the enrichment depth: coarse levels 2..min(L, 1 + depth)
    join the keys; 0 means all of them, a negative value none.  topk_l is None
    (topk at every level) or indexable by level: K_l, the keys kept at level l
    (0 selects topk)."""
    d = LlsaDesc()
    d.B, d.H, d.N, d.D, d.L, d.topk = B, H, N, D, L, topk
    d.dtype = dtype
    d.flags = flags
    d.sm_scale = sm_scale
    d.enrich_levels = int(enrich_levels)
    for l in range(MAX_LEVELS + 1):
        d.level_w[l] = 0.0
    if level_w is not None:
        for l in range(2, L + 1):
            d.level_w[l] = float(level_w[l])
    for l in range(MAX_LEVELS + 1):
        d.topk_l[l] = 0
    if topk_l is not None:
        for l in range(1, L + 1):
            d.topk_l[l] = int(topk_l[l])
    return d


def level_topk(desc: LlsaDesc, l: int) -> int:
    """K_l of a descriptor: the width of I(l)."""
    return desc.topk_l[l] if desc.topk_l[l] > 0 else desc.topk


# ------------------------------------------------------------ entry points
def llsa_pool(desc, q, k, v, pyramid, stream=0, check=True):
    st = lib().llsa_pool(ctypes.byref(desc), q, k, v, ctypes.byref(pyramid), stream)
    return _check(st) if check else st


def llsa_qkv_pool(desc, x, w, C, q, k, v, pyramid, dev_status=None, stream=0, check=True):
    st = lib().llsa_qkv_pool(ctypes.byref(desc), x, w, C, q, k, v, ctypes.byref(pyramid), dev_status, stream)
    return _check(st) if check else st


def llsa_select(desc, pyramid, indices, stream=0, check=True):
    st = lib().llsa_select(ctypes.byref(desc), ctypes.byref(pyramid), ctypes.byref(indices), stream)
    return _check(st) if check else st


def llsa_attn_fwd(desc, q, k, v, pyramid, indices, o, lse, dev_status=None, stream=0, check=True):
    st = lib().llsa_attn_fwd(ctypes.byref(desc), q, k, v, ctypes.byref(pyramid), ctypes.byref(indices),
                             o, lse, dev_status, stream)
    return _check(st) if check else st


def llsa_select_attn_fwd(desc, q, k, v, pyramid, indices, o, lse, dev_status=None, stream=0, check=True):
    st = lib().llsa_select_attn_fwd(ctypes.byref(desc), q, k, v, ctypes.byref(pyramid),
                                    ctypes.byref(indices), o, lse, dev_status, stream)
    return _check(st) if check else st


def llsa_transpose_workspace_bytes(desc) -> int:
    return int(lib().llsa_transpose_workspace_bytes(ctypes.byref(desc)))


def llsa_index_transpose(desc, indices, csr, ws, ws_bytes, dev_status=None, stream=0, check=True):
    st = lib().llsa_index_transpose(ctypes.byref(desc), ctypes.byref(indices), ctypes.byref(csr),
                                    ws, ws_bytes, dev_status, stream)
    return _check(st) if check else st


def llsa_bwd_workspace_bytes(desc) -> int:
    return int(lib().llsa_bwd_workspace_bytes(ctypes.byref(desc)))


def llsa_attn_bwd(desc, q, k, v, pyramid, o, lse, dout, indices, csr, dq, dk, dv, ws, ws_bytes,
                  dev_status=None, stream=0, check=True):
    st = lib().llsa_attn_bwd(ctypes.byref(desc), q, k, v, ctypes.byref(pyramid), o, lse, dout,
                             ctypes.byref(indices), ctypes.byref(csr), dq, dk, dv, ws, ws_bytes,
                             dev_status, stream)
    return _check(st) if check else st


def llsa_attn_fwd_res(desc, q, k, v, pyramid, indices, o, o_res, lse, dev_status=None, stream=0, check=True):
    st = lib().llsa_attn_fwd_res(ctypes.byref(desc), q, k, v, ctypes.byref(pyramid), ctypes.byref(indices),
                                 o, o_res, lse, dev_status, stream)
    return _check(st) if check else st


def llsa_attn_bwd_res(desc, q, k, v, pyramid, o, o_res, lse, dout, indices, csr, dq, dk, dv, ws, ws_bytes,
                      dev_status=None, stream=0, check=True):
    st = lib().llsa_attn_bwd_res(ctypes.byref(desc), q, k, v, ctypes.byref(pyramid), o, o_res, lse, dout,
                                 ctypes.byref(indices), ctypes.byref(csr), dq, dk, dv, ws, ws_bytes,
                                 dev_status, stream)
    return _check(st) if check else st


def llsa_attn_bwd_noalloc(desc, q, k, v, pyramid, o, lse, dout, indices, csr, dq, dk, dv,
                          dev_status=None, stream=0, check=True):
    """llsa_attn_bwd without a caller workspace: scratch comes from a fixed
    16 MiB device array inside the library (for callers that cannot
    allocate); problems needing more return ERR_WORKSPACE."""
    st = lib().llsa_attn_bwd_noalloc(ctypes.byref(desc), q, k, v, ctypes.byref(pyramid), o, lse, dout,
                                     ctypes.byref(indices), ctypes.byref(csr), dq, dk, dv, dev_status,
                                     stream)
    return _check(st) if check else st


def llsa_selftest_wait_timeout(dev_status, limit_us, stream=0, check=True):
    """One launch that drives the kernels' bounded mbarrier wait to expiry
    (nothing arrives): LLSA_DEV_TIMEOUT is OR-ed into *dev_status."""
    st = lib().llsa_selftest_wait_timeout(dev_status, limit_us, stream)
    return _check(st) if check else st


def llsa_reorder(B, H, img_h, img_w, D, dtype, src, dst, to_zorder, stream=0, check=True):
    """Raster <-> Z-order permutation of the token axis of [B, H, N, D]."""
    st = lib().llsa_reorder(B, H, img_h, img_w, D, dtype, src, dst, 1 if to_zorder else 0, stream)
    return _check(st) if check else st


def status_string(status: int) -> str:
    return lib().llsa_status_string(status).decode()


def version() -> int:
    return int(lib().llsa_version())


# --------------------------------------------------- torch-held buffers
class LlsaBuffers:
    """Device buffers of one problem, allocated with torch, and the C structs
    that point at them.  Plumbing only: no computation happens here."""

    def __init__(self, desc: LlsaDesc, device, with_bwd: bool = True):
        import torch

        self.desc = desc
        B, H, N, D, L = desc.B, desc.H, desc.N, desc.D, desc.L
        f32, i32 = torch.float32, torch.int32
        self.pq, self.pk, self.pv, self.idx, self.row_ptr, self.col = {}, {}, {}, {}, {}, {}
        self.pyramid = LlsaPyramid()
        self.indices = LlsaIndices()
        self.csr = LlsaCsr()
        for l in range(1, L + 1):
            n = N // BLOCK**l
            self.pq[l] = torch.empty(B, H, n, D, dtype=f32, device=device)
            self.pk[l] = torch.empty(B, H, n, D, dtype=f32, device=device)
            self.pyramid.q[l] = self.pq[l].data_ptr()
            self.pyramid.k[l] = self.pk[l].data_ptr()
            if l >= 2:
                self.pv[l] = torch.empty(B, H, n, D, dtype=f32, device=device)
                self.pyramid.v[l] = self.pv[l].data_ptr()
            Kl = level_topk(desc, l)
            self.idx[l] = torch.empty(B, H, n, Kl, dtype=i32, device=device)
            self.indices.idx[l] = self.idx[l].data_ptr()
            if with_bwd:
                self.row_ptr[l] = torch.empty(B, H, n + 1, dtype=i32, device=device)
                self.col[l] = torch.empty(B, H, n * Kl, dtype=i32, device=device)
                self.csr.row_ptr[l] = self.row_ptr[l].data_ptr()
                self.csr.col[l] = self.col[l].data_ptr()
        self.ws_bytes = llsa_bwd_workspace_bytes(desc) if with_bwd else 0
        self.ws = torch.empty(max(1, self.ws_bytes), dtype=torch.uint8, device=device)
        self.tr_ws_bytes = llsa_transpose_workspace_bytes(desc) if with_bwd else 0
        self.tr_ws = torch.empty(max(1, self.tr_ws_bytes), dtype=torch.uint8, device=device)
        self.status = torch.zeros(1, dtype=i32, device=device)


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)
