"""Python binding of libkin.so: block top-k sparse decode attention on B200.

Argument marshalling only.  Every function has the name of the C entry point
it wraps (see include/kin.h for the exact semantics, layouts and errors),
takes CUDA tensors, passes their device pointers and the current CUDA stream,
and raises KinError when the library returns a non-OK status.  All
arithmetic runs in the library's CUDA kernels; there is no fallback: if
libkin.so is missing or cannot be loaded, the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkin.so")

KIN_OK = 0
STATUS_NAMES = {
    0: "KIN_OK", 1: "KIN_ERR_INVALID_ARG", 2: "KIN_ERR_WORKSPACE", 3: "KIN_ERR_CAPACITY",
    4: "KIN_ERR_CUDA", 5: "KIN_ERR_DEVICE_DATA", 6: "KIN_ERR_TIMEOUT",
}
EXPORTED = (
    "kin_status_string", "kin_workspace_bytes", "kin_block_means_build",
    "kin_block_means_update", "kin_block_topk_select", "kin_sparse_decode_attn",
    "kin_block_topk_select_noalloc", "kin_block_means_build_paged", "kin_block_means_update_paged",
    "kin_sparse_decode_attn_paged", "kin_block_means_build_ex", "kin_block_means_update_ex",
    "kin_block_topk_select_ex", "kin_token_topk_workspace_bytes", "kin_token_topk_decode_attn",
    "kin_block_topk_select_paged", "kin_dual_means_bytes", "kin_dual_page_means_bytes",
)
KIN_MEANS_F32, KIN_MEANS_BF16, KIN_MEANS_DUAL = 0, 1, 2
KIN_MEANS_PER_PAGE = 0x100
NOALLOC_SCRATCH_FLOATS = 1 << 21  # KIN_NOALLOC_SCRATCH_FLOATS in include/kin.h


class KinError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


class kin_dims(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("block_size", ctypes.c_int32),
        ("max_seq_len", ctypes.c_int32),
    ]

    def __repr__(self):
        return "kin_dims(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


def make_dims(batch, num_kv_heads, num_q_heads, head_dim, block_size, max_seq_len) -> kin_dims:
    return kin_dims(batch, num_kv_heads, num_q_heads, head_dim, block_size, max_seq_len)


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libkin.so (once) and declare the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"libkin.so not found at {path}: build it with "
            "`python -m block_top_sparse_kin_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(path)
    vp, i32, sz, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_float
    dp = ctypes.POINTER(kin_dims)
    lib.kin_status_string.argtypes = [ctypes.c_int]
    lib.kin_status_string.restype = ctypes.c_char_p
    lib.kin_workspace_bytes.argtypes = [dp, i32]
    lib.kin_workspace_bytes.restype = sz
    lib.kin_block_means_build.argtypes = [dp, vp, vp, vp, vp, vp]
    lib.kin_block_means_build.restype = ctypes.c_int
    lib.kin_block_means_update.argtypes = [dp, vp, vp, vp, vp, vp, vp, i32, vp, vp]
    lib.kin_block_means_update.restype = ctypes.c_int
    lib.kin_block_topk_select.argtypes = [dp, vp, vp, vp, i32, vp, vp, vp, sz, vp, vp]
    lib.kin_block_topk_select.restype = ctypes.c_int
    lib.kin_sparse_decode_attn.argtypes = [dp, vp, vp, vp, vp, vp, vp, i32, f32, vp, vp, vp, sz,
                                           vp, vp]
    lib.kin_sparse_decode_attn.restype = ctypes.c_int
    lib.kin_block_topk_select_noalloc.argtypes = [dp, vp, vp, vp, i32, vp, vp, vp, vp]
    lib.kin_block_topk_select_noalloc.restype = ctypes.c_int
    lib.kin_block_means_build_paged.argtypes = [dp, vp, i32, vp, vp, vp, vp, vp]
    lib.kin_block_means_build_paged.restype = ctypes.c_int
    lib.kin_block_means_update_paged.argtypes = [dp, vp, vp, i32, vp, vp, vp, vp, vp, i32, vp, vp]
    lib.kin_block_means_update_paged.restype = ctypes.c_int
    lib.kin_sparse_decode_attn_paged.argtypes = [dp, vp, vp, vp, i32, vp, vp, vp, vp, i32, f32, vp, vp, vp,
                                                 sz, vp, vp]
    lib.kin_sparse_decode_attn_paged.restype = ctypes.c_int
    lib.kin_block_means_build_ex.argtypes = [dp, vp, i32, vp, vp, vp, i32, vp, vp]
    lib.kin_block_means_build_ex.restype = ctypes.c_int
    lib.kin_block_means_update_ex.argtypes = [dp, vp, vp, i32, vp, vp, i32, vp, vp, vp, i32, vp, vp]
    lib.kin_block_means_update_ex.restype = ctypes.c_int
    lib.kin_block_topk_select_ex.argtypes = [dp, vp, vp, i32, vp, i32, vp, vp, vp, sz, vp, vp]
    lib.kin_block_topk_select_ex.restype = ctypes.c_int
    lib.kin_token_topk_workspace_bytes.argtypes = [dp, i32]
    lib.kin_token_topk_workspace_bytes.restype = sz
    lib.kin_token_topk_decode_attn.argtypes = [dp, vp, vp, vp, vp, i32, f32, vp, vp, vp, vp, sz, vp, vp]
    lib.kin_token_topk_decode_attn.restype = ctypes.c_int
    lib.kin_block_topk_select_paged.argtypes = [dp, vp, vp, i32, i32, vp, vp, i32, vp, vp, vp, sz, vp, vp]
    lib.kin_block_topk_select_paged.restype = ctypes.c_int
    lib.kin_dual_means_bytes.argtypes = [dp]
    lib.kin_dual_means_bytes.restype = sz
    lib.kin_dual_page_means_bytes.argtypes = [dp, i32]
    lib.kin_dual_page_means_bytes.restype = sz
    _lib = lib
    return lib


def _dev(t: Optional[torch.Tensor], name: str, dtype=None, nullable=False, count: Optional[int] = None):
    """The device pointer of t after checking that it is a contiguous CUDA
    tensor on the current device, of an accepted dtype and, when count is
    given, of at least count elements (what the library reads or writes
    through it): a short tensor is refused here, on the host, because the C
    ABI receives bare pointers and could not see it."""
    if t is None:
        if nullable:
            return None
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name} is on {t.device}; the calls run on the current device "
                         f"cuda:{torch.cuda.current_device()}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if count is not None and t.numel() < count:
        raise ValueError(f"{name} holds {t.numel()} elements; the dims need {count}")
    return ctypes.c_void_p(t.data_ptr())


class _Counts:
    """Element counts of every buffer a call touches, from the dims (all
    None when the dims are invalid: the call then returns the library's
    own status for them)."""

    def __init__(self, dims: kin_dims):
        ok = load_library().kin_workspace_bytes(ctypes.byref(dims), 2) > 0
        B, Hkv, Hq, D = dims.batch, dims.num_kv_heads, dims.num_q_heads, dims.head_dim
        bs, L = dims.block_size, dims.max_seq_len
        nbcap = -(-L // bs) if ok else 0
        self.ok = ok
        self.q = B * Hq * D if ok else None            # q, out
        self.lse = B * Hq if ok else None
        self.cache = B * Hkv * L * D if ok else None   # k_cache, v_cache
        self.means = B * Hkv * nbcap * D if ok else None
        self.table = B * nbcap if ok else None
        self.lens = B if ok else None
        self.pairs = B * Hkv if ok else None           # sel_cnt
        self.page = Hkv * bs * D if ok else None       # one page of a pool
        self.page_mean = Hkv * D if ok else None       # one per-page mean
        self.bkd = B * Hkv * D if ok else None         # one appended row per (b, h)

    def times(self, n, per):
        return None if per is None else int(n) * per


def _status(dev_status):
    return _dev(dev_status, "dev_status", torch.int32, nullable=True, count=1)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(rc: int, where: str):
    if rc != KIN_OK:
        raise KinError(rc, where)


_BF16 = (torch.bfloat16, torch.uint16, torch.int16)


def kin_status_string(status: int) -> str:
    return load_library().kin_status_string(status).decode()


def kin_workspace_bytes(dims: kin_dims, k_blocks: int) -> int:
    return int(load_library().kin_workspace_bytes(ctypes.byref(dims), k_blocks))


def alloc_workspace(dims: kin_dims, k_blocks: int, device="cuda") -> torch.Tensor:
    """A zero-filled workspace tensor of kin_workspace_bytes (torch allocations are 256-B aligned)."""
    n = kin_workspace_bytes(dims, k_blocks)
    if n == 0:
        raise KinError(1, "kin_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def kin_block_means_build(dims, k_cache, seq_lens, block_means, dev_status=None, stream=None):
    c = _Counts(dims)
    rc = load_library().kin_block_means_build(
        ctypes.byref(dims), _dev(k_cache, "k_cache", _BF16, count=c.cache),
        _dev(seq_lens, "seq_lens", torch.int32, count=c.lens),
        _dev(block_means, "block_means", torch.float32, count=c.means), _status(dev_status), _stream(stream))
    _check(rc, "kin_block_means_build")


def kin_block_means_update(dims, k_cache, v_cache, block_means, seq_lens, k_new, v_new, n_new,
                           dev_status=None, stream=None):
    c = _Counts(dims)
    new_rows = c.times(max(int(n_new), 0), c.bkd)
    rc = load_library().kin_block_means_update(
        ctypes.byref(dims), _dev(k_cache, "k_cache", _BF16, count=c.cache),
        _dev(v_cache, "v_cache", _BF16, count=c.cache), _dev(block_means, "block_means", torch.float32, count=c.means),
        _dev(seq_lens, "seq_lens", torch.int32, count=c.lens), _dev(k_new, "k_new", _BF16, count=new_rows),
        _dev(v_new, "v_new", _BF16, count=new_rows), int(n_new), _status(dev_status), _stream(stream))
    _check(rc, "kin_block_means_update")


def kin_block_topk_select(dims, q, block_means, seq_lens, k_blocks, sel_idx, sel_cnt, workspace,
                          dev_status=None, stream=None):
    c = _Counts(dims)
    rc = load_library().kin_block_topk_select(
        ctypes.byref(dims), _dev(q, "q", _BF16, count=c.q), _dev(block_means, "block_means", torch.float32, count=c.means),
        _dev(seq_lens, "seq_lens", torch.int32, count=c.lens), int(k_blocks),
        _dev(sel_idx, "sel_idx", torch.int32, count=c.times(max(int(k_blocks), 0), c.pairs)),
        _dev(sel_cnt, "sel_cnt", torch.int32, count=c.pairs), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _status(dev_status), _stream(stream))
    _check(rc, "kin_block_topk_select")


def kin_sparse_decode_attn(dims, q, k_cache, v_cache, seq_lens, sel_idx, sel_cnt, k_blocks,
                           softmax_scale, out, lse, workspace, dev_status=None, stream=None):
    c = _Counts(dims)
    rc = load_library().kin_sparse_decode_attn(
        ctypes.byref(dims), _dev(q, "q", _BF16, count=c.q), _dev(k_cache, "k_cache", _BF16, count=c.cache),
        _dev(v_cache, "v_cache", _BF16, count=c.cache), _dev(seq_lens, "seq_lens", torch.int32, count=c.lens),
        _dev(sel_idx, "sel_idx", torch.int32, count=c.times(max(int(k_blocks), 0), c.pairs)),
        _dev(sel_cnt, "sel_cnt", torch.int32, count=c.pairs), int(k_blocks), float(softmax_scale),
        _dev(out, "out", _BF16, count=c.q), _dev(lse, "lse", torch.float32, nullable=True, count=c.lse),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), _status(dev_status),
        _stream(stream))
    _check(rc, "kin_sparse_decode_attn")


def kin_block_topk_select_noalloc(dims, q, block_means, seq_lens, k_blocks, sel_idx, sel_cnt,
                                  dev_status=None, stream=None):
    """kin_block_topk_select without a workspace, for callers that may not
    allocate device memory: the scratch lives in a fixed array inside
    libkin.so (see include/kin.h for its limit and its sharing rules)."""
    c = _Counts(dims)
    rc = load_library().kin_block_topk_select_noalloc(
        ctypes.byref(dims), _dev(q, "q", _BF16, count=c.q), _dev(block_means, "block_means", torch.float32, count=c.means),
        _dev(seq_lens, "seq_lens", torch.int32, count=c.lens), int(k_blocks),
        _dev(sel_idx, "sel_idx", torch.int32, count=c.times(max(int(k_blocks), 0), c.pairs)),
        _dev(sel_cnt, "sel_cnt", torch.int32, count=c.pairs), _status(dev_status), _stream(stream))
    _check(rc, "kin_block_topk_select_noalloc")


# ---------------------------------------------------------------- paged KV
# k_pages / v_pages [num_pages, Hkv, bs, D] bf16; block_table [B, ceil(Lcap / bs)]
# int32 (page of each logical block).  See include/kin.h.

def kin_block_means_build_paged(dims, k_pages, block_table, seq_lens, block_means, dev_status=None,
                                stream=None):
    c = _Counts(dims)
    pages = int(k_pages.shape[0])
    rc = load_library().kin_block_means_build_paged(
        ctypes.byref(dims), _dev(k_pages, "k_pages", _BF16, count=c.times(pages, c.page)), pages,
        _dev(block_table, "block_table", torch.int32, count=c.table),
        _dev(seq_lens, "seq_lens", torch.int32, count=c.lens),
        _dev(block_means, "block_means", torch.float32, count=c.means), _status(dev_status), _stream(stream))
    _check(rc, "kin_block_means_build_paged")


def kin_block_means_update_paged(dims, k_pages, v_pages, block_table, block_means, seq_lens, k_new, v_new,
                                 n_new, dev_status=None, stream=None):
    c = _Counts(dims)
    pages = int(k_pages.shape[0])
    new_rows = c.times(max(int(n_new), 0), c.bkd)
    rc = load_library().kin_block_means_update_paged(
        ctypes.byref(dims), _dev(k_pages, "k_pages", _BF16, count=c.times(pages, c.page)),
        _dev(v_pages, "v_pages", _BF16, count=c.times(pages, c.page)), pages,
        _dev(block_table, "block_table", torch.int32, count=c.table),
        _dev(block_means, "block_means", torch.float32, count=c.means),
        _dev(seq_lens, "seq_lens", torch.int32, count=c.lens), _dev(k_new, "k_new", _BF16, count=new_rows),
        _dev(v_new, "v_new", _BF16, count=new_rows), int(n_new), _status(dev_status), _stream(stream))
    _check(rc, "kin_block_means_update_paged")


def kin_sparse_decode_attn_paged(dims, q, k_pages, v_pages, block_table, seq_lens, sel_idx, sel_cnt, k_blocks,
                                 softmax_scale, out, lse, workspace, dev_status=None, stream=None):
    c = _Counts(dims)
    pages = int(k_pages.shape[0])
    rc = load_library().kin_sparse_decode_attn_paged(
        ctypes.byref(dims), _dev(q, "q", _BF16, count=c.q), _dev(k_pages, "k_pages", _BF16, count=c.times(pages, c.page)),
        _dev(v_pages, "v_pages", _BF16, count=c.times(pages, c.page)), pages,
        _dev(block_table, "block_table", torch.int32, count=c.table),
        _dev(seq_lens, "seq_lens", torch.int32, count=c.lens),
        _dev(sel_idx, "sel_idx", torch.int32, count=c.times(max(int(k_blocks), 0), c.pairs)),
        _dev(sel_cnt, "sel_cnt", torch.int32, count=c.pairs), int(k_blocks), float(softmax_scale),
        _dev(out, "out", _BF16, count=c.q), _dev(lse, "lse", torch.float32, nullable=True, count=c.lse),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), _status(dev_status),
        _stream(stream))
    _check(rc, "kin_sparse_decode_attn_paged")


# ------------------------------------------------ extended: bf16 block means
# The means dtype follows the block_means tensor (float32 or bfloat16);
# block_table None selects the contiguous cache.  See include/kin.h.

def _means(block_means, count=None, name="block_means", dims=None, pages=None):
    """The means pointer and its dtype code, from the tensor: float32 rows,
    bfloat16 rows, or a uint8 buffer of dual means (fp32 rows, their bf16
    rounding and the rows' error radii: see kin_dual_means_bytes; per page
    when `pages` is given, see kin_dual_page_means_bytes)."""
    if block_means is not None and block_means.dtype == torch.float32:
        return _dev(block_means, name, torch.float32, count=count), KIN_MEANS_F32
    if block_means is not None and block_means.dtype == torch.uint8:
        if dims is None:
            nbytes = None
        elif pages is not None:
            nbytes = kin_dual_page_means_bytes(dims, pages)
        else:
            nbytes = kin_dual_means_bytes(dims)
        return _dev(block_means, name, torch.uint8, count=nbytes or None), KIN_MEANS_DUAL
    return _dev(block_means, name, torch.bfloat16, count=count), KIN_MEANS_BF16


def kin_dual_means_bytes(dims: kin_dims) -> int:
    """Bytes of a dual block-means buffer (KIN_MEANS_DUAL) for these dims."""
    return int(load_library().kin_dual_means_bytes(ctypes.byref(dims)))


def kin_dual_page_means_bytes(dims: kin_dims, num_pages: int) -> int:
    """Bytes of a dual block-means buffer stored per page (KIN_MEANS_DUAL |
    KIN_MEANS_PER_PAGE) for a pool of num_pages pages."""
    return int(load_library().kin_dual_page_means_bytes(ctypes.byref(dims), int(num_pages)))


def alloc_dual_page_means(dims: kin_dims, num_pages: int, device="cuda") -> torch.Tensor:
    """A dual block-means buffer per page (uint8), filled by the build/update
    calls with per_page=True and read by kin_block_topk_select_paged."""
    n = kin_dual_page_means_bytes(dims, num_pages)
    if n == 0:
        raise KinError(1, "kin_dual_page_means_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def alloc_dual_means(dims: kin_dims, device="cuda") -> torch.Tensor:
    """A dual block-means buffer (uint8, 256-byte aligned as torch allocates),
    filled by kin_block_means_build_ex / _update_ex and read by
    kin_block_topk_select_ex."""
    n = kin_dual_means_bytes(dims)
    if n == 0:
        raise KinError(1, "kin_dual_means_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def _layout(rows, block_table, c: _Counts):
    """(num_pages, table pointer, rows per K/V tensor): the contiguous cache
    without a table, else the page pool it indexes."""
    if block_table is None:
        return 0, None, c.cache
    pages = int(rows.shape[0])
    return pages, _dev(block_table, "block_table", torch.int32, count=c.table), c.times(pages, c.page)


def kin_block_means_build_ex(dims, k_rows, seq_lens, block_means, block_table=None, dev_status=None,
                             stream=None, per_page=False):
    """per_page: block_means is [num_pages, Hkv, D] (one mean per page; needs block_table)."""
    c = _Counts(dims)
    pages, table, rows = _layout(k_rows, block_table, c)
    means, dtype = _means(block_means, c.times(pages, c.page_mean) if per_page else c.means, dims=dims,
                          pages=pages if per_page else None)
    dtype |= KIN_MEANS_PER_PAGE if per_page else 0
    rc = load_library().kin_block_means_build_ex(
        ctypes.byref(dims), _dev(k_rows, "k_rows", _BF16, count=rows), pages, table,
        _dev(seq_lens, "seq_lens", torch.int32, count=c.lens), means, dtype, _status(dev_status), _stream(stream))
    _check(rc, "kin_block_means_build_ex")


def kin_block_means_update_ex(dims, k_rows, v_rows, block_means, seq_lens, k_new, v_new, n_new,
                              block_table=None, dev_status=None, stream=None, per_page=False):
    c = _Counts(dims)
    pages, table, rows = _layout(k_rows, block_table, c)
    means, dtype = _means(block_means, c.times(pages, c.page_mean) if per_page else c.means, dims=dims,
                          pages=pages if per_page else None)
    dtype |= KIN_MEANS_PER_PAGE if per_page else 0
    new_rows = c.times(max(int(n_new), 0), c.bkd)
    rc = load_library().kin_block_means_update_ex(
        ctypes.byref(dims), _dev(k_rows, "k_rows", _BF16, count=rows), _dev(v_rows, "v_rows", _BF16, count=rows),
        pages, table, means, dtype, _dev(seq_lens, "seq_lens", torch.int32, count=c.lens),
        _dev(k_new, "k_new", _BF16, count=new_rows), _dev(v_new, "v_new", _BF16, count=new_rows), int(n_new),
        _status(dev_status), _stream(stream))
    _check(rc, "kin_block_means_update_ex")


def kin_block_topk_select_ex(dims, q, block_means, seq_lens, k_blocks, sel_idx, sel_cnt, workspace,
                             dev_status=None, stream=None):
    c = _Counts(dims)
    means, dtype = _means(block_means, c.means, dims=dims)
    rc = load_library().kin_block_topk_select_ex(
        ctypes.byref(dims), _dev(q, "q", _BF16, count=c.q), means, dtype,
        _dev(seq_lens, "seq_lens", torch.int32, count=c.lens), int(k_blocks),
        _dev(sel_idx, "sel_idx", torch.int32, count=c.times(max(int(k_blocks), 0), c.pairs)),
        _dev(sel_cnt, "sel_cnt", torch.int32, count=c.pairs), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _status(dev_status), _stream(stream))
    _check(rc, "kin_block_topk_select_ex")


# --------------------------------------------------- token-level top-k attention

def kin_token_topk_workspace_bytes(dims: kin_dims, k_tokens: int) -> int:
    return int(load_library().kin_token_topk_workspace_bytes(ctypes.byref(dims), k_tokens))


def alloc_token_workspace(dims: kin_dims, k_tokens: int, device="cuda") -> torch.Tensor:
    n = kin_token_topk_workspace_bytes(dims, k_tokens)
    if n == 0:
        raise KinError(1, "kin_token_topk_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device)


def kin_token_topk_decode_attn(dims, q, k_cache, v_cache, seq_lens, k_tokens, softmax_scale, out, lse, workspace,
                               sel_tokens=None, dev_status=None, stream=None):
    c = _Counts(dims)
    rc = load_library().kin_token_topk_decode_attn(
        ctypes.byref(dims), _dev(q, "q", _BF16, count=c.q), _dev(k_cache, "k_cache", _BF16, count=c.cache),
        _dev(v_cache, "v_cache", _BF16, count=c.cache), _dev(seq_lens, "seq_lens", torch.int32, count=c.lens),
        int(k_tokens), float(softmax_scale), _dev(out, "out", _BF16, count=c.q),
        _dev(lse, "lse", torch.float32, nullable=True, count=c.lse),
        _dev(sel_tokens, "sel_tokens", torch.int32, nullable=True, count=c.times(max(int(k_tokens), 0), c.lse)),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), _status(dev_status),
        _stream(stream))
    _check(rc, "kin_token_topk_decode_attn")


def kin_block_topk_select_paged(dims, q, page_means, block_table, seq_lens, k_blocks, sel_idx, sel_cnt, workspace,
                                dev_status=None, stream=None, num_pages=None):
    """The select over per-page block means [num_pages, Hkv, D] (fp32 or bf16),
    or a per-page dual buffer (uint8; num_pages then required), found through
    block_table: the shared-prompt layout (see include/kin.h)."""
    c = _Counts(dims)
    if page_means is not None and page_means.dtype == torch.uint8:
        if num_pages is None:
            raise ValueError("page_means: a dual buffer needs num_pages")
        pages = int(num_pages)
        means, dtype = _means(page_means, None, "page_means", dims=dims, pages=pages)
    else:
        pages = int(page_means.shape[0])
        means, dtype = _means(page_means, c.times(pages, c.page_mean), "page_means")
    rc = load_library().kin_block_topk_select_paged(
        ctypes.byref(dims), _dev(q, "q", _BF16, count=c.q), means, dtype, pages,
        _dev(block_table, "block_table", torch.int32, count=c.table),
        _dev(seq_lens, "seq_lens", torch.int32, count=c.lens), int(k_blocks),
        _dev(sel_idx, "sel_idx", torch.int32, count=c.times(max(int(k_blocks), 0), c.pairs)),
        _dev(sel_cnt, "sel_cnt", torch.int32, count=c.pairs), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _status(dev_status), _stream(stream))
    _check(rc, "kin_block_topk_select_paged")
