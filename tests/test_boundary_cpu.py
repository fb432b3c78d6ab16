"""The C ABI library without a GPU: it loads, exports every entry point that
include/kin.h declares, and its host-side checks reject bad arguments before
any CUDA call is made."""
import ctypes
import os
import re
import subprocess

import pytest

import block_top_sparse_kin_b200 as kin
from block_top_sparse_kin_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kin.h")


@pytest.fixture(scope="module")
def lib():
    srcs = [os.path.join(kbuild.CSRC, s) for s in kbuild.SOURCES] + [HEADER]
    if not os.path.exists(kbuild.LIB) or os.path.getmtime(kbuild.LIB) < max(map(os.path.getmtime, srcs)):
        kbuild.build()
    return kin.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kin_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    assert declared_functions() == sorted(kin.EXPORTED)


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", kbuild.LIB], capture_output=True, text=True,
                         check=True).stdout
    exported = set(l.split()[-1] for l in out.splitlines() if " T " in l)
    for name in declared_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None
    # nothing else of ours leaks out of the library
    assert not [s for s in exported if s.startswith("_ZN3kin")]


def test_status_strings(lib):
    for code, name in kin.STATUS_NAMES.items():
        assert kin.kin_status_string(code) == name
    assert kin.kin_status_string(99) == "KIN_ERR_UNKNOWN"


def dims(B=2, Hkv=2, Hq=8, D=128, bs=16, L=256):
    return kin.make_dims(B, Hkv, Hq, D, bs, L)


def test_workspace_bytes(lib):
    # dual block means: fp32 rows, bf16 rows, one fp32 error radius per row
    d = dims()
    rows = d.batch * d.num_kv_heads * -(-d.max_seq_len // d.block_size)
    assert kin.kin_dual_means_bytes(d) == rows * (128 * 4 + 128 * 2 + 4)
    assert kin.kin_dual_means_bytes(dims(D=64)) == 0
    # per page: one row per (page, KV head)
    assert kin.kin_dual_page_means_bytes(d, 5) == 5 * d.num_kv_heads * (128 * 4 + 128 * 2 + 4)
    assert kin.kin_dual_page_means_bytes(d, 0) == 0
    assert kin.kin_dual_page_means_bytes(dims(D=64), 5) == 0
    assert kin.kin_workspace_bytes(dims(), 1) == 0
    assert kin.kin_workspace_bytes(dims(D=64), 8) == 0
    assert kin.kin_workspace_bytes(dims(bs=24), 8) == 0
    assert kin.kin_workspace_bytes(dims(Hq=7), 8) == 0
    assert kin.kin_workspace_bytes(dims(Hq=32, Hkv=2), 8) == 0       # g = 16
    n8 = kin.kin_workspace_bytes(dims(), 8)
    pairs, nbcap = 4, 16
    assert n8 >= pairs * nbcap * 4 + 2 * pairs * 4
    assert n8 % 256 == 0
    assert kin.kin_workspace_bytes(dims(), 16) >= n8
    big = kin.make_dims(32, 8, 32, 128, 16, 32768)
    assert kin.kin_workspace_bytes(big, 256) >= 32 * 8 * 2048 * 4


FAKE = ctypes.c_void_p(1 << 20)   # aligned, never dereferenced: every call below fails its host checks


def test_select_rejects_before_launch(lib):
    d = dims()
    args = lambda k=8, q=FAKE, ws=FAKE, n=1 << 30: (ctypes.byref(d), q, FAKE, FAKE, k, FAKE, FAKE, ws, n,
                                                   None, None)
    assert lib.kin_block_topk_select(*args(k=1)) == 1
    assert lib.kin_block_topk_select(*args(q=None)) == 1
    assert lib.kin_block_topk_select(*args(q=ctypes.c_void_p((1 << 20) + 2))) == 1
    assert lib.kin_block_topk_select(*args(ws=None)) == 2
    assert lib.kin_block_topk_select(*args(ws=ctypes.c_void_p((1 << 20) + 16))) == 2
    assert lib.kin_block_topk_select(*args(n=64)) == 2
    bad = kin.make_dims(2, 2, 8, 128, 16, 0)
    assert lib.kin_block_topk_select(ctypes.byref(bad), FAKE, FAKE, FAKE, 8, FAKE, FAKE, FAKE, 1 << 30,
                                     None, None) == 1
    huge = kin.make_dims(1, 1, 1, 128, 16, 16 * 32768 + 1)
    assert lib.kin_block_topk_select(ctypes.byref(huge), FAKE, FAKE, FAKE, 8, FAKE, FAKE, FAKE, 1 << 40,
                                     None, None) == 3
    assert lib.kin_block_topk_select(None, FAKE, FAKE, FAKE, 8, FAKE, FAKE, FAKE, 1 << 30, None, None) == 1


def test_attn_rejects_before_launch(lib):
    d = dims()
    def call(scale=0.0, ws=FAKE, n=1 << 30, out=FAKE, k=8):
        return lib.kin_sparse_decode_attn(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, k, scale,
                                          out, None, ws, n, None, None)
    assert call(k=0) == 1
    assert call(out=None) == 1
    assert call(scale=float("nan")) == 1
    assert call(scale=float("inf")) == 1
    assert call(ws=None) == 2
    assert call(n=100) == 2


def test_means_calls_reject_before_launch(lib):
    d = dims()
    assert lib.kin_block_means_update(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, -1, None, None) == 1
    assert lib.kin_block_means_update(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, None, None) == 0
    assert lib.kin_block_means_update(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 257, None, None) == 3
    assert lib.kin_block_means_update(ctypes.byref(d), None, FAKE, FAKE, FAKE, FAKE, FAKE, 1, None, None) == 1
    assert lib.kin_block_means_build(ctypes.byref(d), None, FAKE, FAKE, None, None) == 1
    assert lib.kin_block_means_build(ctypes.byref(dims(bs=8)), FAKE, FAKE, FAKE, None, None) == 1


def test_paged_calls_reject_before_launch(lib):
    d = dims()
    bd = ctypes.byref(d)
    # build: pool, table, page count, means
    assert lib.kin_block_means_build_paged(bd, None, 4, FAKE, FAKE, FAKE, None, None) == 1
    assert lib.kin_block_means_build_paged(bd, FAKE, 0, FAKE, FAKE, FAKE, None, None) == 1
    assert lib.kin_block_means_build_paged(bd, FAKE, 4, None, FAKE, FAKE, None, None) == 1
    assert lib.kin_block_means_build_paged(bd, ctypes.c_void_p((1 << 20) + 8), 4, FAKE, FAKE, FAKE, None,
                                           None) == 1
    assert lib.kin_block_means_build_paged(bd, FAKE, 4, FAKE, FAKE, None, None, None) == 1
    # update: counts first (as the contiguous call), then the pool and table
    up = lambda n, pool=FAKE, pages=4, table=FAKE: lib.kin_block_means_update_paged(
        bd, pool, FAKE, pages, table, FAKE, FAKE, FAKE, FAKE, n, None, None)
    assert up(-1) == 1
    assert up(257) == 3
    assert up(0, pool=None) == 0
    assert up(1, pages=0) == 1
    assert up(1, table=None) == 1
    assert up(1, pool=None) == 1
    # attention: pool and table, then the checks of the contiguous call
    at = lambda pages=4, table=FAKE, k=8, ws=FAKE, n=1 << 30: lib.kin_sparse_decode_attn_paged(
        bd, FAKE, FAKE, FAKE, pages, table, FAKE, FAKE, FAKE, k, 0.0, FAKE, None, ws, n, None, None)
    assert at(pages=0) == 1
    assert at(pages=-3) == 1
    assert at(table=None) == 1
    assert at(k=1) == 1
    assert at(ws=None) == 2
    assert at(n=64) == 2


def test_extended_calls_reject_before_launch(lib):
    d = dims()
    bd = ctypes.byref(d)
    sel = lambda dt=1, k=8, ws=FAKE: lib.kin_block_topk_select_ex(bd, FAKE, FAKE, dt, FAKE, k, FAKE, FAKE, ws,
                                                                  1 << 30, None, None)
    assert sel(dt=3) == 1                          # 0 fp32, 1 bf16, 2 dual
    assert sel(dt=-1) == 1
    assert sel(dt=2 | 0x100) == 1                  # per-page means need the paged select
    assert sel(k=1) == 1
    assert sel(ws=None) == 2
    build = lambda dt=1, pool=FAKE, pages=0, table=None: lib.kin_block_means_build_ex(
        bd, pool, pages, table, FAKE, FAKE, dt, None, None)
    assert build(dt=7) == 1
    assert build(dt=2 | 0x100, pages=0, table=None) == 1   # per-page (dual) means need a table
    assert build(pool=None) == 1
    assert build(pages=0, table=FAKE) == 1        # a table needs a pool of >= 1 page
    upd = lambda dt=1, n=1, pages=4, table=FAKE: lib.kin_block_means_update_ex(
        bd, FAKE, FAKE, pages, table, FAKE, dt, FAKE, FAKE, FAKE, n, None, None)
    assert upd(dt=3) == 1
    assert upd(dt=2 | 0x100, table=None) == 1
    assert upd(n=-1) == 1
    assert upd(n=0) == 0
    assert upd(n=257) == 3
    assert upd(pages=0) == 1


def test_token_and_page_means_calls_reject_before_launch(lib):
    d = dims()
    bd = ctypes.byref(d)
    # token workspace: logits + kept indices + counts; a key scratch row only past 32768 tokens
    assert kin.kin_token_topk_workspace_bytes(d, 0) == 0
    assert kin.kin_token_topk_workspace_bytes(dims(D=64), 8) == 0
    rows, L = 2 * 8, 256
    n8 = kin.kin_token_topk_workspace_bytes(d, 8)
    assert n8 >= rows * L * 4 + rows * 8 * 4 + rows * 4 and n8 % 256 == 0
    assert kin.kin_token_topk_workspace_bytes(d, 64) >= n8 + rows * 56 * 4
    at_cap = kin.kin_token_topk_workspace_bytes(kin.make_dims(1, 1, 2, 128, 16, 32768), 8)
    past_cap = kin.kin_token_topk_workspace_bytes(kin.make_dims(1, 1, 2, 128, 16, 32769), 8)
    assert at_cap < 2 * 32768 * 8 and past_cap >= 2 * 32769 * 8
    tok = lambda k=8, q=FAKE, scale=0.0, ws=FAKE, n=1 << 30, dd=bd: lib.kin_token_topk_decode_attn(
        dd, q, FAKE, FAKE, FAKE, k, scale, FAKE, None, None, ws, n, None, None)
    assert tok(k=0) == 1
    assert tok(q=None) == 1
    assert tok(q=ctypes.c_void_p((1 << 20) + 2)) == 1
    assert tok(scale=float("nan")) == 1
    assert tok(scale=float("inf")) == 1
    assert tok(ws=None) == 2
    assert tok(ws=ctypes.c_void_p((1 << 20) + 16)) == 2
    assert tok(n=64) == 2
    rows_cap = kin.make_dims(64, 8, 64, 128, 16, 1 << 19)   # B * Hq * Lcap = 2^31
    assert tok(dd=ctypes.byref(rows_cap)) == 3
    # the select over means stored per page
    sp = lambda dt=0, pages=4, table=FAKE, pool=FAKE, k=8, ws=FAKE: lib.kin_block_topk_select_paged(
        bd, FAKE, pool, dt, pages, table, FAKE, k, FAKE, FAKE, ws, 1 << 30, None, None)
    assert sp(dt=3) == 1                          # an unknown means dtype
    assert sp(pages=0) == 1
    assert sp(table=None) == 1
    assert sp(pool=None) == 1
    assert sp(pool=ctypes.c_void_p((1 << 20) + 8)) == 1
    assert sp(k=1) == 1
    assert sp(ws=None) == 2


def test_binding_refuses_host_tensors(lib):
    import torch
    with pytest.raises(ValueError):
        kin.kin_block_means_build(dims(), torch.zeros(4, dtype=torch.bfloat16),
                                  torch.zeros(2, dtype=torch.int32), torch.zeros(4))


def test_missing_library_fails_loudly(tmp_path):
    saved = kin._lib
    try:
        kin._lib = None
        with pytest.raises(RuntimeError):
            kin.load_library(str(tmp_path / "nope.so"))
    finally:
        kin._lib = saved
