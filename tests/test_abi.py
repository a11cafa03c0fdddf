"""The C-ABI library loads on a machine without a GPU, exports every symbol
include/dash.h declares, and rejects invalid arguments before touching CUDA."""

import ctypes
import os
import re

import pytest

from sparse_hierarchical_attention_chunk_b200 import build as dash_build
from sparse_hierarchical_attention_chunk_b200 import dash

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    dash_build.build()
    return dash.lib()


def _declared():
    text = open(os.path.join(ROOT, "include", "dash.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dash_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding_names():
    assert set(_declared()) == set(dash.EXPORTED)


def test_every_declared_symbol_is_exported(L):
    for name in _declared():
        assert hasattr(L, name), name


def test_status_strings_and_version(L):
    assert dash.status_str(0) == "DASH_OK"
    assert dash.status_str(4) == "DASH_ERR_TIMEOUT"
    assert dash.status_str(99) == "DASH_ERR_UNKNOWN"
    assert L.dash_version() >> 16 == 3


def _p(**kw):
    base = dict(batch=1, n_q_heads=32, n_kv_heads=2, seq_len=1024, head_dim=128, chunk=64,
                alpha=1.5, gamma=1.0, sigma=1.0, dtype="bf16")
    base.update(kw)
    return dash.problem(**base)


FAKE = ctypes.c_void_p(1 << 20)      # never dereferenced: validation fails first

# These calls hand the library fake device addresses and rely on host-side
# validation rejecting them before any launch.  They are host-logic tests: on
# a machine with a GPU they are skipped, so a validation bug can never turn
# into a kernel reading a fake address.
host_only = pytest.mark.skipif(__import__("torch").cuda.is_available(),
                               reason="fake device pointers are only passed where no GPU exists")


@pytest.mark.parametrize("kw", [
    dict(head_dim=96), dict(chunk=32), dict(n_q_heads=31), dict(seq_len=1000), dict(alpha=1.0),
    dict(alpha=2.5), dict(gamma=0.0), dict(sigma=-1.0), dict(batch=0),
])
@host_only
def test_invalid_problem_rejected(L, kw):
    p = _p(**kw)
    st = L.dash_route(ctypes.byref(p), FAKE, FAKE, None, None, FAKE, FAKE, None)
    assert st == dash.DASH_ERR_INVALID_ARG


@host_only
def test_null_and_misaligned_pointers_rejected(L):
    p = _p()
    assert L.dash_route(None, FAKE, FAKE, None, None, FAKE, FAKE, None) == dash.DASH_ERR_INVALID_ARG
    assert L.dash_route(ctypes.byref(p), None, FAKE, None, None, FAKE, FAKE, None) == dash.DASH_ERR_INVALID_ARG
    odd = ctypes.c_void_p((1 << 20) + 8)
    assert L.dash_route(ctypes.byref(p), odd, FAKE, None, None, FAKE, FAKE, None) == dash.DASH_ERR_INVALID_ARG
    assert L.dash_attn_fwd(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, 0,
                           None) == dash.DASH_ERR_INVALID_ARG
    assert L.dash_summarize(ctypes.byref(p), FAKE, FAKE, 0, 17, FAKE, None) == dash.DASH_ERR_INVALID_ARG
    assert L.dash_summarize(ctypes.byref(p), FAKE, FAKE, 3, 2, FAKE, None) == dash.DASH_ERR_INVALID_ARG


@host_only
def test_unsupported_shapes(L):
    # bf16 stage 2 wants 128 / G positions per tile inside one chunk
    p = _p(n_q_heads=2, n_kv_heads=2)
    assert L.dash_attn_fwd(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 0,
                           None) == dash.DASH_ERR_UNSUPPORTED
    # routing keeps a row of chunk scores per warp in registers: n_c <= 2048
    p = _p(seq_len=2048 * 64 + 64)
    assert L.dash_route(ctypes.byref(p), FAKE, FAKE, None, None, FAKE, FAKE, None) == dash.DASH_ERR_UNSUPPORTED
    # decode runs in bf16
    p = _p(dtype="f32", seq_len=1000)
    assert L.dash_decode(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, None, FAKE, None, None, None,
                         FAKE, 1 << 30, None) == dash.DASH_ERR_UNSUPPORTED


@host_only
def test_decode_varlen_lengths_pointer_checked(L):
    p = _p(batch=8, seq_len=131072)
    need = dash.dash_workspace_bytes(p, True)
    assert L.dash_decode_varlen(ctypes.byref(p), None, FAKE, FAKE, FAKE, FAKE, None, FAKE, None,
                                None, None, FAKE, need, None) == dash.DASH_ERR_INVALID_ARG
    odd = ctypes.c_void_p((1 << 20) + 2)
    assert L.dash_decode_varlen(ctypes.byref(p), odd, FAKE, FAKE, FAKE, FAKE, None, FAKE, None,
                                None, None, FAKE, need, None) == dash.DASH_ERR_INVALID_ARG
    # the rest is dash_decode's validation
    assert L.dash_decode_varlen(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, None,
                                None, None, FAKE, need - 1, None) == dash.DASH_ERR_WORKSPACE
    p = _p(dtype="f32", seq_len=1000)
    assert L.dash_decode_varlen(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, None,
                                None, None, FAKE, 1 << 30, None) == dash.DASH_ERR_UNSUPPORTED


@host_only
def test_decode_paged_arguments_checked(L):
    p = _p(batch=8, seq_len=131072, chunk=64)
    need = dash.dash_workspace_bytes(p, True)
    n_c = 131072 // 64
    args = lambda lens, table, max_pages, n_pages: (ctypes.byref(p), lens, table, max_pages, n_pages,
                                                    FAKE, FAKE, FAKE, FAKE, None, FAKE, None, None,
                                                    None, FAKE, need, None)
    odd = ctypes.c_void_p((1 << 20) + 2)
    assert L.dash_decode_paged(*args(None, FAKE, n_c, 10)) == dash.DASH_ERR_INVALID_ARG
    assert L.dash_decode_paged(*args(FAKE, None, n_c, 10)) == dash.DASH_ERR_INVALID_ARG
    assert L.dash_decode_paged(*args(FAKE, odd, n_c, 10)) == dash.DASH_ERR_INVALID_ARG
    assert L.dash_decode_paged(*args(FAKE, FAKE, n_c - 1, 10)) == dash.DASH_ERR_INVALID_ARG
    assert L.dash_decode_paged(*args(FAKE, FAKE, n_c, 0)) == dash.DASH_ERR_INVALID_ARG
    # 32-bit row coordinates of the page pool
    assert L.dash_decode_paged(*args(FAKE, FAKE, n_c, 1 << 24)) == dash.DASH_ERR_UNSUPPORTED


@host_only
def test_route_topk_arguments_checked(L):
    p = _p()
    assert L.dash_route_topk(ctypes.byref(p), FAKE, FAKE, 0, FAKE, FAKE, None) == dash.DASH_ERR_INVALID_ARG
    assert L.dash_route_topk(ctypes.byref(p), None, FAKE, 4, FAKE, FAKE, None) == dash.DASH_ERR_INVALID_ARG
    p = _p(n_q_heads=34, n_kv_heads=2)                # G = 17
    assert L.dash_route_topk(ctypes.byref(p), FAKE, FAKE, 4, FAKE, FAKE, None) == dash.DASH_ERR_UNSUPPORTED


def test_attn_bwd_arguments_checked(L):
    p = _p()
    args = [FAKE] * 11
    for k in range(11):                                # every required pointer
        a = list(args)
        a[k] = None
        assert L.dash_attn_bwd(ctypes.byref(p), *a, None, None, 0, None) == dash.DASH_ERR_INVALID_ARG
    odd = ctypes.c_void_p((1 << 20) + 8)
    assert L.dash_attn_bwd(ctypes.byref(p), *args, odd, None, 0, None) == dash.DASH_ERR_INVALID_ARG


@host_only
def test_attn_bwd_workspace_checked(L):
    # the tensor-core backward (bf16, d = 128, G in {4, 8, 16}) needs scratch
    # for its D rows and tile unions; the reference kernel needs none
    p = _p()
    need = dash.dash_workspace_bytes(p, 2)
    # D rows [1, 32, 1024] fp32, tile unions [2, 1, 1024 / 8] u32 (256-byte
    # rounded), and 8 splits of the 16 key blocks' partial dK | dV rows
    # [8, 2 * 1024, 256] fp32
    assert need == 1 * 32 * 1024 * 4 + 1024 + 8 * 2 * 1024 * 256 * 4
    # long sequences have enough key blocks: no split, no partials
    pl = _p(seq_len=131072, chunk=128)
    assert dash.dash_workspace_bytes(pl, 2) == 32 * 131072 * 4 + 2 * 32 * (131072 // 8) * 4
    assert dash.dash_workspace_bytes(_p(dtype="f32"), 2) == 0
    assert dash.dash_workspace_bytes(_p(head_dim=64), 2) == 0
    assert dash.dash_workspace_bytes(p, 3) == 0
    args = [FAKE] * 11
    assert L.dash_attn_bwd(ctypes.byref(p), *args, None, None, need, None) == dash.DASH_ERR_WORKSPACE
    assert L.dash_attn_bwd(ctypes.byref(p), *args, None, FAKE, need - 1, None) == dash.DASH_ERR_WORKSPACE
    odd = ctypes.c_void_p((1 << 20) + 16)
    assert L.dash_attn_bwd(ctypes.byref(p), *args, None, odd, need, None) == dash.DASH_ERR_WORKSPACE


@host_only
def test_decode_workspace_checked(L):
    p = _p(batch=8, seq_len=131072)
    need = dash.dash_workspace_bytes(p, True)
    assert need > 0 and need % 256 == 0
    assert dash.dash_workspace_bytes(p, False) == 0
    assert L.dash_decode(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, None, FAKE, None, None, None,
                         FAKE, need - 1, None) == dash.DASH_ERR_WORKSPACE
    assert L.dash_decode(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, None, FAKE, None, None, None,
                         None, need, None) == dash.DASH_ERR_WORKSPACE


@host_only
def test_estimate_diagonal_arguments_checked(L):
    # the flag is 0 or 1; with it, routing needs K and qbar, decode needs qbar
    p = _p()
    p.estimate_diagonal = 2
    assert L.dash_route(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None) == \
        dash.DASH_ERR_INVALID_ARG
    p.estimate_diagonal = 1
    assert L.dash_route(ctypes.byref(p), FAKE, FAKE, None, FAKE, FAKE, FAKE, None) == \
        dash.DASH_ERR_INVALID_ARG
    assert L.dash_route(ctypes.byref(p), FAKE, FAKE, FAKE, None, FAKE, FAKE, None) == \
        dash.DASH_ERR_INVALID_ARG
    odd = ctypes.c_void_p((1 << 20) + 8)
    assert L.dash_route(ctypes.byref(p), FAKE, FAKE, odd, FAKE, FAKE, FAKE, None) == \
        dash.DASH_ERR_INVALID_ARG
    # no entmax normalisation in top-k routing, no gradient through the
    # diagonal candidate, no qbar argument in the no-allocation decode
    assert L.dash_route_topk(ctypes.byref(p), FAKE, FAKE, 4, FAKE, FAKE, None) == \
        dash.DASH_ERR_UNSUPPORTED
    assert L.dash_route_bwd(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None) == \
        dash.DASH_ERR_UNSUPPORTED
    pd = _p(batch=8, seq_len=131072)
    pd.estimate_diagonal = 1
    need = dash.dash_workspace_bytes(pd, True)
    assert L.dash_decode(ctypes.byref(pd), FAKE, FAKE, FAKE, FAKE, None, FAKE, None, None, None,
                         FAKE, need, None) == dash.DASH_ERR_INVALID_ARG
    assert L.dash_decode_noalloc(ctypes.byref(pd), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None,
                                 None) == dash.DASH_ERR_UNSUPPORTED


def test_bwd_split_hook_sets_the_workspace(L):
    # the forced split count of the tensor-core backward: no partial rows when
    # unsplit, n_split of them otherwise; 0 restores the automatic choice
    p = _p()
    base = 1 * 32 * 1024 * 4 + 1024
    rows = 2 * 1024 * 256 * 4
    try:
        assert dash.dash_selftest_bwd_split(1) == 0
        assert dash.dash_workspace_bytes(p, 2) == base
        assert dash.dash_selftest_bwd_split(3) == 1
        assert dash.dash_workspace_bytes(p, 2) == base + 3 * rows
    finally:
        assert dash.dash_selftest_bwd_split(0) == 3
    assert dash.dash_workspace_bytes(p, 2) == base + 8 * rows
    assert L.dash_selftest_bwd_split(9) == -1 and L.dash_selftest_bwd_split(-1) == -1
