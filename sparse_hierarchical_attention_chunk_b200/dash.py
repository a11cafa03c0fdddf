"""Thin Python binding of the C ABI in ``include/dash.h`` (ctypes).

Argument marshalling only: shape/dtype/device checks, device pointers and the
current CUDA stream are passed to ``libdash.so``; every step of the path runs
in its CUDA kernels.  There is no CPU fallback: if the library is missing or
a call fails, an exception is raised.

Functions keep the C names: :func:`dash_summarize`, :func:`dash_route`,
:func:`dash_attn_fwd`, :func:`dash_decode`, :func:`dash_workspace_bytes`,
:func:`dash_get_error`.  :func:`prefill` and :func:`decode` chain them with
freshly allocated outputs.
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdash.so")

DASH_OK = 0
DASH_ERR_INVALID_ARG = 1
DASH_ERR_UNSUPPORTED = 2
DASH_ERR_CUDA = 3
DASH_ERR_TIMEOUT = 4
DASH_ERR_WORKSPACE = 5
DASH_F32 = 0
DASH_BF16 = 1

EXPORTED = ("dash_status_str", "dash_version", "dash_summarize", "dash_route", "dash_attn_fwd",
            "dash_workspace_bytes", "dash_decode", "dash_decode_varlen", "dash_decode_paged",
            "dash_get_error", "dash_decode_noalloc", "dash_summarize_append", "dash_route_topk",
            "dash_attn_bwd", "dash_route_bwd", "dash_summarize_bwd", "dash_selftest_wait_timeout",
            "dash_selftest_exp2_poly", "dash_route_packed", "dash_attn_fwd_packed",
            "dash_selftest_bwd_split")


class DashError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {status_str(status)} ({status})")


class DashProblem(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("n_q_heads", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("seq_len", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("chunk", ctypes.c_int32),
        ("alpha", ctypes.c_float),
        ("gamma", ctypes.c_float),
        ("sigma", ctypes.c_float),
        ("dtype", ctypes.c_int32),
        ("estimate_diagonal", ctypes.c_int32),
    ]


_lib = None


def lib():
    """Load libdash.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m sparse_hierarchical_attention_chunk_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        P = ctypes.POINTER(DashProblem)
        L.dash_status_str.restype = ctypes.c_char_p
        L.dash_status_str.argtypes = [i32]
        L.dash_version.restype = i32
        L.dash_summarize.restype = i32
        L.dash_summarize.argtypes = [P, vp, vp, i32, i32, vp, vp]
        L.dash_summarize_append.restype = i32
        L.dash_summarize_append.argtypes = [P, vp, vp, i32, i32, vp, vp, vp, vp]
        L.dash_route_topk.restype = i32
        L.dash_route_topk.argtypes = [P, vp, vp, i32, vp, vp, vp]
        L.dash_route_bwd.restype = i32
        L.dash_route_bwd.argtypes = [P, vp, vp, vp, vp, vp, vp]
        L.dash_summarize_bwd.restype = i32
        L.dash_summarize_bwd.argtypes = [P, vp, vp, vp, vp, vp, vp]
        L.dash_attn_bwd.restype = i32
        L.dash_attn_bwd.argtypes = [P] + [vp] * 13 + [ctypes.c_size_t, vp]
        L.dash_route.restype = i32
        L.dash_route.argtypes = [P, vp, vp, vp, vp, vp, vp, vp]
        L.dash_route_packed.restype = i32
        L.dash_route_packed.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.dash_attn_fwd_packed.restype = i32
        L.dash_attn_fwd_packed.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp]
        L.dash_attn_fwd.restype = i32
        L.dash_attn_fwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.dash_workspace_bytes.restype = ctypes.c_size_t
        L.dash_workspace_bytes.argtypes = [P, i32]
        L.dash_decode.restype = i32
        L.dash_decode.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.dash_decode_varlen.restype = i32
        L.dash_decode_varlen.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                         ctypes.c_size_t, vp]
        L.dash_decode_paged.restype = i32
        L.dash_decode_paged.argtypes = [P, vp, vp, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                        ctypes.c_size_t, vp]
        L.dash_selftest_wait_timeout.restype = i32
        L.dash_selftest_wait_timeout.argtypes = [vp]
        L.dash_selftest_exp2_poly.restype = i32
        L.dash_selftest_exp2_poly.argtypes = [vp, vp, i32, vp]
        L.dash_selftest_bwd_split.restype = i32
        L.dash_selftest_bwd_split.argtypes = [i32]
        L.dash_get_error.restype = i32
        L.dash_get_error.argtypes = [vp]
        L.dash_decode_noalloc.restype = i32
        L.dash_decode_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        _lib = L
    return _lib


def status_str(status):
    return lib().dash_status_str(int(status)).decode()


def problem(batch, n_q_heads, n_kv_heads, seq_len, head_dim, chunk, alpha=1.5, gamma=1.0,
            sigma=1.0, dtype="bf16", estimate_diagonal=False):
    return DashProblem(batch, n_q_heads, n_kv_heads, seq_len, head_dim, chunk, alpha, gamma, sigma,
                       DASH_BF16 if dtype in ("bf16", torch.bfloat16) else DASH_F32,
                       1 if estimate_diagonal else 0)


def problem_for(wl, sigma=None, estimate_diagonal=False):
    """DashProblem for a :class:`configs.Workload`."""
    return problem(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.seq, wl.head_dim, wl.chunk,
                   wl.alpha, wl.gamma, wl.sigma if sigma is None else sigma, wl.dtype,
                   estimate_diagonal)


def _tdtype(p):
    return torch.bfloat16 if p.dtype == DASH_BF16 else torch.float32


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(t, name, shape, dtype):
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _raise(fn, st):
    if st != DASH_OK:
        raise DashError(fn, st)


def n_chunks(p):
    return (p.seq_len + p.chunk - 1) // p.chunk


def n_words(p):
    return (n_chunks(p) + 31) // 32


def dash_summarize(p, K, qbar, Kbar, chunk_begin=0, chunk_end=None, stream=None):
    dt = _tdtype(p)
    full = p.seq_len // p.chunk
    chunk_end = full if chunk_end is None else chunk_end
    _check(K, "K", (p.batch, p.n_kv_heads, p.seq_len, p.head_dim), dt)
    _check(qbar, "qbar", (p.n_kv_heads, p.head_dim), torch.float32)
    _check(Kbar, "Kbar", (p.batch, p.n_kv_heads, full, p.head_dim), dt)
    _raise("dash_summarize", lib().dash_summarize(ctypes.byref(p), _ptr(K), _ptr(qbar), chunk_begin,
                                                  chunk_end, _ptr(Kbar), _stream(stream)))


def dash_summarize_append(p, cache_lens, K, qbar, Kbar, page_table=None, stream=None):
    """Write the summary of the chunk each sequence's newest token completed
    (sequences whose length is a multiple of the chunk size); K is the cache,
    or with page_table the page pool of dash_decode_paged."""
    dt = _tdtype(p)
    full = p.seq_len // p.chunk
    if page_table is None:
        _check(K, "K", (p.batch, p.n_kv_heads, p.seq_len, p.head_dim), dt)
    else:
        _check(K, "Kpool", (K.shape[0], p.n_kv_heads, p.chunk, p.head_dim), dt)
        _check(page_table, "page_table", (p.batch, page_table.shape[1]), torch.int32)
    _check(cache_lens, "cache_lens", (p.batch,), torch.int32)
    _check(qbar, "qbar", (p.n_kv_heads, p.head_dim), torch.float32)
    _check(Kbar, "Kbar", (p.batch, p.n_kv_heads, full, p.head_dim), dt)
    mp = int(page_table.shape[1]) if page_table is not None else 0
    npg = int(K.shape[0]) if page_table is not None else 0
    _raise("dash_summarize_append",
           lib().dash_summarize_append(ctypes.byref(p), _ptr(cache_lens), _ptr(page_table), mp, npg,
                                       _ptr(K), _ptr(qbar), _ptr(Kbar), _stream(stream)))


def dash_route_topk(p, Q, Kbar, k, w, mask, stream=None):
    """Fixed-budget top-k routing (the NSA / InfLLMv2-style baseline) into
    dash_route's w and mask layouts."""
    dt = _tdtype(p)
    _check(Q, "Q", (p.batch, p.n_q_heads, p.seq_len, p.head_dim), dt)
    _check(Kbar, "Kbar", (p.batch, p.n_kv_heads, p.seq_len // p.chunk, p.head_dim), dt)
    _check(w, "w", (p.batch, p.n_kv_heads, p.seq_len, n_chunks(p)), torch.float32)
    _check(mask, "mask", (p.batch, p.n_kv_heads, p.seq_len, n_words(p)), torch.int32)
    _raise("dash_route_topk", lib().dash_route_topk(ctypes.byref(p), _ptr(Q), _ptr(Kbar), int(k),
                                                    _ptr(w), _ptr(mask), _stream(stream)))


def dash_attn_bwd(p, Q, K, V, w, mask, O, lse, dO, dQ, dK, dV, dw=None, workspace=None, stream=None):
    """Stage-2 gradients (fp32 dQ, dK, dV, and dw if given) for the cotangent dO.
    `workspace` (uint8, dash_workspace_bytes(p, 2) bytes) is allocated here
    when not given."""
    dt = _tdtype(p)
    f32 = torch.float32
    _check(Q, "Q", (p.batch, p.n_q_heads, p.seq_len, p.head_dim), dt)
    _check(K, "K", (p.batch, p.n_kv_heads, p.seq_len, p.head_dim), dt)
    _check(V, "V", (p.batch, p.n_kv_heads, p.seq_len, p.head_dim), dt)
    _check(w, "w", (p.batch, p.n_kv_heads, p.seq_len, n_chunks(p)), f32)
    _check(mask, "mask", (p.batch, p.n_kv_heads, p.seq_len, n_words(p)), torch.int32)
    _check(O, "O", (p.batch, p.n_q_heads, p.seq_len, p.head_dim), dt)
    _check(lse, "lse", (p.batch, p.n_q_heads, p.seq_len), f32)
    _check(dO, "dO", (p.batch, p.n_q_heads, p.seq_len, p.head_dim), dt)
    _check(dQ, "dQ", (p.batch, p.n_q_heads, p.seq_len, p.head_dim), f32)
    _check(dK, "dK", (p.batch, p.n_kv_heads, p.seq_len, p.head_dim), f32)
    _check(dV, "dV", (p.batch, p.n_kv_heads, p.seq_len, p.head_dim), f32)
    if dw is not None:
        _check(dw, "dw", (p.batch, p.n_kv_heads, p.seq_len, n_chunks(p)), f32)
    need = dash_workspace_bytes(p, 2)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=Q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _raise("dash_attn_bwd", lib().dash_attn_bwd(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(w),
                                                _ptr(mask), _ptr(O), _ptr(lse), _ptr(dO), _ptr(dQ),
                                                _ptr(dK), _ptr(dV), _ptr(dw), _ptr(workspace),
                                                ws_bytes, _stream(stream)))


def dash_route_bwd(p, Q, Kbar, dw, dQ, dKbar, stream=None):
    """Stage-1 gradients accumulated into dQ and dKbar (fp32) for the cotangent dw."""
    dt, f32 = _tdtype(p), torch.float32
    _check(Q, "Q", (p.batch, p.n_q_heads, p.seq_len, p.head_dim), dt)
    _check(Kbar, "Kbar", (p.batch, p.n_kv_heads, p.seq_len // p.chunk, p.head_dim), dt)
    _check(dw, "dw", (p.batch, p.n_kv_heads, p.seq_len, n_chunks(p)), f32)
    _check(dQ, "dQ", (p.batch, p.n_q_heads, p.seq_len, p.head_dim), f32)
    _check(dKbar, "dKbar", (p.batch, p.n_kv_heads, p.seq_len // p.chunk, p.head_dim), f32)
    _raise("dash_route_bwd", lib().dash_route_bwd(ctypes.byref(p), _ptr(Q), _ptr(Kbar), _ptr(dw),
                                                  _ptr(dQ), _ptr(dKbar), _stream(stream)))


def dash_summarize_bwd(p, K, qbar, dKbar, dK, dqbar, stream=None):
    """Stage-0 gradients accumulated into dK and dqbar (fp32) for the cotangent dKbar."""
    dt, f32 = _tdtype(p), torch.float32
    _check(K, "K", (p.batch, p.n_kv_heads, p.seq_len, p.head_dim), dt)
    _check(qbar, "qbar", (p.n_kv_heads, p.head_dim), f32)
    _check(dKbar, "dKbar", (p.batch, p.n_kv_heads, p.seq_len // p.chunk, p.head_dim), f32)
    _check(dK, "dK", (p.batch, p.n_kv_heads, p.seq_len, p.head_dim), f32)
    _check(dqbar, "dqbar", (p.n_kv_heads, p.head_dim), f32)
    _raise("dash_summarize_bwd", lib().dash_summarize_bwd(ctypes.byref(p), _ptr(K), _ptr(qbar),
                                                          _ptr(dKbar), _ptr(dK), _ptr(dqbar),
                                                          _stream(stream)))


def backward(p, Q, K, V, qbar, out, dO, stream=None):
    """Gradients of the whole forward path (stages 2, 1, 0) for the cotangent
    dO, from dash.prefill's outputs (lse required): dQ, dK, dV, dqbar (fp32)."""
    f32 = dict(dtype=torch.float32, device=Q.device)
    dQ, dK, dV = torch.empty(Q.shape, **f32), torch.empty(K.shape, **f32), torch.empty(V.shape, **f32)
    dw = torch.empty(out["w"].shape, **f32)
    dKbar = torch.zeros(out["Kbar"].shape, **f32)
    dqbar = torch.zeros(qbar.shape, **f32)
    dash_attn_bwd(p, Q, K, V, out["w"], out["mask"], out["O"], out["lse"], dO, dQ, dK, dV, dw,
                  stream=stream)
    dash_route_bwd(p, Q, out["Kbar"], dw, dQ, dKbar, stream)
    dash_summarize_bwd(p, K, qbar, dKbar, dK, dqbar, stream)
    return {"dQ": dQ, "dK": dK, "dV": dV, "dqbar": dqbar, "dw": dw, "dKbar": dKbar}


def dash_route(p, Q, Kbar, w, mask, stream=None, K=None, qbar=None):
    """Stage 1; with p.estimate_diagonal the keys K and learned queries qbar
    of stage 0 are required as well."""
    dt = _tdtype(p)
    _check(Q, "Q", (p.batch, p.n_q_heads, p.seq_len, p.head_dim), dt)
    _check(Kbar, "Kbar", (p.batch, p.n_kv_heads, p.seq_len // p.chunk, p.head_dim), dt)
    _check(w, "w", (p.batch, p.n_kv_heads, p.seq_len, n_chunks(p)), torch.float32)
    _check(mask, "mask", (p.batch, p.n_kv_heads, p.seq_len, n_words(p)), torch.int32)
    if p.estimate_diagonal:
        if K is None or qbar is None:
            raise ValueError("estimate_diagonal needs K and qbar")
        _check(K, "K", (p.batch, p.n_kv_heads, p.seq_len, p.head_dim), dt)
        _check(qbar, "qbar", (p.n_kv_heads, p.head_dim), torch.float32)
    _raise("dash_route", lib().dash_route(ctypes.byref(p), _ptr(Q), _ptr(Kbar), _ptr(K), _ptr(qbar),
                                          _ptr(w), _ptr(mask), _stream(stream)))


def dash_route_packed(p, Q, Kbar, mask, weight, count=None, index=None, stream=None, K=None,
                      qbar=None):
    """Stage 1 with compact weights: per row, the weights of the routed chunks
    in increasing chunk order (weight), optionally their count and chunk
    numbers (index).  Rows keep the dense row length n_c."""
    dt = _tdtype(p)
    rows = (p.batch, p.n_kv_heads, p.seq_len)
    _check(Q, "Q", (p.batch, p.n_q_heads, p.seq_len, p.head_dim), dt)
    _check(Kbar, "Kbar", (p.batch, p.n_kv_heads, p.seq_len // p.chunk, p.head_dim), dt)
    _check(mask, "mask", rows + (n_words(p),), torch.int32)
    _check(weight, "weight", rows + (n_chunks(p),), torch.float32)
    if count is not None:
        _check(count, "count", rows, torch.int32)
    if index is not None:
        _check(index, "index", rows + (n_chunks(p),), torch.int32)
    if p.estimate_diagonal:
        if K is None or qbar is None:
            raise ValueError("estimate_diagonal needs K and qbar")
        _check(K, "K", (p.batch, p.n_kv_heads, p.seq_len, p.head_dim), dt)
        _check(qbar, "qbar", (p.n_kv_heads, p.head_dim), torch.float32)
    _raise("dash_route_packed",
           lib().dash_route_packed(ctypes.byref(p), _ptr(Q), _ptr(Kbar), _ptr(K), _ptr(qbar),
                                   _ptr(mask), _ptr(count), _ptr(index), _ptr(weight),
                                   _stream(stream)))


def dash_attn_fwd_packed(p, Q, K, V, weight, mask, O, lse=None, stream=None):
    """Stage 2 on the compact weights of dash_route_packed."""
    dt = _tdtype(p)
    _check(Q, "Q", (p.batch, p.n_q_heads, p.seq_len, p.head_dim), dt)
    _check(K, "K", (p.batch, p.n_kv_heads, p.seq_len, p.head_dim), dt)
    _check(V, "V", (p.batch, p.n_kv_heads, p.seq_len, p.head_dim), dt)
    _check(weight, "weight", (p.batch, p.n_kv_heads, p.seq_len, n_chunks(p)), torch.float32)
    _check(mask, "mask", (p.batch, p.n_kv_heads, p.seq_len, n_words(p)), torch.int32)
    _check(O, "O", (p.batch, p.n_q_heads, p.seq_len, p.head_dim), dt)
    if lse is not None:
        _check(lse, "lse", (p.batch, p.n_q_heads, p.seq_len), torch.float32)
    _raise("dash_attn_fwd_packed",
           lib().dash_attn_fwd_packed(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(weight),
                                      _ptr(mask), _ptr(O), _ptr(lse), _stream(stream)))


def dash_workspace_bytes(p, which):
    """Scratch bytes of dash_attn_fwd (which = 0 or False), the decode entry
    points (1 or True) or dash_attn_bwd (2)."""
    return int(lib().dash_workspace_bytes(ctypes.byref(p), int(which)))


def dash_attn_fwd(p, Q, K, V, w, mask, O, lse=None, workspace=None, stream=None):
    dt = _tdtype(p)
    _check(Q, "Q", (p.batch, p.n_q_heads, p.seq_len, p.head_dim), dt)
    _check(K, "K", (p.batch, p.n_kv_heads, p.seq_len, p.head_dim), dt)
    _check(V, "V", (p.batch, p.n_kv_heads, p.seq_len, p.head_dim), dt)
    _check(w, "w", (p.batch, p.n_kv_heads, p.seq_len, n_chunks(p)), torch.float32)
    _check(mask, "mask", (p.batch, p.n_kv_heads, p.seq_len, n_words(p)), torch.int32)
    _check(O, "O", (p.batch, p.n_q_heads, p.seq_len, p.head_dim), dt)
    if lse is not None:
        _check(lse, "lse", (p.batch, p.n_q_heads, p.seq_len), torch.float32)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _raise("dash_attn_fwd", lib().dash_attn_fwd(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(w),
                                                _ptr(mask), _ptr(O), _ptr(lse), _ptr(workspace),
                                                ws_bytes, _stream(stream)))


def dash_decode(p, q, Kc, Vc, Kbar, o, lse=None, w=None, mask=None, workspace=None, stream=None,
                cache_lens=None, page_table=None, qbar=None):
    """One decode step; with cache_lens (int32 [batch] on the device) each
    sequence has its own length and p.seq_len is the caches' capacity; with
    page_table (int32 [batch, max_pages]) as well, Kc and Vc are page pools
    [n_pages, n_kv_heads, chunk, head_dim].  p.estimate_diagonal needs qbar."""
    dt = _tdtype(p)
    L = p.seq_len
    _check(q, "q", (p.batch, p.n_q_heads, p.head_dim), dt)
    if page_table is None:
        _check(Kc, "Kcache", (p.batch, p.n_kv_heads, L, p.head_dim), dt)
        _check(Vc, "Vcache", (p.batch, p.n_kv_heads, L, p.head_dim), dt)
    else:
        if cache_lens is None:
            raise ValueError("a paged decode needs cache_lens")
        n_pages = Kc.shape[0]
        _check(Kc, "Kpool", (n_pages, p.n_kv_heads, p.chunk, p.head_dim), dt)
        _check(Vc, "Vpool", (n_pages, p.n_kv_heads, p.chunk, p.head_dim), dt)
        _check(page_table, "page_table", (p.batch, page_table.shape[1]), torch.int32)
    _check(Kbar, "Kbar", (p.batch, p.n_kv_heads, L // p.chunk, p.head_dim), dt)
    _check(o, "o", (p.batch, p.n_q_heads, p.head_dim), dt)
    if lse is not None:
        _check(lse, "lse", (p.batch, p.n_q_heads), torch.float32)
    if w is not None:
        _check(w, "w", (p.batch, p.n_kv_heads, n_chunks(p)), torch.float32)
    if mask is not None:
        _check(mask, "mask", (p.batch, p.n_kv_heads, n_words(p)), torch.int32)
    if p.estimate_diagonal:
        if qbar is None:
            raise ValueError("estimate_diagonal needs qbar")
        _check(qbar, "qbar", (p.n_kv_heads, p.head_dim), torch.float32)
    if workspace is None:
        workspace = torch.empty(dash_workspace_bytes(p, True), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    if cache_lens is None:
        _raise("dash_decode", lib().dash_decode(ctypes.byref(p), _ptr(q), _ptr(Kc), _ptr(Vc), _ptr(Kbar),
                                                _ptr(qbar), _ptr(o), _ptr(lse), _ptr(w), _ptr(mask),
                                                _ptr(workspace), ws_bytes, _stream(stream)))
        return
    _check(cache_lens, "cache_lens", (p.batch,), torch.int32)
    if page_table is not None:
        _raise("dash_decode_paged",
               lib().dash_decode_paged(ctypes.byref(p), _ptr(cache_lens), _ptr(page_table),
                                       int(page_table.shape[1]), int(Kc.shape[0]), _ptr(q), _ptr(Kc),
                                       _ptr(Vc), _ptr(Kbar), _ptr(qbar), _ptr(o), _ptr(lse), _ptr(w),
                                       _ptr(mask), _ptr(workspace), ws_bytes, _stream(stream)))
        return
    _raise("dash_decode_varlen",
           lib().dash_decode_varlen(ctypes.byref(p), _ptr(cache_lens), _ptr(q), _ptr(Kc), _ptr(Vc),
                                    _ptr(Kbar), _ptr(qbar), _ptr(o), _ptr(lse), _ptr(w), _ptr(mask),
                                    _ptr(workspace), ws_bytes, _stream(stream)))


def dash_decode_varlen(p, cache_lens, q, Kc, Vc, Kbar, o, lse=None, w=None, mask=None,
                       workspace=None, stream=None, qbar=None):
    dash_decode(p, q, Kc, Vc, Kbar, o, lse, w, mask, workspace, stream, cache_lens=cache_lens,
                qbar=qbar)


def dash_decode_paged(p, cache_lens, page_table, q, Kpool, Vpool, Kbar, o, lse=None, w=None,
                      mask=None, workspace=None, stream=None, qbar=None):
    dash_decode(p, q, Kpool, Vpool, Kbar, o, lse, w, mask, workspace, stream,
                cache_lens=cache_lens, page_table=page_table, qbar=qbar)


def dash_decode_noalloc(p, q, Kc, Vc, Kbar, o, lse=None, w=None, mask=None, stream=None):
    """dash_decode for callers that cannot allocate device memory.

    An engine that owns all GPU memory through its own pool, or a plugin API
    that forbids allocation, cannot hand dash_decode a workspace.  This call
    uses a fixed 8 MiB device array inside the library instead (held on every
    GPU that loads it).  Calls on the same device share that array: do not
    let two of them overlap on the GPU.  The first call on a device looks up
    the array's address; make it before any stream capture.
    """
    dt = _tdtype(p)
    L = p.seq_len
    _check(q, "q", (p.batch, p.n_q_heads, p.head_dim), dt)
    _check(Kc, "Kcache", (p.batch, p.n_kv_heads, L, p.head_dim), dt)
    _check(Vc, "Vcache", (p.batch, p.n_kv_heads, L, p.head_dim), dt)
    _check(Kbar, "Kbar", (p.batch, p.n_kv_heads, L // p.chunk, p.head_dim), dt)
    _check(o, "o", (p.batch, p.n_q_heads, p.head_dim), dt)
    if lse is not None:
        _check(lse, "lse", (p.batch, p.n_q_heads), torch.float32)
    if w is not None:
        _check(w, "w", (p.batch, p.n_kv_heads, n_chunks(p)), torch.float32)
    if mask is not None:
        _check(mask, "mask", (p.batch, p.n_kv_heads, n_words(p)), torch.int32)
    _raise("dash_decode_noalloc",
           lib().dash_decode_noalloc(ctypes.byref(p), _ptr(q), _ptr(Kc), _ptr(Vc), _ptr(Kbar),
                                     _ptr(o), _ptr(lse), _ptr(w), _ptr(mask), _stream(stream)))


def dash_selftest_wait_timeout(stream=None):
    """Run the library's bounded-wait timeout path once (about 2 s); the next
    dash_get_error returns DASH_ERR_TIMEOUT."""
    _raise("dash_selftest_wait_timeout", lib().dash_selftest_wait_timeout(_stream(stream)))


def dash_selftest_exp2_poly(x, y, stream=None):
    """y = the attention kernel's FMA-pipe 2^x on a float32 device tensor x."""
    _check(x, "x", (x.numel(),), torch.float32)
    _check(y, "y", (x.numel(),), torch.float32)
    _raise("dash_selftest_exp2_poly",
           lib().dash_selftest_exp2_poly(_ptr(x), _ptr(y), int(x.numel()), _stream(stream)))


def dash_selftest_bwd_split(n):
    """Force the tensor-core backward's split count (1..8; 0 = automatic) for
    later calls; returns the previous setting (a test hook)."""
    prev = int(lib().dash_selftest_bwd_split(int(n)))
    if prev < 0:
        raise ValueError(f"split count {n} outside 0..8")
    return prev


def dash_get_error(stream=None):
    """Synchronises the stream; returns (and clears) the device error status: DASH_OK,
    DASH_ERR_TIMEOUT, DASH_ERR_INVALID_ARG (a cache length out of range) or
    DASH_ERR_UNSUPPORTED."""
    return int(lib().dash_get_error(_stream(stream)))


# ----------------------------------------------------------------------------
# chained calls with freshly allocated outputs
# ----------------------------------------------------------------------------

def alloc_prefill(p, device="cuda"):
    dt = _tdtype(p)
    n_c, n_w = n_chunks(p), n_words(p)
    return {
        "Kbar": torch.empty(p.batch, p.n_kv_heads, p.seq_len // p.chunk, p.head_dim, dtype=dt, device=device),
        "w": torch.empty(p.batch, p.n_kv_heads, p.seq_len, n_c, dtype=torch.float32, device=device),
        "mask": torch.empty(p.batch, p.n_kv_heads, p.seq_len, n_w, dtype=torch.int32, device=device),
        "O": torch.empty(p.batch, p.n_q_heads, p.seq_len, p.head_dim, dtype=dt, device=device),
        "lse": torch.empty(p.batch, p.n_q_heads, p.seq_len, dtype=torch.float32, device=device),
    }


def prefill(p, Q, K, V, qbar, out=None, stream=None, with_lse=True, packed=False):
    """Stage 0 -> stage 1 -> stage 2 on the device; returns the output dict.
    With packed, stage 1 writes the compact weights (out["w"] then holds, per
    row, the routed chunks' weights in chunk order) and stage 2 reads them."""
    out = alloc_prefill(p, Q.device) if out is None else out
    dash_summarize(p, K, qbar, out["Kbar"], stream=stream)
    lse = out["lse"] if with_lse else None
    if packed:
        dash_route_packed(p, Q, out["Kbar"], out["mask"], out["w"], stream=stream, K=K, qbar=qbar)
        dash_attn_fwd_packed(p, Q, K, V, out["w"], out["mask"], out["O"], lse, stream=stream)
        return out
    dash_route(p, Q, out["Kbar"], out["w"], out["mask"], stream=stream, K=K, qbar=qbar)
    dash_attn_fwd(p, Q, K, V, out["w"], out["mask"], out["O"], lse, stream=stream)
    return out


def alloc_decode(p, device="cuda"):
    dt = _tdtype(p)
    return {
        "o": torch.empty(p.batch, p.n_q_heads, p.head_dim, dtype=dt, device=device),
        "lse": torch.empty(p.batch, p.n_q_heads, dtype=torch.float32, device=device),
        "w": torch.empty(p.batch, p.n_kv_heads, n_chunks(p), dtype=torch.float32, device=device),
        "mask": torch.empty(p.batch, p.n_kv_heads, n_words(p), dtype=torch.int32, device=device),
        "workspace": torch.empty(dash_workspace_bytes(p, True), dtype=torch.uint8, device=device),
    }


def decode(p, q, Kc, Vc, Kbar, out=None, stream=None, cache_lens=None, page_table=None,
           qbar=None):
    out = alloc_decode(p, q.device) if out is None else out
    dash_decode(p, q, Kc, Vc, Kbar, out["o"], out["lse"], out["w"], out["mask"], out["workspace"],
                stream=stream, cache_lens=cache_lens, page_table=page_table, qbar=qbar)
    return out
