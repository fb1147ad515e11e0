"""ctypes binding of libdash_b200.so (include/dash.h).

Argument marshalling only: every step of the forward pass runs in the library's CUDA kernels.
PyTorch supplies device memory and streams.  There is no fallback: if the shared library is
missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdash_b200.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "dash.h")

DASH_OK, DASH_EINVAL, DASH_EUNSUPPORTED, DASH_EWORKSPACE, DASH_EALIGN, DASH_ELAUNCH = 0, -1, -2, -3, -4, -5
DASH_F32, DASH_BF16 = 0, 1
DASH_OP_PREFILL, DASH_OP_DECODE, DASH_OP_BACKWARD = 0, 1, 2
DASH_STAGE0, DASH_STAGE1, DASH_STAGE2, DASH_STAGE2_BITMASK = 0, 1, 2, 3


class dash_params(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("seqlen", ctypes.c_int), ("h_q", ctypes.c_int),
                ("h_kv", ctypes.c_int), ("d_h", ctypes.c_int), ("chunk", ctypes.c_int),
                ("alpha", ctypes.c_float), ("gamma", ctypes.c_float), ("inv_sigma", ctypes.c_float),
                ("dtype", ctypes.c_int),
                ("q_strides", ctypes.c_longlong * 3), ("k_strides", ctypes.c_longlong * 3),
                ("v_strides", ctypes.c_longlong * 3), ("o_strides", ctypes.c_longlong * 3)]


class dash_route_out(ctypes.Structure):
    _fields_ = [("counts", ctypes.c_void_p), ("chunk_idx", ctypes.c_void_p),
                ("bias", ctypes.c_void_p), ("bitmask", ctypes.c_void_p)]


class dash_paged_kv(ctypes.Structure):
    _fields_ = [("page_table", ctypes.c_void_p), ("max_pages", ctypes.c_int), ("page_size", ctypes.c_int),
                ("num_pages", ctypes.c_int), ("k_page_stride", ctypes.c_longlong),
                ("v_page_stride", ctypes.c_longlong)]


class DashError(RuntimeError):
    pass


_lib = None


def load():
    """Load the library (raises when it is missing: there is no CPU path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise DashError(f"{LIB_PATH} is missing; build it with adaptive_sparse_hierarchical_b200.build.build()")
        lib = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(dash_params)
        R = ctypes.POINTER(dash_route_out)
        vp, sz = ctypes.c_void_p, ctypes.c_size_t
        lib.dash_workspace_size.argtypes = [P, ctypes.c_int]
        lib.dash_workspace_size.restype = sz
        lib.dash_error_word_offset.argtypes = [P, ctypes.c_int]
        lib.dash_error_word_offset.restype = ctypes.c_longlong
        lib.dash_prefill_order_offset.argtypes = [P]
        lib.dash_prefill_order_offset.restype = ctypes.c_longlong
        lib.dash_route_capacity.argtypes = [P]
        lib.dash_route_capacity.restype = ctypes.c_longlong
        lib.dash_prefill.argtypes = [P, vp, vp, vp, vp, vp, vp, R, vp, sz, vp]
        lib.dash_prefill.restype = ctypes.c_int
        lib.dash_prefill_stage.argtypes = [P, ctypes.c_int, vp, vp, vp, vp, vp, vp, R, vp, sz, vp]
        lib.dash_prefill_stage.restype = ctypes.c_int
        lib.dash_summary_build.argtypes = [P, vp, vp, vp, vp, vp, vp]
        lib.dash_summary_build.restype = ctypes.c_int
        lib.dash_summary_append.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        lib.dash_summary_append.restype = ctypes.c_int
        lib.dash_decode.argtypes = [P, vp, vp, vp, vp, vp, vp, R, vp, sz, vp]
        lib.dash_decode.restype = ctypes.c_int
        PK = ctypes.POINTER(dash_paged_kv)
        lib.dash_summary_build_paged.argtypes = [P, PK, vp, vp, vp, vp, vp, vp]
        lib.dash_summary_build_paged.restype = ctypes.c_int
        lib.dash_summary_append_paged.argtypes = [P, PK, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        lib.dash_summary_append_paged.restype = ctypes.c_int
        lib.dash_decode_paged.argtypes = [P, PK, vp, vp, vp, vp, vp, vp, R, vp, sz, vp]
        lib.dash_decode_paged.restype = ctypes.c_int
        lib.dash_backward.argtypes = [P, vp, vp, vp, vp, vp, vp, R, vp, vp, vp, vp, vp, sz, vp]
        lib.dash_backward.restype = ctypes.c_int
        lib.dash_status_string.argtypes = [ctypes.c_int]
        lib.dash_status_string.restype = ctypes.c_char_p
        lib.dash_set_wait_limit.argtypes = [ctypes.c_longlong]
        lib.dash_set_wait_limit.restype = ctypes.c_longlong
        _lib = lib
    return _lib


def header_symbols():
    """Entry points declared in include/dash.h."""
    with open(HEADER) as fh:
        text = fh.read()
    return sorted(set(re.findall(r"^\s*(?:size_t|int|long long|const char\*)\s+(dash_\w+)\s*\(", text, re.M)))


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, what: str):
    if rc != DASH_OK:
        raise DashError(f"{what}: {load().dash_status_string(rc).decode()} ({rc})")


def params(*, batch, seqlen, h_q, h_kv, d_h, chunk, alpha, gamma, inv_sigma=1.0, dtype=DASH_BF16,
           q_strides=(0, 0, 0), k_strides=(0, 0, 0), v_strides=(0, 0, 0), o_strides=(0, 0, 0)):
    p = dash_params()
    p.batch, p.seqlen, p.h_q, p.h_kv, p.d_h, p.chunk = batch, seqlen, h_q, h_kv, d_h, chunk
    p.alpha, p.gamma, p.inv_sigma, p.dtype = alpha, gamma, inv_sigma, dtype
    for name, st in (("q_strides", q_strides), ("k_strides", k_strides), ("v_strides", v_strides),
                     ("o_strides", o_strides)):
        getattr(p, name)[:] = [int(x) for x in st[:3]]
    return p


def route_out(counts=None, chunk_idx=None, bias=None, bitmask=None):
    return dash_route_out(_ptr(counts), _ptr(chunk_idx), _ptr(bias), _ptr(bitmask))


def dash_workspace_size(p: dash_params, op: int) -> int:
    return int(load().dash_workspace_size(ctypes.byref(p), op))


def dash_error_word_offset(p: dash_params, op: int) -> int:
    return int(load().dash_error_word_offset(ctypes.byref(p), op))


def dash_prefill_order_offset(p: dash_params) -> int:
    return int(load().dash_prefill_order_offset(ctypes.byref(p)))


def dash_route_capacity(p: dash_params) -> int:
    return int(load().dash_route_capacity(ctypes.byref(p)))


def dash_status_string(rc: int) -> str:
    return load().dash_status_string(rc).decode()


def dash_set_wait_limit(polls: int) -> int:
    """Poll limit of the tensor-core Stage 2 kernels' bounded waits for later launches (a
    diagnostic knob; 0 makes the first wait give up).  Returns the previous limit."""
    return int(load().dash_set_wait_limit(int(polls)))


def dash_prefill(p, Q, K, V, qbar, O, kbar_out=None, route=None, workspace=None, ws_bytes=None,
                 stream=None, check=True) -> int:
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None and workspace is not None else (ws_bytes or 0)
    rc = load().dash_prefill(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(qbar), _ptr(O), _ptr(kbar_out),
                             ctypes.byref(route) if route is not None else None, _ptr(workspace), ws_bytes,
                             _stream(stream) if check or stream is not None else None)
    if check:
        _check(rc, "dash_prefill")
    return rc


def dash_prefill_stage(p, stage, Q, K, V, qbar, O, kbar_out=None, route=None, workspace=None, ws_bytes=None,
                       stream=None) -> int:
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None and workspace is not None else (ws_bytes or 0)
    rc = load().dash_prefill_stage(ctypes.byref(p), int(stage), _ptr(Q), _ptr(K), _ptr(V), _ptr(qbar), _ptr(O),
                                   _ptr(kbar_out), ctypes.byref(route) if route is not None else None,
                                   _ptr(workspace), ws_bytes, _stream(stream))
    _check(rc, "dash_prefill_stage")
    return rc


def dash_summary_build(p, K_cache, qbar, seqlens, kbar_cache, partial_state, stream=None) -> int:
    rc = load().dash_summary_build(ctypes.byref(p), _ptr(K_cache), _ptr(qbar), _ptr(seqlens), _ptr(kbar_cache),
                                   _ptr(partial_state), _stream(stream))
    _check(rc, "dash_summary_build")
    return rc


def dash_summary_append(p, k_new, v_new, qbar, K_cache, V_cache, kbar_cache, partial_state, seqlens,
                        stream=None) -> int:
    rc = load().dash_summary_append(ctypes.byref(p), _ptr(k_new), _ptr(v_new), _ptr(qbar), _ptr(K_cache),
                                    _ptr(V_cache), _ptr(kbar_cache), _ptr(partial_state), _ptr(seqlens),
                                    _stream(stream))
    _check(rc, "dash_summary_append")
    return rc


def dash_decode(p, q, K_cache, V_cache, kbar_cache, seqlens, O, route=None, workspace=None, ws_bytes=None,
                stream=None) -> int:
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None and workspace is not None else (ws_bytes or 0)
    rc = load().dash_decode(ctypes.byref(p), _ptr(q), _ptr(K_cache), _ptr(V_cache), _ptr(kbar_cache),
                            _ptr(seqlens), _ptr(O), ctypes.byref(route) if route is not None else None,
                            _ptr(workspace), ws_bytes, _stream(stream))
    _check(rc, "dash_decode")
    return rc


def paged_kv(page_table, page_size, num_pages, k_page_stride, v_page_stride):
    """Page description of paged K/V pools (page_table: device int32 [batch, max_pages])."""
    return dash_paged_kv(_ptr(page_table), int(page_table.shape[1]), int(page_size), int(num_pages),
                         int(k_page_stride), int(v_page_stride))


def dash_summary_build_paged(p, pk, K_pool, qbar, seqlens, kbar_cache, partial_state, stream=None) -> int:
    rc = load().dash_summary_build_paged(ctypes.byref(p), ctypes.byref(pk), _ptr(K_pool), _ptr(qbar), _ptr(seqlens),
                                         _ptr(kbar_cache), _ptr(partial_state), _stream(stream))
    _check(rc, "dash_summary_build_paged")
    return rc


def dash_summary_append_paged(p, pk, k_new, v_new, qbar, K_pool, V_pool, kbar_cache, partial_state, seqlens,
                              stream=None) -> int:
    rc = load().dash_summary_append_paged(ctypes.byref(p), ctypes.byref(pk), _ptr(k_new), _ptr(v_new), _ptr(qbar),
                                          _ptr(K_pool), _ptr(V_pool), _ptr(kbar_cache), _ptr(partial_state),
                                          _ptr(seqlens), _stream(stream))
    _check(rc, "dash_summary_append_paged")
    return rc


def dash_decode_paged(p, pk, q, K_pool, V_pool, kbar_cache, seqlens, O, route=None, workspace=None, ws_bytes=None,
                      stream=None) -> int:
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None and workspace is not None else (ws_bytes or 0)
    rc = load().dash_decode_paged(ctypes.byref(p), ctypes.byref(pk), _ptr(q), _ptr(K_pool), _ptr(V_pool),
                                  _ptr(kbar_cache), _ptr(seqlens), _ptr(O),
                                  ctypes.byref(route) if route is not None else None, _ptr(workspace), ws_bytes,
                                  _stream(stream))
    _check(rc, "dash_decode_paged")
    return rc


def dash_backward(p, Q, K, V, qbar, dO, kbar, route, dQ, dK, dV, dqbar, workspace=None, ws_bytes=None,
                  stream=None) -> int:
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None and workspace is not None else (ws_bytes or 0)
    rc = load().dash_backward(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(qbar), _ptr(dO), _ptr(kbar),
                              ctypes.byref(route) if route is not None else None, _ptr(dQ), _ptr(dK), _ptr(dV),
                              _ptr(dqbar), _ptr(workspace), ws_bytes, _stream(stream))
    _check(rc, "dash_backward")
    return rc
