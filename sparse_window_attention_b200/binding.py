"""ctypes binding of libbasa (include/basa.h): argument marshalling only.

Every function here converts its arguments (torch tensors -> device pointers,
the current CUDA stream -> cudaStream_t, a parameter dict -> basa_params) and
calls the C entry point of the same name; all computation runs in the CUDA
kernels behind it. A missing library raises at import time: there is no
fallback path.
"""
from __future__ import annotations

import ctypes
import os

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libbasa.so")

BASA_OK = 0
STATUS_NAMES = {
    0: "BASA_OK",
    1: "BASA_ERR_INVALID_ARG",
    2: "BASA_ERR_SHAPE",
    3: "BASA_ERR_UNSUPPORTED",
    4: "BASA_ERR_CUDA",
    5: "BASA_ERR_DEVICE_TIMEOUT",
    6: "BASA_ERR_BAD_INDEX",
}
BASA_BF16 = 0
BASA_F32 = 1
BASA_FLAG_TEST_SKIP_FIRST_KEY_LOAD = 0x1
BASA_DEVERR_BAD_ROUTE = 0x8
BASA_KEYS_WINDOWS, BASA_KEYS_POOLED, BASA_KEYS_TEXT, BASA_KEYS_ALL = 1, 2, 4, 7
BASA_MAX_BRANCHES = 4
EXPORTED = (
    "basa_pool_kv",
    "basa_route_workspace_bytes",
    "basa_route_windows",
    "basa_route_windows_noalloc",
    "basa_pool_route_workspace_bytes",
    "basa_pool_route",
    "basa_window_attn_fwd",
    "basa_window_attn_fwd_lse",
    "basa_merge_branches",
    "basa_text_attn_workspace_bytes",
    "basa_text_attn_fwd",
    "basa_window_attn_bwd_workspace_bytes",
    "basa_window_attn_bwd",
    "basa_status_string",
    "basa_device_error_status",
)


class BasaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


class basa_params(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("heads", ctypes.c_int), ("head_dim", ctypes.c_int),
        ("T", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
        ("wt", ctypes.c_int), ("wh", ctypes.c_int), ("ww", ctypes.c_int),
        ("st", ctypes.c_int), ("sy", ctypes.c_int), ("sx", ctypes.c_int),
        ("pt", ctypes.c_int), ("ph", ctypes.c_int), ("pw", ctypes.c_int),
        ("n_text", ctypes.c_int), ("routed_k", ctypes.c_int),
        ("dtype", ctypes.c_int),
        ("dev_err", ctypes.c_void_p),
        ("flags", ctypes.c_uint32),
        ("wait_timeout_us", ctypes.c_uint32),
        ("route_radius", ctypes.c_int),
    ]


def load_library(path: str = _LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"libbasa.so not built at {path}: run `python -m sparse_window_attention_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(basa_params)
    vp = ctypes.c_void_p
    lib.basa_pool_kv.argtypes = [vp, vp, vp, vp, P, vp]
    lib.basa_pool_kv.restype = ctypes.c_int
    lib.basa_route_workspace_bytes.argtypes = [P]
    lib.basa_route_workspace_bytes.restype = ctypes.c_size_t
    lib.basa_route_windows.argtypes = [vp, vp, vp, vp, vp, P, vp]
    lib.basa_route_windows.restype = ctypes.c_int
    lib.basa_route_windows_noalloc.argtypes = [vp, vp, vp, vp, P, vp]
    lib.basa_route_windows_noalloc.restype = ctypes.c_int
    lib.basa_pool_route_workspace_bytes.argtypes = [P]
    lib.basa_pool_route_workspace_bytes.restype = ctypes.c_size_t
    lib.basa_pool_route.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, P, vp]
    lib.basa_pool_route.restype = ctypes.c_int
    lib.basa_window_attn_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, P, vp]
    lib.basa_window_attn_fwd.restype = ctypes.c_int
    lib.basa_window_attn_fwd_lse.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_uint32, P, vp]
    lib.basa_window_attn_fwd_lse.restype = ctypes.c_int
    lib.basa_merge_branches.argtypes = [ctypes.c_int, ctypes.POINTER(vp), ctypes.POINTER(vp), vp, vp, P, vp]
    lib.basa_merge_branches.restype = ctypes.c_int
    lib.basa_text_attn_workspace_bytes.argtypes = [P]
    lib.basa_text_attn_workspace_bytes.restype = ctypes.c_size_t
    lib.basa_text_attn_fwd.argtypes = [vp, vp, vp, vp, vp, P, vp]
    lib.basa_text_attn_fwd.restype = ctypes.c_int
    lib.basa_window_attn_bwd_workspace_bytes.argtypes = [P]
    lib.basa_window_attn_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.basa_window_attn_bwd.argtypes = [vp] * 13 + [P, vp]
    lib.basa_window_attn_bwd.restype = ctypes.c_int
    lib.basa_status_string.argtypes = [ctypes.c_int]
    lib.basa_status_string.restype = ctypes.c_char_p
    lib.basa_device_error_status.argtypes = [ctypes.c_int32]
    lib.basa_device_error_status.restype = ctypes.c_int
    return lib


_lib = load_library()


def make_params(B, heads, head_dim, grid, window, shift=(0, 0, 0), pool=(0, 0, 0), n_text=0, routed_k=0,
                dtype="bf16", dev_err=None, flags=0, wait_timeout_us=0, route_radius=0) -> basa_params:
    p = basa_params()
    p.B, p.heads, p.head_dim = B, heads, head_dim
    p.T, p.H, p.W = grid
    p.wt, p.wh, p.ww = window
    p.st, p.sy, p.sx = shift
    p.pt, p.ph, p.pw = pool
    p.n_text, p.routed_k = n_text, routed_k
    p.dtype = BASA_BF16 if dtype in ("bf16", BASA_BF16) else BASA_F32
    p.dev_err = _ptr(dev_err)
    p.flags = flags
    p.wait_timeout_us = wait_timeout_us
    p.route_radius = route_radius
    return p


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    return stream if isinstance(stream, int) else stream.cuda_stream


def _check(status: int, where: str):
    if status != BASA_OK:
        raise BasaError(status, where)


def basa_status_string(status: int) -> str:
    return _lib.basa_status_string(status).decode()


def basa_device_error_status(word: int) -> int:
    return _lib.basa_device_error_status(word)


def basa_route_workspace_bytes(params: basa_params) -> int:
    return _lib.basa_route_workspace_bytes(ctypes.byref(params))


def basa_pool_kv(k, v, kp, vp, params: basa_params, stream=None, check=True) -> int:
    st = _lib.basa_pool_kv(_ptr(k), _ptr(v), _ptr(kp), _ptr(vp), ctypes.byref(params), _stream(stream))
    if check:
        _check(st, "basa_pool_kv")
    return st


def basa_route_windows(q, k, route_idx, route_score, workspace, params: basa_params, stream=None, check=True) -> int:
    st = _lib.basa_route_windows(_ptr(q), _ptr(k), _ptr(route_idx), _ptr(route_score), _ptr(workspace),
                                 ctypes.byref(params), _stream(stream))
    if check:
        _check(st, "basa_route_windows")
    return st


def basa_route_windows_noalloc(q, k, route_idx, route_score, params: basa_params, stream=None, check=True) -> int:
    """basa_route_windows without a workspace argument (uses the library's fixed
    device scratch; see include/basa.h for its limits)."""
    st = _lib.basa_route_windows_noalloc(_ptr(q), _ptr(k), _ptr(route_idx), _ptr(route_score),
                                         ctypes.byref(params), _stream(stream))
    if check:
        _check(st, "basa_route_windows_noalloc")
    return st


def basa_pool_route_workspace_bytes(params: basa_params) -> int:
    return _lib.basa_pool_route_workspace_bytes(ctypes.byref(params))


def basa_pool_route(q, k, v, kp, vp, route_idx, route_score, workspace, params: basa_params, stream=None,
                    check=True) -> int:
    st = _lib.basa_pool_route(_ptr(q), _ptr(k), _ptr(v), _ptr(kp), _ptr(vp), _ptr(route_idx), _ptr(route_score),
                              _ptr(workspace), ctypes.byref(params), _stream(stream))
    if check:
        _check(st, "basa_pool_route")
    return st


def basa_window_attn_fwd(q, k, v, kp, vp, route_idx, out, params: basa_params, stream=None, check=True) -> int:
    st = _lib.basa_window_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(kp), _ptr(vp), _ptr(route_idx), _ptr(out),
                                   ctypes.byref(params), _stream(stream))
    if check:
        _check(st, "basa_window_attn_fwd")
    return st


def basa_window_attn_fwd_lse(q, k, v, kp, vp, route_idx, out, lse, keys: int, params: basa_params, stream=None,
                             check=True) -> int:
    st = _lib.basa_window_attn_fwd_lse(_ptr(q), _ptr(k), _ptr(v), _ptr(kp), _ptr(vp), _ptr(route_idx), _ptr(out),
                                       _ptr(lse), keys, ctypes.byref(params), _stream(stream))
    if check:
        _check(st, "basa_window_attn_fwd_lse")
    return st


def basa_merge_branches(outs, lses, out, lse, params: basa_params, stream=None, check=True) -> int:
    n = len(outs)
    arr_o = (ctypes.c_void_p * max(n, 1))(*[_ptr(x) for x in outs])
    arr_l = (ctypes.c_void_p * max(n, 1))(*[_ptr(x) for x in lses])
    st = _lib.basa_merge_branches(n, arr_o, arr_l, _ptr(out), _ptr(lse), ctypes.byref(params), _stream(stream))
    if check:
        _check(st, "basa_merge_branches")
    return st


def basa_text_attn_workspace_bytes(params: basa_params) -> int:
    return _lib.basa_text_attn_workspace_bytes(ctypes.byref(params))


def basa_text_attn_fwd(q_text, k, v, out_text, workspace, params: basa_params, stream=None, check=True) -> int:
    st = _lib.basa_text_attn_fwd(_ptr(q_text), _ptr(k), _ptr(v), _ptr(out_text), _ptr(workspace),
                                 ctypes.byref(params), _stream(stream))
    if check:
        _check(st, "basa_text_attn_fwd")
    return st


def basa_window_attn_bwd_workspace_bytes(params: basa_params) -> int:
    return _lib.basa_window_attn_bwd_workspace_bytes(ctypes.byref(params))


def basa_window_attn_bwd(q, k, v, kp, vp, route_idx, out, lse, dout, dq, dk, dv, workspace, params: basa_params,
                         stream=None, check=True) -> int:
    st = _lib.basa_window_attn_bwd(*[_ptr(x) for x in (q, k, v, kp, vp, route_idx, out, lse, dout, dq, dk, dv,
                                                        workspace)], ctypes.byref(params), _stream(stream))
    if check:
        _check(st, "basa_window_attn_bwd")
    return st
