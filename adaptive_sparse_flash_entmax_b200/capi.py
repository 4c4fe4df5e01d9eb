"""ctypes binding of libentattn.so: the C ABI of include/entattn.h, same names.

Each function here marshals arguments only; every step of the computation
runs in the CUDA library.  The library is loaded on first use and a missing
or unbuildable library raises immediately: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libentattn.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "entattn.h")

ENT_OK, ENT_EINVAL, ENT_EUNSUPPORTED, ENT_ECUDA, ENT_ETIMEOUT = 0, 1, 2, 3, 4
ENT_F32, ENT_BF16 = 0, 1
ENT_SOLVE_HIST, ENT_SOLVE_HALLEY, ENT_SOLVE_BISECT = 0, 1, 2
STATUS_NAMES = {0: "ENT_OK", 1: "ENT_EINVAL", 2: "ENT_EUNSUPPORTED", 3: "ENT_ECUDA",
                4: "ENT_ETIMEOUT"}


class EntAttnError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load (once) and return the CUDA library; raises if it is not built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is not built; run `python -m adaptive_sparse_flash_entmax_b200.build` "
            "(the attention ops have no non-CUDA fallback)")
    lib = ctypes.CDLL(path)
    vp, sz, ci, cf = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
    lib.ent_attn_block_size.argtypes = []
    lib.ent_attn_block_size.restype = ci
    for fn in (lib.ent_attn_fwd_workspace_size, lib.ent_attn_bwd_workspace_size):
        fn.argtypes = [ci, ci, ci, ci, ci]
        fn.restype = sz
    lib.ent_attn_fwd.argtypes = [vp, vp, vp, ci, ci, ci, ci, ci, cf, ci, vp, vp, vp, vp, vp, sz, vp]
    lib.ent_attn_fwd.restype = ci
    lib.ent_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, ci, vp, vp,
                                 vp, vp, sz, vp]
    lib.ent_attn_bwd.restype = ci
    lib.ent_attn_fwd_otilde.argtypes = [vp, vp, vp, ci, ci, ci, ci, ci, cf, ci, vp, vp, vp, vp, vp,
                                        vp, sz, vp]
    lib.ent_attn_fwd_otilde.restype = ci
    lib.ent_attn_bwd_otilde.argtypes = [vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, ci, vp,
                                        vp, vp, vp, sz, vp]
    lib.ent_attn_bwd_otilde.restype = ci
    lib.ent_attn_read_status.argtypes = [vp, ctypes.POINTER(ctypes.c_longlong), vp]
    lib.ent_attn_read_status.restype = ci
    lib.ent_attn_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, ci,
                                         vp, vp, vp, vp]
    lib.ent_attn_bwd_noalloc.restype = ci
    lib.ent_attn_noalloc_read_status.argtypes = [ctypes.POINTER(ctypes.c_longlong), vp]
    lib.ent_attn_noalloc_read_status.restype = ci
    lib.ent_attn_list_cap.argtypes = []
    lib.ent_attn_list_cap.restype = ci
    lib.ent_attn_bwd_lists_workspace_size.argtypes = [ci, ci, ci, ci, ci]
    lib.ent_attn_bwd_lists_workspace_size.restype = sz
    lib.ent_attn_fwd_lists.argtypes = [vp, vp, vp, ci, ci, ci, ci, ci, cf, ci, vp, vp, vp, vp, vp,
                                       vp, vp, vp, sz, vp]
    lib.ent_attn_fwd_lists.restype = ci
    lib.ent_attn_bwd_lists.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf,
                                       ci, vp, vp, vp, vp, sz, vp]
    lib.ent_attn_bwd_lists.restype = ci
    lib.ent_attn_last_error.argtypes = []
    lib.ent_attn_last_error.restype = ctypes.c_char_p
    lib.ent_entmax_rows_max_n.argtypes = []
    lib.ent_entmax_rows_max_n.restype = ci
    lib.ent_entmax_rows_fwd.argtypes = [vp, ci, ci, ci, cf, ci, vp, vp, vp, vp]
    lib.ent_entmax_rows_fwd.restype = ci
    lib.ent_entmax_rows_bwd.argtypes = [vp, vp, vp, ci, ci, ci, cf, vp, vp]
    lib.ent_entmax_rows_bwd.restype = ci
    _lib = lib
    return lib


def header_symbols(header: str = HEADER) -> list[str]:
    """Names of the functions include/entattn.h declares."""
    text = open(header).read()
    return sorted(set(re.findall(r"^\s*(?:[\w\s\*]+?)\b(ent_(?:attn|entmax)_\w+)\s*\(", text, re.M)))


def ent_attn_block_size() -> int:
    return load().ent_attn_block_size()


def ent_attn_fwd_workspace_size(B, H, N, d, dtype) -> int:
    return load().ent_attn_fwd_workspace_size(B, H, N, d, dtype)


def ent_attn_bwd_workspace_size(B, H, N, d, dtype) -> int:
    return load().ent_attn_bwd_workspace_size(B, H, N, d, dtype)


def ent_attn_last_error() -> str:
    return load().ent_attn_last_error().decode()


def ent_attn_fwd(q, k, v, B, H, N, d, dtype, alpha, causal, o, tau, block_mask, iters, ws,
                 ws_bytes, stream) -> int:
    """Raw call with integer device pointers; returns the ent_status code."""
    return load().ent_attn_fwd(q, k, v, B, H, N, d, dtype, float(alpha), int(causal), o, tau,
                               block_mask, iters, ws, ws_bytes, stream)


def ent_attn_bwd(q, k, v, o, dout, tau, block_mask, B, H, N, d, dtype, alpha, causal, dq, dk,
                 dv, ws, ws_bytes, stream) -> int:
    return load().ent_attn_bwd(q, k, v, o, dout, tau, block_mask, B, H, N, d, dtype,
                               float(alpha), int(causal), dq, dk, dv, ws, ws_bytes, stream)


def ent_attn_fwd_otilde(q, k, v, B, H, N, d, dtype, alpha, causal, o, tau, block_mask, iters,
                        otilde, ws, ws_bytes, stream) -> int:
    return load().ent_attn_fwd_otilde(q, k, v, B, H, N, d, dtype, float(alpha), int(causal), o,
                                      tau, block_mask, iters, otilde, ws, ws_bytes, stream)


def ent_attn_bwd_otilde(q, k, v, otilde, dout, tau, block_mask, B, H, N, d, dtype, alpha, causal,
                        dq, dk, dv, ws, ws_bytes, stream) -> int:
    return load().ent_attn_bwd_otilde(q, k, v, otilde, dout, tau, block_mask, B, H, N, d, dtype,
                                      float(alpha), int(causal), dq, dk, dv, ws, ws_bytes, stream)


def ent_entmax_rows_max_n() -> int:
    return load().ent_entmax_rows_max_n()


def ent_entmax_rows_fwd(z, rows, n, dtype, alpha, method, p, tau, iters, stream) -> int:
    return load().ent_entmax_rows_fwd(z, rows, n, dtype, float(alpha), int(method), p, tau, iters,
                                      stream)


def ent_entmax_rows_bwd(z, tau, dp, rows, n, dtype, alpha, dz, stream) -> int:
    return load().ent_entmax_rows_bwd(z, tau, dp, rows, n, dtype, float(alpha), dz, stream)


def ent_attn_read_status(ws, stream) -> tuple[int, list[int]]:
    """(status, counters[8]) of a workspace; synchronises the stream."""
    arr = (ctypes.c_longlong * 8)()
    st = load().ent_attn_read_status(ws, arr, stream)
    return st, list(arr)


def ent_attn_bwd_noalloc(q, k, v, o, dout, tau, block_mask, B, H, N, d, dtype, alpha, causal,
                         dq, dk, dv, stream) -> int:
    return load().ent_attn_bwd_noalloc(q, k, v, o, dout, tau, block_mask, B, H, N, d, dtype,
                                       float(alpha), int(causal), dq, dk, dv, stream)


def ent_attn_noalloc_read_status(stream) -> tuple[int, list[int]]:
    """(status, counters[8]) of the last ent_attn_bwd_noalloc call on the current device."""
    arr = (ctypes.c_longlong * 8)()
    st = load().ent_attn_noalloc_read_status(arr, stream)
    return st, list(arr)


def ent_attn_list_cap() -> int:
    return load().ent_attn_list_cap()


def ent_attn_bwd_lists_workspace_size(B, H, N, d, dtype) -> int:
    return load().ent_attn_bwd_lists_workspace_size(B, H, N, d, dtype)


def ent_attn_fwd_lists(q, k, v, B, H, N, d, dtype, alpha, causal, o, tau, block_mask, iters,
                       list_key, list_u, list_n, ws, ws_bytes, stream) -> int:
    return load().ent_attn_fwd_lists(q, k, v, B, H, N, d, dtype, float(alpha), int(causal), o,
                                     tau, block_mask, iters, list_key, list_u, list_n, ws,
                                     ws_bytes, stream)


def ent_attn_bwd_lists(q, k, v, list_key, list_u, list_n, dout, tau, block_mask, B, H, N, d,
                       dtype, alpha, causal, dq, dk, dv, ws, ws_bytes, stream) -> int:
    return load().ent_attn_bwd_lists(q, k, v, list_key, list_u, list_n, dout, tau, block_mask, B,
                                     H, N, d, dtype, float(alpha), int(causal), dq, dk, dv, ws,
                                     ws_bytes, stream)
