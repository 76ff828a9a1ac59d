"""ctypes view of libwkv.so: the types and signatures of include/wkv.h.

Argument marshalling only; every step of the operator runs in the library's
CUDA kernels. Loading fails loudly if the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# WKV_LIBRARY=debug selects the bounds-checked build (libwkv_debug.so)
LIB_PATH = os.path.join(HERE, "_build", "libwkv_debug.so" if os.environ.get("WKV_LIBRARY") == "debug"
                        else "libwkv.so")

WKV_OK = 0
WKV_ERR_INVALID_ARG = 1
WKV_ERR_UNSUPPORTED_DTYPE = 2
WKV_ERR_MISALIGNED = 3
WKV_ERR_WORKSPACE_TOO_SMALL = 4
WKV_ERR_CUDA = 5
WKV_ERR_WAIT_TIMEOUT = 6
WKV_ERR_BOUNDS = 7

WKV_F32 = 0
WKV_BF16 = 1

# entry points declared in include/wkv.h
EXPORTS = ("wkv_forward_workspace_size", "wkv_forward_kernel", "wkv_forward_launches", "wkv_forward",
           "wkv_forward_ext", "wkv_step", "wkv_step_ext", "wkv_query_status", "wkv_status_string", "wkv_version",
           "wkv_forward_noalloc", "wkv_last_cuda_error", "wkv_backward_workspace_size", "wkv_backward",
           "wkv_v6_forward", "wkv_forward_host_buffer_size", "wkv_forward_host")

# size of the library's built-in scratch array used by wkv_forward_noalloc
NOALLOC_SCRATCH_BYTES = 16 << 20


class wkv_cstate(ctypes.Structure):
    _fields_ = [("num", ctypes.c_void_p), ("den", ctypes.c_void_p), ("max_e", ctypes.c_void_p)]


class wkv_state(ctypes.Structure):
    _fields_ = [("num", ctypes.c_void_p), ("den", ctypes.c_void_p), ("max_e", ctypes.c_void_p)]


class wkv_options(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_int32), ("chunk_len", ctypes.c_int32),
                ("lookback_group", ctypes.c_int32), ("inject_enable", ctypes.c_int32),
                ("wait_timeout_ns", ctypes.c_int64), ("inject_unpublished_tile", ctypes.c_int64),
                ("span", ctypes.c_int32), ("seq_threads", ctypes.c_int32),
                ("scan_segments", ctypes.c_int32), ("stages", ctypes.c_int32),
                ("seq_vec", ctypes.c_int32), ("replay_chunks", ctypes.c_int32),
                ("cta_warps", ctypes.c_int32)]


class wkv_ext(ctypes.Structure):
    _fields_ = [("w_t", ctypes.c_void_p), ("r", ctypes.c_void_p)]


class WkvError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = f"{where}: {status_string(code)} (status {code})"
        if code == WKV_ERR_CUDA:
            msg += f", last CUDA error {lib().wkv_last_cuda_error().decode()}"
        super().__init__(msg)


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it is missing (no fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libwkv.so is not built ({LIB_PATH}); run python -m wkv_recurrence_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, SZ, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
        L.wkv_forward_workspace_size.argtypes = [I64, I64, I64, ctypes.POINTER(wkv_options)]
        L.wkv_forward_workspace_size.restype = SZ
        L.wkv_forward_kernel.argtypes = [I64, I64, I64, I, ctypes.POINTER(wkv_options)]
        L.wkv_forward_kernel.restype = ctypes.c_int32
        L.wkv_forward_launches.argtypes = [I64, I64, I64, I, ctypes.POINTER(wkv_options)]
        L.wkv_forward_launches.restype = ctypes.c_int32
        L.wkv_forward.argtypes = [I64, I64, I64, P, P, I, P, P, P, I,
                                  ctypes.POINTER(wkv_cstate), ctypes.POINTER(wkv_state),
                                  P, SZ, P, ctypes.POINTER(wkv_options)]
        L.wkv_forward.restype = I
        L.wkv_step.argtypes = [I64, I64, P, P, I, P, P, P, I,
                               ctypes.POINTER(wkv_cstate), ctypes.POINTER(wkv_state), P]
        L.wkv_step.restype = I
        L.wkv_forward_ext.argtypes = [I64, I64, I64, P, P, I, P, P, P, I,
                                      ctypes.POINTER(wkv_cstate), ctypes.POINTER(wkv_state),
                                      P, SZ, P, ctypes.POINTER(wkv_options), ctypes.POINTER(wkv_ext)]
        L.wkv_forward_ext.restype = I
        L.wkv_step_ext.argtypes = [I64, I64, P, P, I, P, P, P, I,
                                   ctypes.POINTER(wkv_cstate), ctypes.POINTER(wkv_state), P,
                                   ctypes.POINTER(wkv_ext)]
        L.wkv_step_ext.restype = I
        L.wkv_forward_noalloc.argtypes = [I64, I64, I64, P, P, I, P, P, P, I,
                                          ctypes.POINTER(wkv_cstate), ctypes.POINTER(wkv_state), P]
        L.wkv_forward_noalloc.restype = I
        L.wkv_forward_host_buffer_size.argtypes = [I64, I64, I64, I, I, I64]
        L.wkv_forward_host_buffer_size.restype = SZ
        L.wkv_forward_host.argtypes = [I64, I64, I64, P, P, I, P, P, P, I,
                                       ctypes.POINTER(wkv_cstate), ctypes.POINTER(wkv_state), P, SZ, I64, P]
        L.wkv_forward_host.restype = I
        L.wkv_backward_workspace_size.argtypes = [I64, I64, I64]
        L.wkv_backward_workspace_size.restype = SZ
        L.wkv_backward.argtypes = [I64, I64, I64, P, P, I, P, P, ctypes.POINTER(wkv_cstate), P,
                                   P, P, P, P, ctypes.POINTER(wkv_state), P, SZ, P]
        L.wkv_backward.restype = I
        L.wkv_v6_forward.argtypes = [I64, I64, I64, I64, P, P, P, P, I, P, I, P, P, P, SZ, P]
        L.wkv_v6_forward.restype = I
        L.wkv_query_status.argtypes = [P, P]
        L.wkv_query_status.restype = I
        L.wkv_status_string.argtypes = [I]
        L.wkv_status_string.restype = ctypes.c_char_p
        L.wkv_version.argtypes = []
        L.wkv_version.restype = ctypes.c_int32
        L.wkv_last_cuda_error.argtypes = []
        L.wkv_last_cuda_error.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().wkv_status_string(int(code)).decode()


def check(code: int, where: str) -> None:
    if code != WKV_OK:
        raise WkvError(code, where)
