"""ctypes binding of libdsa.so: the C ABI of ``include/dsa.h`` with the same names.

Argument marshalling only.  Every step of index building and attention runs in
the library's CUDA kernels; torch is used for device memory and streams.  If the
library is missing, loading fails loudly: there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdsa.so")

DSA_OK = 0
DSA_ERR_INVALID_ARG = 1
DSA_ERR_UNSUPPORTED = 2
DSA_ERR_CAPACITY = 3
DSA_ERR_CUDA = 4
DSA_ERR_TIMEOUT = 5
DSA_ERR_DEVICE = 6

DSA_KIND_ASHAPE = 0
DSA_KIND_VS = 1
DSA_KIND_BLOCK_TOPK = 2
DSA_KIND_BLOCK_THRESHOLD = 3
DSA_KIND_MOBA = 4
DSA_KIND_UNIFIED = 5
DSA_KIND_VS_WINDOWS = 6

KIND_CODES = {"ashape": DSA_KIND_ASHAPE, "vs": DSA_KIND_VS, "block_topk": DSA_KIND_BLOCK_TOPK,
              "block_threshold": DSA_KIND_BLOCK_THRESHOLD, "moba": DSA_KIND_MOBA,
              "unified": DSA_KIND_UNIFIED, "vs_windows": DSA_KIND_VS_WINDOWS}

EXPORTS = ("dsa_workspace_size", "dsa_build_indices", "dsa_sparse_prefill", "dsa_count_pairs",
           "dsa_get_device_status", "dsa_selftest_wait_timeout", "dsa_status_string",
           "dsa_last_cuda_error", "dsa_build_indices_static", "dsa_set_wait_limit")


class dsa_problem(ctypes.Structure):
    _fields_ = [("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("N", ctypes.c_int32),
                ("d", ctypes.c_int32), ("block", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("q_head_stride", ctypes.c_int64), ("q_token_stride", ctypes.c_int64),
                ("k_head_stride", ctypes.c_int64), ("k_token_stride", ctypes.c_int64),
                ("v_head_stride", ctypes.c_int64), ("v_token_stride", ctypes.c_int64),
                ("o_head_stride", ctypes.c_int64), ("o_token_stride", ctypes.c_int64)]


class dsa_pattern(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("sink", ctypes.c_int32), ("window", ctypes.c_int32),
                ("last_q", ctypes.c_int32), ("n_vert", ctypes.c_int32), ("n_slash", ctypes.c_int32),
                ("topk", ctypes.c_int32), ("alpha", ctypes.c_float), ("keep_sink", ctypes.c_int32),
                ("keep_local", ctypes.c_int32), ("conv_width", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("conv_weight", ctypes.c_void_p),
                ("conv_bias", ctypes.c_void_p)]


class dsa_indices(ctypes.Structure):
    _fields_ = [("head_info", ctypes.c_void_p), ("blk_ptr", ctypes.c_void_p),
                ("blk_idx", ctypes.c_void_p), ("dist_ptr", ctypes.c_void_p), ("dist", ctypes.c_void_p),
                ("col_ptr", ctypes.c_void_p), ("col_idx", ctypes.c_void_p),
                ("vert_idx", ctypes.c_void_p), ("slash_idx", ctypes.c_void_p),
                ("blk_cap", ctypes.c_int64), ("dist_cap", ctypes.c_int64), ("col_cap", ctypes.c_int64),
                ("vert_stride", ctypes.c_int32), ("slash_stride", ctypes.c_int32),
                ("kinds_present", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class dsa_sizes(ctypes.Structure):
    _fields_ = [("nqb", ctypes.c_int32), ("vert_stride", ctypes.c_int32),
                ("slash_stride", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("head_info_len", ctypes.c_int64), ("blk_ptr_len", ctypes.c_int64),
                ("blk_cap", ctypes.c_int64), ("dist_ptr_len", ctypes.c_int64),
                ("dist_cap", ctypes.c_int64), ("col_ptr_len", ctypes.c_int64),
                ("col_cap", ctypes.c_int64), ("workspace_bytes", ctypes.c_int64)]


_lib = None


def lib():
    """The loaded libdsa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libdsa.so not built at {LIB_PATH}; run "
                               "`python -m dynamic_sparse_attention_build_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER
        L.dsa_workspace_size.argtypes = [P(dsa_problem), P(dsa_pattern), P(dsa_sizes)]
        L.dsa_build_indices.argtypes = [P(dsa_problem), ctypes.c_void_p, ctypes.c_void_p, P(dsa_pattern),
                                        P(dsa_indices), ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
        L.dsa_sparse_prefill.argtypes = [P(dsa_problem), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                         P(dsa_indices), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        L.dsa_build_indices_static.argtypes = [P(dsa_problem), ctypes.c_void_p, ctypes.c_void_p,
                                               P(dsa_pattern), P(dsa_indices), ctypes.c_void_p]
        L.dsa_count_pairs.argtypes = [P(dsa_problem), P(dsa_indices), ctypes.c_void_p, ctypes.c_void_p]
        L.dsa_get_device_status.argtypes = [ctypes.c_void_p, P(ctypes.c_int32)]
        L.dsa_selftest_wait_timeout.argtypes = [ctypes.c_uint32, ctypes.c_void_p]
        L.dsa_set_wait_limit.argtypes = [ctypes.c_uint64]
        L.dsa_status_string.argtypes = [ctypes.c_int]
        L.dsa_status_string.restype = ctypes.c_char_p
        L.dsa_last_cuda_error.argtypes = []
        for name in EXPORTS:
            if name not in ("dsa_status_string",):
                getattr(L, name).restype = ctypes.c_int if name != "dsa_last_cuda_error" else ctypes.c_int32
        _lib = L
    return _lib


class DSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = lib().dsa_status_string(status).decode()
        if status == DSA_ERR_CUDA:
            msg += f" (cudaError {lib().dsa_last_cuda_error()})"
        super().__init__(f"{where}: {msg}")
        self.status = status


def check(status: int, where: str):
    if status != DSA_OK:
        raise DSAError(status, where)


# ---- the C ABI, same names -------------------------------------------------
def dsa_workspace_size(problem, patterns):
    sz = dsa_sizes()
    check(lib().dsa_workspace_size(ctypes.byref(problem), patterns, ctypes.byref(sz)), "dsa_workspace_size")
    return sz


def dsa_build_indices(problem, Q_ptr, K_ptr, patterns, indices, ws_ptr, ws_bytes, stream_ptr):
    return lib().dsa_build_indices(ctypes.byref(problem), Q_ptr, K_ptr, patterns, ctypes.byref(indices),
                                   ws_ptr, ws_bytes, stream_ptr)


def dsa_build_indices_static(problem, Q_ptr, K_ptr, patterns, indices, stream_ptr):
    return lib().dsa_build_indices_static(ctypes.byref(problem), Q_ptr, K_ptr, patterns,
                                          ctypes.byref(indices), stream_ptr)


def dsa_sparse_prefill(problem, Q_ptr, K_ptr, V_ptr, indices, O_ptr, lse_ptr, stream_ptr):
    return lib().dsa_sparse_prefill(ctypes.byref(problem), Q_ptr, K_ptr, V_ptr, ctypes.byref(indices),
                                    O_ptr, lse_ptr, stream_ptr)


def dsa_count_pairs(problem, indices, pairs_ptr, stream_ptr):
    return lib().dsa_count_pairs(ctypes.byref(problem), ctypes.byref(indices), pairs_ptr, stream_ptr)


def dsa_get_device_status(stream_ptr):
    detail = ctypes.c_int32(0)
    s = lib().dsa_get_device_status(stream_ptr, ctypes.byref(detail))
    return s, detail.value


def dsa_selftest_wait_timeout(timeout_us, stream_ptr):
    return lib().dsa_selftest_wait_timeout(timeout_us, stream_ptr)


def dsa_set_wait_limit(limit_ns):
    return lib().dsa_set_wait_limit(limit_ns)


def dsa_status_string(status):
    return lib().dsa_status_string(status).decode()


def dsa_last_cuda_error():
    return lib().dsa_last_cuda_error()
