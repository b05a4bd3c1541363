"""ctypes view of libfvattn.so (the C ABI of include/fvattn.h). Marshalling only."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfvattn.so")
# The checked build (-DFVATTN_DEBUG): the same entry points; its kernels check every CSR list
# before reading it and report a failed check as FVATTN_ERR_INVALID (status[1] = 101: row
# offsets, 102: a key block out of range, 103: a list not ascending).
DEBUG_LIB_PATH = os.path.join(_HERE, "libfvattn_debug.so")
DEBUG_OFFSETS, DEBUG_COLUMN, DEBUG_ORDER = 101, 102, 103

FVATTN_OK = 0
FVATTN_ERR_INVALID = -1
FVATTN_ERR_UNSUPPORTED = -2
FVATTN_ERR_CAPACITY = -3
FVATTN_ERR_CUDA = -4
FVATTN_ERR_TIMEOUT = -5

FVATTN_BF16 = 0
FVATTN_F32 = 1
FVATTN_MODE_TOPP = 0
FVATTN_MODE_FRAME_TOPK = 1
FVATTN_MODE_TOPK_BLOCKS = 2


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("H", ctypes.c_int64), ("S", ctypes.c_int64), ("d", ctypes.c_int64),
                ("block", ctypes.c_int32), ("dtype", ctypes.c_int32), ("scale", ctypes.c_float)]


class RouteCfg(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("p", ctypes.c_float), ("force_diag", ctypes.c_int32),
                ("local_window", ctypes.c_int32), ("frame_len", ctypes.c_int32), ("topk_frames", ctypes.c_int32),
                ("frame_window", ctypes.c_int32), ("force_first_frame", ctypes.c_int32),
                ("topk_blocks", ctypes.c_int32), ("sasa_coef", ctypes.c_float), ("sasa_trigger", ctypes.c_int32),
                ("frame_exact", ctypes.c_int32)]


class Csr(ctypes.Structure):
    _fields_ = [("row_ptr", ctypes.c_void_p), ("col_idx", ctypes.c_void_p), ("col_capacity", ctypes.c_int64),
                ("head_load", ctypes.c_void_p), ("tile_cost", ctypes.c_void_p), ("tile_order", ctypes.c_void_p),
                ("nnz", ctypes.c_void_p), ("status", ctypes.c_void_p), ("col_code", ctypes.c_void_p)]


class FvattnError(RuntimeError):
    def __init__(self, code: int, what: str):
        msg = f"{what}: {status_string(code)} ({code})"
        if code == FVATTN_ERR_CUDA:
            lib = load()
            err = lib.fvattn_last_cuda_error()
            msg += f" [{lib.fvattn_cuda_error_name(err).decode()} ({err})]"
        super().__init__(msg)
        self.code = code


_lib = None


def use_debug_build() -> None:
    """Make this process load the checked build. Must come before the first load()."""
    global LIB_PATH
    if _lib is not None and LIB_PATH != DEBUG_LIB_PATH:
        raise RuntimeError("the library is already loaded; select the checked build before the first call")
    LIB_PATH = DEBUG_LIB_PATH


def load() -> ctypes.CDLL:
    """Load the in-tree library. Raises if it has not been built: there is no other path."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with `python -m block_sparse_top_fvattn_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER
    vp = ctypes.c_void_p
    lib.fvattn_version.restype = ctypes.c_int
    lib.fvattn_version.argtypes = []
    lib.fvattn_status_string.restype = ctypes.c_char_p
    lib.fvattn_status_string.argtypes = [ctypes.c_int]
    lib.fvattn_last_cuda_error.restype = ctypes.c_int
    lib.fvattn_last_cuda_error.argtypes = []
    lib.fvattn_cuda_error_name.restype = ctypes.c_char_p
    lib.fvattn_cuda_error_name.argtypes = [ctypes.c_int]
    lib.fvattn_csr_max_nnz.restype = ctypes.c_int64
    lib.fvattn_csr_max_nnz.argtypes = [P(Shape)]
    lib.fvattn_num_tiles.restype = ctypes.c_int64
    lib.fvattn_num_tiles.argtypes = [P(Shape)]
    lib.fvattn_route_workspace_bytes.restype = ctypes.c_size_t
    lib.fvattn_route_workspace_bytes.argtypes = [P(Shape), P(RouteCfg)]
    lib.fvattn_route.restype = ctypes.c_int
    lib.fvattn_route.argtypes = [vp, vp, P(Shape), P(RouteCfg), P(Csr), vp, ctypes.c_size_t, vp]
    lib.fvattn_route_pool.restype = ctypes.c_int
    lib.fvattn_route_pool.argtypes = [vp, vp, P(Shape), P(RouteCfg), ctypes.c_int64, ctypes.c_int64, vp,
                                      ctypes.c_size_t, vp]
    lib.fvattn_route_finish.restype = ctypes.c_int
    lib.fvattn_route_finish.argtypes = [P(Shape), P(RouteCfg), P(Csr), vp, ctypes.c_size_t, vp]
    lib.fvattn_sparse_attn.restype = ctypes.c_int
    lib.fvattn_sparse_attn.argtypes = [vp, vp, vp, P(Shape), P(Csr), vp, vp, vp]
    lib.fvattn_block_means.restype = ctypes.c_int
    lib.fvattn_block_means.argtypes = [vp, P(Shape), vp, vp]
    lib.fvattn_block_scores_workspace_bytes.restype = ctypes.c_size_t
    lib.fvattn_block_scores_workspace_bytes.argtypes = [P(Shape)]
    lib.fvattn_block_scores_ld.restype = ctypes.c_int64
    lib.fvattn_block_scores_ld.argtypes = [P(Shape)]
    lib.fvattn_block_scores.restype = ctypes.c_int
    lib.fvattn_block_scores.argtypes = [vp, vp, P(Shape), vp, vp, ctypes.c_size_t, vp, vp]
    lib.fvattn_attn_stamp_words.restype = ctypes.c_int64
    lib.fvattn_attn_stamp_words.argtypes = [P(Shape)]
    lib.fvattn_sparse_attn_stamped.restype = ctypes.c_int
    lib.fvattn_sparse_attn_stamped.argtypes = [vp, vp, vp, P(Shape), P(Csr), vp, vp, vp, ctypes.c_int64, vp]
    lib.fvattn_sparse_attn_timeout_check.restype = ctypes.c_int
    lib.fvattn_sparse_attn_timeout_check.argtypes = [vp, vp, vp, P(Shape), P(Csr), vp, ctypes.c_uint32, vp]
    lib.fvattn_block_scores_timeout_check.restype = ctypes.c_int
    lib.fvattn_block_scores_timeout_check.argtypes = [vp, vp, P(Shape), vp, vp, ctypes.c_size_t, vp, ctypes.c_uint32,
                                                      vp]
    lib.fvattn_read_status.restype = ctypes.c_int
    lib.fvattn_read_status.argtypes = [P(Csr), vp]
    lib.fvattn_route_static_scratch.restype = ctypes.c_int
    lib.fvattn_route_static_scratch.argtypes = [vp, vp, P(Shape), P(RouteCfg), P(Csr), vp]
    lib.fvattn_rlb_plan.restype = ctypes.c_int
    lib.fvattn_rlb_plan.argtypes = [vp, ctypes.c_int32, ctypes.c_int32, ctypes.c_double, ctypes.c_int32, vp,
                                    ctypes.c_int64, P(ctypes.c_int32), vp]
    lib.fvattn_select_heads.restype = ctypes.c_int
    lib.fvattn_select_heads.argtypes = [P(Shape), P(Csr), vp, vp]
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load().fvattn_status_string(int(code)).decode()


def check(code: int, what: str) -> None:
    if code != FVATTN_OK:
        raise FvattnError(code, what)
