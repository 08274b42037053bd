"""ctypes mirror of include/tm.h.  Argument marshalling only: no compute here."""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_float, c_int, c_size_t, c_void_p

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtm.so")

TM_OK, TM_ERR_INVALID_ARG, TM_ERR_UNSUPPORTED, TM_ERR_WORKSPACE, TM_ERR_CUDA, TM_ERR_DEVICE_TIMEOUT, \
    TM_ERR_DEVICE_BOUNDS = range(7)
TM_F32, TM_BF16 = 0, 1
TM_LAYOUT_ROWS, TM_LAYOUT_MIXED = 0, 1
TM_TP_TOKEN_SHARD, TM_TP_HEAD_SHARD = 0, 1

# Every entry point declared in include/tm.h (the CPU test checks the library exports each one).
EXPORTS = ["tm_status_string", "tm_version", "tm_sublayer_workspace_bytes", "tm_route_workspace_bytes",
           "tm_workspace_bytes", "tm_tokenize_stub", "tm_mix", "tm_revert", "tm_route_topk", "tm_route_topk_noalloc",
           "tm_pertoken_swiglu", "tm_sparse_pertoken_moe", "tm_block_forward", "tm_stack_step", "tm_stack_forward",
           "tm_sublayer_forward",
           "tm_profile_start", "tm_profile_stop", "tm_last_cuda_error", "tm_launch_count",
           "tm_get_device_error", "tm_quantize_fp8_weights", "tm_quantize_fp8_act",
           "tm_pertoken_swiglu_fp8_workspace_bytes", "tm_pertoken_swiglu_fp8", "tm_block_fp8_workspace_bytes",
           "tm_block_forward_fp8", "tm_head_forward", "tm_model_workspace_bytes", "tm_model_forward",
           "tm_pertoken_swiglu_backward_workspace_bytes", "tm_pertoken_swiglu_backward",
           "tm_block_backward_workspace_bytes", "tm_block_backward", "tm_stack_backward_workspace_bytes",
           "tm_stack_backward", "tm_last_device_error_site", "tm_set_wait_limit_ns", "tm_selftest_wait",
           "tm_selftest_bucket_scatter", "tm_sublayer_fp8_workspace_bytes", "tm_sublayer_forward_fp8",
           "tm_sparse_pertoken_moe_fp8", "tm_tp_exchange_layout"]


class tm_shape(ctypes.Structure):
    _fields_ = [("B", c_int), ("T", c_int), ("D", c_int), ("H", c_int), ("dtype", c_int), ("eps", c_float)]


class tm_swiglu_w(ctypes.Structure):
    _fields_ = [("banks", c_int), ("width", c_int), ("hidden", c_int),
                ("w_gate", c_void_p), ("w_up", c_void_p), ("w_down", c_void_p)]


class tm_moe_w(ctypes.Structure):
    _fields_ = [("banks", c_int), ("width", c_int), ("E", c_int), ("k", c_int), ("hidden_e", c_int),
                ("hidden_s", c_int), ("alpha", c_float), ("w_router", c_void_p),
                ("we_gate", c_void_p), ("we_up", c_void_p), ("we_down", c_void_p),
                ("ws_gate", c_void_p), ("ws_up", c_void_p), ("ws_down", c_void_p)]


class tm_sublayer(ctypes.Structure):
    _fields_ = [("norm_gain", c_void_p), ("is_moe", c_int), ("dense", tm_swiglu_w), ("moe", tm_moe_w)]


class tm_block(ctypes.Structure):
    _fields_ = [("mix", tm_sublayer), ("rev", tm_sublayer)]


class tm_swiglu_w8(ctypes.Structure):
    _fields_ = [("banks", c_int), ("width", c_int), ("hidden", c_int), ("q_gate", c_void_p), ("q_up", c_void_p),
                ("s_gate", c_void_p), ("s_up", c_void_p), ("w_down", c_void_p)]


class tm_block_fp8(ctypes.Structure):
    _fields_ = [("mix", tm_swiglu_w8), ("rev", tm_swiglu_w8)]


class tm_moe_w8(ctypes.Structure):
    _fields_ = [("banks", c_int), ("width", c_int), ("E", c_int), ("k", c_int), ("hidden_e", c_int),
                ("hidden_s", c_int), ("alpha", c_float), ("w_router", c_void_p),
                ("qe_gate", c_void_p), ("qe_up", c_void_p), ("se_gate", c_void_p), ("se_up", c_void_p),
                ("we_down", c_void_p), ("qs_gate", c_void_p), ("qs_up", c_void_p), ("ss_gate", c_void_p),
                ("ss_up", c_void_p), ("ws_down", c_void_p)]


class tm_sublayer8(ctypes.Structure):
    _fields_ = [("norm_gain", c_void_p), ("is_moe", c_int), ("dense", tm_swiglu_w8), ("moe", tm_moe_w8)]


class tm_swiglu_grads(ctypes.Structure):
    _fields_ = [("dw_gate", c_void_p), ("dw_up", c_void_p), ("dw_down", c_void_p)]


class tm_block_grads(ctypes.Structure):
    _fields_ = [("mix", tm_swiglu_grads), ("rev", tm_swiglu_grads)]


class tm_kernel_time(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", c_int), ("total_ms", ctypes.c_double)]


_P = c_void_p
_SIGS = {
    "tm_status_string": (ctypes.c_char_p, [c_int]),
    "tm_version": (c_int, []),
    "tm_sublayer_workspace_bytes": (c_size_t, [POINTER(tm_shape), c_int, POINTER(tm_sublayer)]),
    "tm_route_workspace_bytes": (c_size_t, [POINTER(tm_shape), c_int, POINTER(tm_moe_w)]),
    "tm_workspace_bytes": (c_size_t, [POINTER(tm_shape), POINTER(tm_block), c_int, c_int]),
    "tm_tokenize_stub": (c_int, [_P, _P, _P, c_int, POINTER(tm_shape), _P, _P]),
    "tm_mix": (c_int, [_P, _P, POINTER(tm_shape), _P]),
    "tm_revert": (c_int, [_P, _P, POINTER(tm_shape), _P]),
    "tm_route_topk": (c_int, [_P, c_int, POINTER(tm_shape), _P, POINTER(tm_moe_w), _P, _P, _P, _P, _P, _P, _P, _P,
                              c_size_t, _P]),
    "tm_route_topk_noalloc": (c_int, [_P, c_int, POINTER(tm_shape), _P, POINTER(tm_moe_w), _P, _P, _P, _P, _P, _P,
                                      _P, _P]),
    "tm_pertoken_swiglu": (c_int, [_P, _P, c_int, POINTER(tm_shape), _P, POINTER(tm_swiglu_w), _P, _P, c_size_t, _P]),
    "tm_sparse_pertoken_moe": (c_int, [_P, _P, c_int, POINTER(tm_shape), _P, POINTER(tm_moe_w), _P, _P, c_size_t, _P]),
    "tm_block_forward": (c_int, [_P, POINTER(tm_block), POINTER(tm_shape), _P, _P, _P, c_size_t, _P]),
    "tm_stack_step": (c_int, [_P, _P, POINTER(tm_block), POINTER(tm_shape), _P, _P, _P, c_size_t, _P]),
    "tm_sublayer_forward": (c_int, [_P, _P, _P, c_int, POINTER(tm_shape), POINTER(tm_sublayer), _P, _P, c_size_t, _P]),
    "tm_stack_forward": (c_int, [_P, POINTER(tm_block), c_int, c_int, POINTER(tm_shape), _P, _P, c_size_t, _P]),
    "tm_profile_start": (c_int, []),
    "tm_profile_stop": (c_int, [POINTER(tm_kernel_time), c_int, POINTER(c_int)]),
    "tm_last_cuda_error": (ctypes.c_char_p, []),
    "tm_launch_count": (ctypes.c_ulonglong, []),
    "tm_get_device_error": (c_int, [_P]),
    "tm_last_device_error_site": (ctypes.c_uint, []),
    "tm_set_wait_limit_ns": (c_int, [ctypes.c_uint64]),
    "tm_selftest_wait": (c_int, [_P, _P]),
    "tm_selftest_bucket_scatter": (c_int, [_P, _P, _P, c_int, c_int, c_int, c_int, _P, c_int, _P, _P]),
    "tm_quantize_fp8_weights": (c_int, [_P, _P, c_int, c_size_t, c_int, _P, _P, _P]),
    "tm_quantize_fp8_act": (c_int, [_P, c_int, POINTER(tm_shape), c_int, c_int, _P, _P, _P]),
    "tm_pertoken_swiglu_fp8_workspace_bytes": (c_size_t, [POINTER(tm_shape), c_int, POINTER(tm_swiglu_w8)]),
    "tm_pertoken_swiglu_fp8": (c_int, [_P, _P, c_int, POINTER(tm_shape), POINTER(tm_swiglu_w8), _P, _P, c_size_t, _P]),
    "tm_block_fp8_workspace_bytes": (c_size_t, [POINTER(tm_shape), POINTER(tm_block_fp8)]),
    "tm_block_forward_fp8": (c_int, [_P, POINTER(tm_block_fp8), POINTER(tm_shape), _P, _P, _P, c_size_t, _P]),
    "tm_sublayer_fp8_workspace_bytes": (c_size_t, [POINTER(tm_shape), c_int, POINTER(tm_sublayer8)]),
    "tm_sublayer_forward_fp8": (c_int, [_P, _P, _P, c_int, POINTER(tm_shape), POINTER(tm_sublayer8), _P, _P, c_size_t,
                                        _P]),
    "tm_sparse_pertoken_moe_fp8": (c_int, [_P, _P, c_int, POINTER(tm_shape), _P, POINTER(tm_moe_w8), _P, _P, c_size_t,
                                           _P]),
    "tm_tp_exchange_layout": (c_int, [_P, _P, c_int, c_int, c_int, c_int, c_int, c_int, c_int, _P]),
    "tm_head_forward": (c_int, [_P, POINTER(tm_shape), _P, _P, _P]),
    "tm_model_workspace_bytes": (c_size_t, [POINTER(tm_shape), POINTER(tm_block), c_int, c_int]),
    "tm_model_forward": (c_int, [_P, _P, _P, c_int, POINTER(tm_block), c_int, c_int, _P, POINTER(tm_shape), _P, _P,
                                 c_size_t, _P]),
    "tm_pertoken_swiglu_backward_workspace_bytes": (c_size_t, [POINTER(tm_shape), c_int, POINTER(tm_swiglu_w)]),
    "tm_pertoken_swiglu_backward": (c_int, [_P, _P, _P, c_int, POINTER(tm_shape), _P, POINTER(tm_swiglu_w), _P,
                                            POINTER(tm_swiglu_grads), _P, c_size_t, _P]),
    "tm_block_backward_workspace_bytes": (c_size_t, [POINTER(tm_shape), POINTER(tm_block)]),
    "tm_block_backward": (c_int, [_P, _P, POINTER(tm_block), POINTER(tm_shape), _P, POINTER(tm_block_grads), _P,
                                  c_size_t, _P]),
    "tm_stack_backward_workspace_bytes": (c_size_t, [POINTER(tm_shape), POINTER(tm_block), c_int, c_int]),
    "tm_stack_backward": (c_int, [_P, _P, POINTER(tm_block), c_int, c_int, POINTER(tm_shape), _P,
                                  POINTER(tm_block_grads), _P, c_size_t, _P]),
}

_lib = None


class TMError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = status
        msg = load().tm_status_string(status).decode() if _lib is not None else str(status)
        detail = load().tm_last_cuda_error().decode() if _lib is not None else ""
        super().__init__(f"{where}: tm status {status} ({msg}){' -- ' + detail if detail else ''}")


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libtm.so.  There is no fallback: a missing library is an error."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise ImportError(f"libtm.so not found at {path}; build it with `python -m token_sparse_moe_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def check(status: int, where: str) -> None:
    if status != TM_OK:
        raise TMError(status, where)
