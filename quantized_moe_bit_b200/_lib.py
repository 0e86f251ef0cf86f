"""ctypes binding of libmoe.so: argument marshalling only.

Every function here forwards device pointers (torch tensors' data_ptr) and
sizes to the C-ABI declared in include/moe.h and raises MoeError on a non-OK
status.  No computation happens in Python.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe.so")

MOE_OK = 0
# per-call path flags (include/moe.h)
MOE_FLAG_GEMV, MOE_FLAG_TC, MOE_FLAG_LAYERED = 1, 2, 4
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_CUDA", 3: "MOE_ERR_TIMEOUT",
          4: "MOE_ERR_DEVICE_CHECK", 5: "MOE_ERR_UNSUPPORTED"}


class MoeError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class moe_qmat(C.Structure):
    _fields_ = [("q", C.c_void_p), ("s", C.c_void_p), ("b", C.c_void_p),
                ("out", C.c_int32), ("inn", C.c_int32), ("bits", C.c_int32)]


_lib = None

# name -> (restype, argtypes)
_P, _I, _F, _Z = C.c_void_p, C.c_int, C.c_float, C.c_size_t
SIGNATURES = {
    "moe_last_error_string": (C.c_char_p, []),
    "moe_version": (_I, []),
    "moe_sync": (_I, [_P]),
    "moe_blob_bytes": (_Z, [_I, _I, C.POINTER(C.c_size_t)]),
    "moe_rmsnorm": (_I, [_P, _I, _I, _F, _P, _P]),
    "moe_router_topk": (_I, [_P, _I, _I, C.POINTER(moe_qmat), _P, _I, _I, _I, _P, _P, _P, _P]),
    "moe_bucket": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _P]),
    "moe_expert_workspace_size": (_Z, [_I, _I, _I, _I]),
    "moe_expert_forward": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _Z, _I, _P]),
    "moe_expert_forward_noalloc": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P]),
    "moe_shared_workspace_size": (_Z, [_I, _I, _I]),
    "moe_shared_forward": (_I, [_P, _I, _I, _I, C.POINTER(moe_qmat), _P, _P, _Z, _I, _P]),
    "moe_combine": (_I, [_P, _P, _P, _I, _I, _I, _P, _P, _P]),
    "moe_layer_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I]),
    "moe_layer_forward": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, C.POINTER(moe_qmat), _P, _I, _P,
                               C.POINTER(moe_qmat), _P, _P, _P, _P, _P, _Z, _I, _P]),
    "moe_decode_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I]),
    "moe_decode_launches": (_I, [_I, _I, _I]),
    "moe_set_decode_profile": (_I, [_P]),
    "moe_decode_grid": (_I, []),
    "moe_decode_forward": (_I, [_P, _I, _I, _I, _I, _I, _I, _I, C.POINTER(moe_qmat), C.POINTER(C.c_void_p), _I,
                                C.POINTER(C.c_void_p), C.POINTER(moe_qmat), _P, _P, _P, _P, _P, _Z, _I, _P]),
    "moe_decode_session_create": (_I, [_P, _I, _I, _I, _I, _I, _I, C.POINTER(moe_qmat), C.POINTER(C.c_void_p), _I,
                                       C.POINTER(C.c_void_p), C.POINTER(moe_qmat), _P, _Z, _I,
                                       C.POINTER(C.c_void_p)]),
    "moe_decode_session_step": (_I, [_P, _P, _P]),
    "moe_decode_session_stream": (_P, [_P]),
    "moe_decode_session_destroy": (_I, [_P]),
    "moe_lfu_create": (_I, [_I, _I, _I, _Z, _P, _P, _Z, C.POINTER(C.c_void_p)]),
    "moe_lfu_plan": (_I, [_P, _I, _P, _I, _P, _P]),
    "moe_lfu_step": (_I, [_P, _I, _P, _I, _P, _P, _P, _P, _I]),
    "moe_lfu_wait": (_I, [_P, _I]),
    "moe_lfu_get_log": (_I, [_P, _P, _Z, C.POINTER(C.c_size_t)]),
    "moe_lfu_stats": (_I, [_P, C.POINTER(C.c_int64), C.POINTER(C.c_int64), C.POINTER(C.c_int64)]),
    "moe_lfu_set_fault": (_I, [_P, _I, _I]),
    "moe_lfu_set_prefetch": (_I, [_P, _I]),
    "moe_lfu_plan_prefetch": (_I, [_P, _I, _I, _P, _P, C.POINTER(C.c_int)]),
    "moe_lfu_destroy": (_I, [_P]),
    "moe_streamed_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I]),
    "moe_streamed_layer_forward": (_I, [_P, _I, _P, _I, _I, _I, _I, _I, _I, C.POINTER(moe_qmat), _P, _I,
                                        C.POINTER(moe_qmat), _P, _P, _P, _P, _P, _Z, _I, _P, _P, _I]),
    "moe_ep_dispatch": (_I, [_P, _I, _I, _I, _I, _I, _I, _P, _P, _P, C.POINTER(C.c_void_p),
                             C.POINTER(C.c_void_p), _I, _P, _P, _P, _P, _P]),
    "moe_ep_return": (_I, [_P, _I, _I, _I, _I, _P, _P, _I, _I, C.POINTER(C.c_void_p), _P]),
    "moe_device_alloc": (_I, [_Z, C.POINTER(C.c_void_p)]),
    "moe_device_free": (_I, [_P]),
    "moe_ipc_handle_bytes": (_I, []),
    "moe_ipc_get_handle": (_I, [_P, _P]),
    "moe_ipc_open": (_I, [_P, C.POINTER(C.c_void_p)]),
    "moe_ipc_close": (_I, [_P]),
}


def lib():
    """Load libmoe.so (built in-tree); raise if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libmoe.so not built ({LIB_PATH}); run quantized_moe_bit_b200._build.build()")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def exported_symbols():
    return list(SIGNATURES)


def check(status: int):
    if status != MOE_OK:
        raise MoeError(status, lib().moe_last_error_string().decode(errors="replace"))


def ptr(t):
    """Device (or host) address of a tensor, or None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def stream_ptr(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def qmat(q, s, b, out, inn, bits) -> moe_qmat:
    return moe_qmat(ptr(q), ptr(s), ptr(b), out, inn, bits)
