"""Python entry points with the C-ABI's names (see include/moe.h).

Tensors are torch CUDA tensors; the functions pass their addresses and sizes
to libmoe and check the status.  `stream` defaults to torch's current stream.
"""
from __future__ import annotations

import ctypes as C

from ._lib import check, lib, moe_qmat, ptr, stream_ptr


def moe_version() -> int:
    return lib().moe_version()


def moe_sync(stream=None):
    check(lib().moe_sync(stream_ptr(stream)))


def moe_blob_bytes(H: int, I: int):
    offs = (C.c_size_t * 9)()
    n = lib().moe_blob_bytes(H, I, offs)
    return n, list(offs)


def moe_set_gemv_max_rows(rows: int):
    check(lib().moe_set_gemv_max_rows(rows))


def moe_rmsnorm(h, x, eps: float = 1e-6, stream=None):
    T, H = h.shape
    check(lib().moe_rmsnorm(ptr(h), T, H, eps, ptr(x), stream_ptr(stream)))


def moe_router_topk(x, router: moe_qmat, bias, bias_per_row: int, E: int, k: int, idx, gates,
                    logits=None, stream=None):
    T, H = x.shape
    check(lib().moe_router_topk(ptr(x), T, H, C.byref(router), ptr(bias), bias_per_row, E, k,
                                ptr(idx), ptr(gates), ptr(logits), stream_ptr(stream)))


def moe_bucket(idx, E: int, offsets, pairs, active, n_active, stream=None):
    T, k = idx.shape
    check(lib().moe_bucket(ptr(idx), T, k, E, ptr(offsets), ptr(pairs), ptr(active), ptr(n_active),
                           stream_ptr(stream)))


def moe_expert_workspace_size(T: int, H: int, I: int, k: int) -> int:
    return lib().moe_expert_workspace_size(T, H, I, k)


def moe_expert_forward(x, I: int, E: int, k: int, blob_ptrs, offsets, pairs, active, n_active, y_pairs,
                       ws, stream=None):
    T, H = x.shape
    check(lib().moe_expert_forward(ptr(x), T, H, I, E, k, ptr(blob_ptrs), ptr(offsets), ptr(pairs),
                                   ptr(active), ptr(n_active), ptr(y_pairs), ptr(ws), ws.numel() * ws.element_size(),
                                   stream_ptr(stream)))


def moe_expert_forward_noalloc(x, I: int, E: int, k: int, blob_ptrs, offsets, pairs, active, n_active,
                               y_pairs, stream=None):
    """moe_expert_forward with its scratch in the library's static device
    array (no workspace argument; see include/moe.h for the size limit)."""
    T, H = x.shape
    check(lib().moe_expert_forward_noalloc(ptr(x), T, H, I, E, k, ptr(blob_ptrs), ptr(offsets), ptr(pairs),
                                           ptr(active), ptr(n_active), ptr(y_pairs), stream_ptr(stream)))


def moe_shared_workspace_size(T: int, H: int, Is: int) -> int:
    return lib().moe_shared_workspace_size(T, H, Is)


def _qmat3(shared):
    arr = (moe_qmat * 3)(*shared)
    return arr


def moe_shared_forward(x, Is: int, shared, ysh, ws, stream=None):
    T, H = x.shape
    arr = _qmat3(shared)
    check(lib().moe_shared_forward(ptr(x), T, H, Is, arr, ptr(ysh), ptr(ws), ws.numel() * ws.element_size(),
                                   stream_ptr(stream)))


def moe_combine(y_pairs, gates, ysh, y=None, residual=None, stream=None):
    T, k = gates.shape
    H = y_pairs.shape[1]
    check(lib().moe_combine(ptr(y_pairs), ptr(gates), ptr(ysh), T, H, k, ptr(y), ptr(residual),
                            stream_ptr(stream)))


def moe_layer_workspace_size(T: int, H: int, I: int, Is: int, E: int, k: int) -> int:
    return lib().moe_layer_workspace_size(T, H, I, Is, E, k)


def moe_layer_forward(T: int, H: int, I: int, Is: int, E: int, k: int, router: moe_qmat, bias,
                      bias_per_row: int, blob_ptrs, shared, ws, h_in=None, h_out=None, x_in=None,
                      x_out=None, y=None, idx=None, gates=None, stream=None):
    arr = _qmat3(shared)
    check(lib().moe_layer_forward(ptr(h_in), ptr(h_out), ptr(x_in), T, H, I, Is, E, k, C.byref(router),
                                  ptr(bias), bias_per_row, ptr(blob_ptrs), arr, ptr(x_out), ptr(y), ptr(idx),
                                  ptr(gates), ptr(ws), ws.numel() * ws.element_size(), stream_ptr(stream)))


def moe_set_decode_fused(enable: bool, spec_experts: int = 0):
    check(lib().moe_set_decode_fused(1 if enable else 0, spec_experts))


def moe_set_decode_profile(stamps=None):
    check(lib().moe_set_decode_profile(ptr(stamps)))


def moe_set_decode_prefetch(flags: int):
    check(lib().moe_set_decode_prefetch(flags))


def moe_decode_grid() -> int:
    return lib().moe_decode_grid()


def moe_decode_launches(T: int, L: int) -> int:
    return lib().moe_decode_launches(T, L)


def moe_decode_workspace_size(T: int, H: int, I: int, Is: int, E: int, k: int) -> int:
    return lib().moe_decode_workspace_size(T, H, I, Is, E, k)


class DecodeStack:
    """Host-side argument arrays of a layer stack, built once (marshalling only)."""

    def __init__(self, layers, per_row_bias=None):
        L = len(layers)
        self.L = L
        self.routers = (moe_qmat * L)(*[dl.router.c for dl in layers])
        self.shared = (moe_qmat * (3 * L))(*[m for dl in layers for m in dl.shared_c])
        self.tables = (C.c_void_p * L)(*[dl.blob_ptrs.data_ptr() for dl in layers])
        self.set_biases([dl.bias for dl in layers] if per_row_bias is None else per_row_bias,
                        per_row=per_row_bias is not None)

    def set_biases(self, biases, per_row=False):
        self.bias_per_row = 1 if per_row else 0
        self._bias_refs = biases
        self.biases = (C.c_void_p * self.L)(*[None if b is None else b.data_ptr() for b in biases])


def moe_decode_forward(h, I: int, Is: int, E: int, k: int, stack: "DecodeStack", ws, x_trace=None,
                       y_trace=None, idx_trace=None, gates_trace=None, stream=None):
    T, H = h.shape
    check(lib().moe_decode_forward(ptr(h), T, H, I, Is, E, k, stack.L, stack.routers, stack.biases,
                                   stack.bias_per_row, stack.tables, stack.shared, ptr(x_trace), ptr(y_trace),
                                   ptr(idx_trace), ptr(gates_trace), ptr(ws), ws.numel() * ws.element_size(),
                                   stream_ptr(stream)))
