"""Python entry points with the C-ABI's names (see include/moe.h).

Tensors are torch CUDA tensors; the functions pass their addresses and sizes
to libmoe and check the status.  `stream` defaults to torch's current stream.
"""
from __future__ import annotations

import ctypes as C

from ._lib import MOE_FLAG_GEMV, MOE_FLAG_LAYERED, MOE_FLAG_TC, check, lib, moe_qmat, ptr, stream_ptr  # noqa: F401


def moe_version() -> int:
    return lib().moe_version()


def moe_sync(stream=None):
    check(lib().moe_sync(stream_ptr(stream)))


def moe_blob_bytes(H: int, I: int):
    offs = (C.c_size_t * 9)()
    n = lib().moe_blob_bytes(H, I, offs)
    return n, list(offs)


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
                       ws, flags: int = 0, stream=None):
    T, H = x.shape
    check(lib().moe_expert_forward(ptr(x), T, H, I, E, k, ptr(blob_ptrs), ptr(offsets), ptr(pairs),
                                   ptr(active), ptr(n_active), ptr(y_pairs), ptr(ws), ws.numel() * ws.element_size(),
                                   flags, stream_ptr(stream)))


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


def moe_shared_forward(x, Is: int, shared, ysh, ws, flags: int = 0, stream=None):
    T, H = x.shape
    arr = _qmat3(shared)
    check(lib().moe_shared_forward(ptr(x), T, H, Is, arr, ptr(ysh), ptr(ws), ws.numel() * ws.element_size(),
                                   flags, stream_ptr(stream)))


def moe_combine(y_pairs, gates, ysh, y=None, residual=None, stream=None):
    T, k = gates.shape
    H = y_pairs.shape[1]
    check(lib().moe_combine(ptr(y_pairs), ptr(gates), ptr(ysh), T, H, k, ptr(y), ptr(residual),
                            stream_ptr(stream)))


def moe_layer_workspace_size(T: int, H: int, I: int, Is: int, E: int, k: int) -> int:
    return lib().moe_layer_workspace_size(T, H, I, Is, E, k)


def moe_layer_forward(T: int, H: int, I: int, Is: int, E: int, k: int, router: moe_qmat, bias,
                      bias_per_row: int, blob_ptrs, shared, ws, h_in=None, h_out=None, x_in=None,
                      x_out=None, y=None, idx=None, gates=None, flags: int = 0, stream=None):
    arr = _qmat3(shared)
    check(lib().moe_layer_forward(ptr(h_in), ptr(h_out), ptr(x_in), T, H, I, Is, E, k, C.byref(router),
                                  ptr(bias), bias_per_row, ptr(blob_ptrs), arr, ptr(x_out), ptr(y), ptr(idx),
                                  ptr(gates), ptr(ws), ws.numel() * ws.element_size(), flags, stream_ptr(stream)))


def moe_set_decode_profile(stamps=None):
    check(lib().moe_set_decode_profile(ptr(stamps)))


def moe_decode_grid() -> int:
    return lib().moe_decode_grid()


def moe_decode_launches(T: int, L: int, flags: int = 0) -> int:
    return lib().moe_decode_launches(T, L, flags)


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
                       y_trace=None, idx_trace=None, gates_trace=None, flags: int = 0, stream=None):
    T, H = h.shape
    check(lib().moe_decode_forward(ptr(h), T, H, I, Is, E, k, stack.L, stack.routers, stack.biases,
                                   stack.bias_per_row, stack.tables, stack.shared, ptr(x_trace), ptr(y_trace),
                                   ptr(idx_trace), ptr(gates_trace), ptr(ws), ws.numel() * ws.element_size(),
                                   flags, stream_ptr(stream)))


class DecodeSession:
    """moe_decode_session_*: batch-1 steps from host rows to host rows (the
    arguments marshalled once; a step is one C call)."""

    def __init__(self, h_dev, I: int, Is: int, E: int, k: int, stack: "DecodeStack", ws, flags: int = 0):
        H = h_dev.shape[-1]
        self._refs = (h_dev, stack, ws)
        hnd = C.c_void_p()
        check(lib().moe_decode_session_create(ptr(h_dev), H, I, Is, E, k, stack.L, stack.routers, stack.biases,
                                              stack.bias_per_row, stack.tables, stack.shared, ptr(ws),
                                              ws.numel() * ws.element_size(), flags, C.byref(hnd)))
        self._h = hnd.value
        self._step = lib().moe_decode_session_step

    @property
    def stream(self) -> int:
        return lib().moe_decode_session_stream(self._h)

    def step(self, h_in, h_out):
        """h_in, h_out: host addresses (ints) or CPU tensors of H fp32."""
        st = self._step(self._h, h_in if isinstance(h_in, int) else h_in.data_ptr(),
                        h_out if isinstance(h_out, int) else h_out.data_ptr())
        if st:
            check(st)

    def close(self):
        if self._h:
            check(lib().moe_decode_session_destroy(self._h))
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ------------------------------------------------------------------ LFU cache
class MoeLfu:
    """Handle of the per-layer LFU expert-slot cache (moe_lfu_* calls)."""

    def __init__(self, n_layers: int, n_experts: int, n_slots: int, blob_bytes: int = 0, host_blob_ptrs=None,
                 slot_pool=None, slot_stride: int = 0):
        self._h = C.c_void_p()
        self._blobs = None
        if host_blob_ptrs is not None:
            self._blobs = (C.c_void_p * len(host_blob_ptrs))(*host_blob_ptrs)
        check(lib().moe_lfu_create(n_layers, n_experts, n_slots, blob_bytes, self._blobs, ptr(slot_pool),
                                   slot_stride, C.byref(self._h)))
        self.n_slots = n_slots

    @property
    def handle(self):
        return self._h

    def plan(self, layer: int, ids):
        n = len(ids)
        a = (C.c_int32 * max(n, 1))(*ids)
        so = (C.c_int32 * max(n, 1))()
        ho = (C.c_int32 * max(n, 1))()
        check(lib().moe_lfu_plan(self._h, layer, a, n, so, ho))
        return list(so)[:n], list(ho)[:n]

    def step(self, layer: int, ids, side_stream, wait_event, done_event, dev_table, timeout_ms: int = 2000):
        n = len(ids)
        a = (C.c_int32 * max(n, 1))(*ids)
        check(lib().moe_lfu_step(self._h, layer, a, n, stream_ptr(side_stream),
                                 None if wait_event is None else wait_event.cuda_event,
                                 done_event.cuda_event, ptr(dev_table), timeout_ms))

    def log(self):
        n = C.c_size_t()
        check(lib().moe_lfu_get_log(self._h, None, 0, C.byref(n)))
        buf = (C.c_int32 * (5 * max(n.value, 1)))()
        check(lib().moe_lfu_get_log(self._h, buf, n.value, C.byref(n)))
        v = list(buf)[:5 * n.value]
        return [tuple(v[i:i + 5]) for i in range(0, len(v), 5)]

    def stats(self):
        h, m, b = C.c_int64(), C.c_int64(), C.c_int64()
        check(lib().moe_lfu_stats(self._h, C.byref(h), C.byref(m), C.byref(b)))
        return h.value, m.value, b.value

    def set_fault(self, kind: int, after_n: int):
        check(lib().moe_lfu_set_fault(self._h, kind, after_n))

    def set_prefetch(self, per_call: int):
        check(lib().moe_lfu_set_prefetch(self._h, per_call))

    def plan_prefetch(self, layer: int, per_call: int):
        ids = (C.c_int32 * max(per_call, 1))()
        slots = (C.c_int32 * max(per_call, 1))()
        n = C.c_int()
        check(lib().moe_lfu_plan_prefetch(self._h, layer, per_call, ids, slots, C.byref(n)))
        return list(ids)[:n.value], list(slots)[:n.value]

    def close(self):
        if self._h:
            lib().moe_lfu_destroy(self._h)
            self._h = C.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def moe_lfu_wait(event, timeout_ms: int):
    check(lib().moe_lfu_wait(event.cuda_event, timeout_ms))


def moe_streamed_workspace_size(T: int, H: int, I: int, Is: int, E: int, k: int) -> int:
    return lib().moe_streamed_workspace_size(T, H, I, Is, E, k)


def moe_streamed_layer_forward(lfu: "MoeLfu", layer: int, h, I: int, Is: int, E: int, k: int, router: moe_qmat,
                               bias, bias_per_row: int, shared, dev_table, ws, x_out=None, y_out=None, idx_out=None,
                               flags: int = 0, main_stream=None, side_stream=None, timeout_ms: int = 5000):
    T, H = h.shape
    arr = _qmat3(shared)
    check(lib().moe_streamed_layer_forward(lfu.handle, layer, ptr(h), T, H, I, Is, E, k, C.byref(router), ptr(bias),
                                           bias_per_row, arr, ptr(dev_table), ptr(x_out), ptr(y_out), ptr(idx_out),
                                           ptr(ws), ws.numel() * ws.element_size(), flags, stream_ptr(main_stream),
                                           stream_ptr(side_stream), timeout_ms))


# --------------------------------------------------------------- expert parallelism
def _peer_table(ptrs):
    """Host array of device pointers (ints or tensors) for a peer table."""
    return (C.c_void_p * len(ptrs))(*[ptr(p) for p in ptrs])


def moe_ep_dispatch(x, k: int, E: int, G: int, rank: int, idx, pairs, all_offsets, recv_x, recv_meta,
                    cap_rows: int, plan_offsets, plan_pairs, plan_active, plan_n_active, stream=None):
    T, H = x.shape
    check(lib().moe_ep_dispatch(ptr(x), T, H, k, E, G, rank, ptr(idx), ptr(pairs), ptr(all_offsets),
                                _peer_table(recv_x), _peer_table(recv_meta), cap_rows, ptr(plan_offsets),
                                ptr(plan_pairs), ptr(plan_active), ptr(plan_n_active), stream_ptr(stream)))


def moe_ep_return(y_rows, E: int, G: int, rank: int, recv_meta, offsets, n_pair_slots: int, y_pairs,
                  stream=None):
    cap_rows, H = y_rows.shape
    check(lib().moe_ep_return(ptr(y_rows), H, E, G, rank, ptr(recv_meta), ptr(offsets), n_pair_slots, cap_rows,
                              _peer_table(y_pairs), stream_ptr(stream)))


def moe_device_alloc(nbytes: int) -> int:
    p = C.c_void_p()
    check(lib().moe_device_alloc(nbytes, C.byref(p)))
    return p.value


def moe_device_free(p: int):
    check(lib().moe_device_free(p))


def moe_ipc_get_handle(p: int) -> bytes:
    buf = C.create_string_buffer(lib().moe_ipc_handle_bytes())
    check(lib().moe_ipc_get_handle(p, buf))
    return buf.raw


def moe_ipc_open(handle: bytes) -> int:
    p = C.c_void_p()
    check(lib().moe_ipc_open(C.c_char_p(handle), C.byref(p)))
    return p.value


def moe_ipc_close(p: int):
    check(lib().moe_ipc_close(p))
