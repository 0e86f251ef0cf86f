"""The C-ABI library loads on the host and exports every declared symbol.

No CUDA work is issued here: only symbol lookups, pure-host queries and
argument checks that fail before any launch.
"""
import ctypes as C
import os
import re

import gen

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared():
    names = []
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            names += re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported():
    from quantized_moe_bit_b200 import _lib
    L = C.CDLL(_lib.LIB_PATH)
    names = declared()
    assert len(names) >= 15
    for n in names:
        assert hasattr(L, n), n
        assert n in _lib.SIGNATURES, f"{n} has no Python binding"


def test_blob_layout_agrees_with_generator():
    import quantized_moe_bit_b200 as M
    for H, I in ((2816, 704), (256, 128), (64, 64)):
        n, offs = M.moe_blob_bytes(H, I)
        o, end = gen.blob_layout(H, I)
        assert n == end and offs == o


def test_host_argument_checks():
    from quantized_moe_bit_b200 import _lib
    L = _lib.lib()
    assert L.moe_version() >= 100
    assert L.moe_rmsnorm(None, 1, 100, 1e-6, None, None) == 1       # H % 64
    assert b"H" in L.moe_last_error_string()
    assert L.moe_bucket(None, 1, 9, 128, None, None, None, None, None) == 1   # k > 8
    assert L.moe_blob_bytes(100, 64, None) == 0


# A host address that is 16-byte aligned and non-NULL.  Every call below
# fails its argument checks (or returns early for T = 0 / L = 0) before any
# pointer is dereferenced or any CUDA call is made, so nothing ever reads
# through it; the exact status each one expects also shows that no call got
# as far as the CUDA runtime (which would answer MOE_ERR_CUDA).
_FAKE = 0x10000
_INVALID, _OK = 1, 0


def _q(out, inn, bits):
    from quantized_moe_bit_b200._lib import moe_qmat
    return moe_qmat(_FAKE, _FAKE, _FAKE, out, inn, bits)


def test_router_and_bucket_argument_checks():
    from quantized_moe_bit_b200 import _lib
    L = _lib.lib()
    r = _q(128, 2816, 8)
    f = _FAKE
    assert L.moe_router_topk(f, 1, 2800, C.byref(r), None, 0, 128, 8, f, f, None, None) == _INVALID  # H % 64
    assert L.moe_router_topk(f, 1, 2816, C.byref(r), None, 0, 100, 8, f, f, None, None) == _INVALID  # E % 8
    assert L.moe_router_topk(f, 1, 2816, C.byref(r), None, 0, 128, 9, f, f, None, None) == _INVALID  # k > 8
    assert L.moe_router_topk(None, 1, 2816, C.byref(r), None, 0, 128, 8, f, f, None, None) == _INVALID
    r4 = _q(128, 2816, 4)
    assert L.moe_router_topk(f, 1, 2816, C.byref(r4), None, 0, 128, 8, f, f, None, None) == _INVALID  # 4-bit
    rs = _q(64, 2816, 8)
    assert L.moe_router_topk(f, 1, 2816, C.byref(rs), None, 0, 128, 8, f, f, None, None) == _INVALID  # [E, H]
    assert L.moe_router_topk(f + 2, 1, 2816, C.byref(r), None, 0, 128, 8, f, f, None, None) == _INVALID  # align
    assert L.moe_router_topk(f, 0, 2816, C.byref(r), None, 0, 128, 8, f, f, None, None) == _OK        # T = 0
    assert L.moe_bucket(f, 1, 8, 100, f, f, f, f, None) == _INVALID                                  # E % 8
    assert L.moe_bucket(f, 20000, 8, 128, f, f, f, f, None) == 5             # T*k cap: MOE_ERR_UNSUPPORTED
    assert L.moe_bucket(None, 1, 8, 128, f, f, f, f, None) == _INVALID


def test_expert_shared_combine_argument_checks():
    from quantized_moe_bit_b200 import _lib
    L = _lib.lib()
    f = _FAKE
    T, H, I, Is, E, k = 4, 2816, 704, 2112, 128, 8
    ews = L.moe_expert_workspace_size(T, H, I, k)
    assert ews > 0 and L.moe_expert_workspace_size(T + 1, H, I, k) >= ews
    args = [f, T, H, I, E, k, f, f, f, f, f, f, f]
    assert L.moe_expert_forward(*args, ews - 1, 0, None) == _INVALID                    # workspace
    assert b"workspace" in L.moe_last_error_string()
    assert L.moe_expert_forward(f + 2, *args[1:], ews, 0, None) == _INVALID             # alignment
    assert L.moe_expert_forward(*args[:6], None, *args[7:], ews, 0, None) == _INVALID    # NULL blobs
    assert L.moe_expert_forward(f, T, H, 700, E, k, *args[6:], ews, 0, None) == _INVALID  # I % 64
    assert L.moe_expert_forward(*args, ews, 8, None) == _INVALID                        # unknown flag bit
    assert L.moe_expert_forward(*args, ews, 3, None) == _INVALID                        # GEMV and TC together
    assert L.moe_expert_forward(f, 0, H, I, E, k, *args[6:], 0, 0, None) == _OK         # T = 0
    sh = (_lib.moe_qmat * 3)(_q(Is, H, 4), _q(Is, H, 4), _q(H, Is, 4))
    sws = L.moe_shared_workspace_size(T, H, Is)
    assert sws > 0
    assert L.moe_shared_forward(f, T, H, Is, sh, f, f, sws - 1, 0, None) == _INVALID    # workspace
    bad = (_lib.moe_qmat * 3)(_q(Is, H, 4), _q(Is, H, 8), _q(H, Is, 4))
    assert L.moe_shared_forward(f, T, H, Is, bad, f, f, sws, 0, None) == _INVALID       # 8-bit up
    shape = (_lib.moe_qmat * 3)(_q(Is, H, 4), _q(Is, H, 4), _q(Is, H, 4))
    assert L.moe_shared_forward(f, T, H, Is, shape, f, f, sws, 0, None) == _INVALID     # down is [H, Is]
    mis = (_lib.moe_qmat * 3)(_q(Is, H, 4), _q(Is, H, 4), _q(H, Is, 4))
    mis[1].s = f + 8
    assert L.moe_shared_forward(f, T, H, Is, mis, f, f, sws, 0, None) == _INVALID       # misaligned scales
    assert L.moe_combine(f, f, f, T, H, 9, f, None, None) == _INVALID                   # k > 8
    assert L.moe_combine(None, f, f, T, H, k, f, None, None) == _INVALID
    assert L.moe_combine(f, f, f, 0, H, k, f, None, None) == _OK


def test_layer_and_decode_argument_checks():
    from quantized_moe_bit_b200 import _lib
    L = _lib.lib()
    f = _FAKE
    T, H, I, Is, E, k = 2, 2816, 704, 2112, 128, 8
    r = _q(E, H, 8)
    sh = (_lib.moe_qmat * 3)(_q(Is, H, 4), _q(Is, H, 4), _q(H, Is, 4))
    lws = L.moe_layer_workspace_size(T, H, I, Is, E, k)
    assert lws >= L.moe_expert_workspace_size(T, H, I, k) + L.moe_shared_workspace_size(T, H, Is)
    tail = [T, H, I, Is, E, k, C.byref(r), None, 0, f, sh, None, None, None, None]
    assert L.moe_layer_forward(None, None, None, *tail, f, lws, 0, None) == _INVALID    # no input
    assert L.moe_layer_forward(None, f, f, *tail, f, lws, 0, None) == _INVALID          # h_out without h_in
    assert L.moe_layer_forward(f, f, None, *tail, f, lws - 1, 0, None) == _INVALID      # workspace
    assert L.moe_layer_forward(f, f, None, *tail, f, lws, 16, None) == _INVALID         # unknown flag bit
    dws = L.moe_decode_workspace_size(1, H, I, Is, E, k)
    assert dws >= L.moe_layer_workspace_size(1, H, I, Is, E, k)
    routers = (_lib.moe_qmat * 2)(r, r)
    shared = (_lib.moe_qmat * 6)(*(list(sh) * 2))
    blobs = (C.c_void_p * 2)(f, f)
    d = [1, H, I, Is, E, k]
    assert L.moe_decode_forward(f, *d, -1, routers, None, 0, blobs, shared, None, None, None, None, f, dws,
                                0, None) == _INVALID                                     # L < 0
    assert L.moe_decode_forward(f, *d, 2, routers, None, 0, blobs, shared, None, None, None, None, f, dws - 1,
                                0, None) == _INVALID                                     # workspace
    assert L.moe_decode_forward(None, *d, 2, routers, None, 0, blobs, shared, None, None, None, None, f, dws,
                                0, None) == _INVALID                                     # NULL h
    assert L.moe_decode_forward(f, *d, 0, routers, None, 0, blobs, shared, None, None, None, None, f, dws,
                                0, None) == _OK                                          # L = 0
    assert L.moe_decode_launches(1, 30, 0) == 1 and L.moe_decode_launches(1, 30, 4) == 240
    assert L.moe_decode_launches(64, 30, 0) == 210 and L.moe_decode_launches(64, 30, 1) == 240


def test_noalloc_argument_checks_come_before_any_cuda_call():
    """Every rejected request of the no-allocation entry point is rejected by
    its own checks (MOE_ERR_INVALID_ARG), before the scratch lookup or any
    other CUDA call (which, without a GPU, would answer MOE_ERR_CUDA)."""
    from quantized_moe_bit_b200 import _lib
    L = _lib.lib()
    f = _FAKE
    H, I, E, k = 2816, 704, 128, 8
    limit = 4 * 1024 * 1024
    T_max = max(T for T in range(1, 400) if L.moe_expert_workspace_size(T, H, I, k) <= limit)
    rest = [f, f, f, f, f, f]
    assert L.moe_expert_forward_noalloc(f, T_max + 1, H, I, E, k, *rest, None) == _INVALID   # beyond the scratch
    assert b"static scratch" in L.moe_last_error_string()
    assert L.moe_expert_forward_noalloc(None, T_max, H, I, E, k, *rest, None) == _INVALID    # NULL x
    assert L.moe_expert_forward_noalloc(f, 4, H, I, E, k, None, *rest[1:], None) == _INVALID  # NULL blob table
    assert L.moe_expert_forward_noalloc(f, 4, H, I, E, k, *rest[:5], None, None) == _INVALID  # NULL y_pairs
    assert L.moe_expert_forward_noalloc(f + 4, 4, H, I, E, k, *rest, None) == _INVALID        # misaligned x
    assert L.moe_expert_forward_noalloc(f, 4, H, 100, E, k, *rest, None) == _INVALID          # I % 64
    assert L.moe_expert_forward_noalloc(f, 0, H, I, E, k, *rest, None) == _OK                 # T = 0


def test_expert_parallel_argument_checks():
    from quantized_moe_bit_b200 import _lib
    L = _lib.lib()
    f = _FAKE
    T, H, k, E = 4, 2816, 8, 128
    peers = lambda n, bad=None: (C.c_void_p * 8)(*[(bad if i == 0 and bad is not None else f) for i in range(n)])  # noqa: E731
    ok2 = peers(2)
    d = lambda *a: L.moe_ep_dispatch(*a[:-1], f, f, f, f, None)  # noqa: E731  (plan outputs, stream)
    assert d(f, T, H, k, E, 0, 0, f, f, f, ok2, ok2, 64, None) == _INVALID               # G = 0
    assert d(f, T, H, k, E, 9, 0, f, f, f, peers(8), peers(8), 64, None) == _INVALID      # G > 8
    assert d(f, T, H, k, 24, 2, 0, f, f, f, ok2, ok2, 64, None) == _INVALID              # E/G = 12
    assert d(f, T, H, k, E, 2, 2, f, f, f, ok2, ok2, 64, None) == _INVALID               # rank >= G
    assert d(f, T, H, k, E, 2, 0, f, f, f, peers(2, 0), ok2, 64, None) == _INVALID       # NULL peer
    assert d(f, T, H, k, E, 2, 0, f, f, f, ok2, peers(2, f + 4), 64, None) == _INVALID   # misaligned peer
    assert d(f + 2, T, H, k, E, 2, 0, f, f, f, ok2, ok2, 64, None) == _INVALID           # misaligned x
    assert d(f, T, H, k, E, 2, 0, f, f, f, None, ok2, 64, None) == _INVALID              # no table
    assert d(f, T, H, k, E, 2, 0, f, f, f, ok2, ok2, -1, None) == _INVALID               # capacity
    assert L.moe_ep_dispatch(f, T, H, k, E, 2, 0, f, f, f, ok2, ok2, 64, None, f, f, f, None) == _INVALID  # plan
    assert L.moe_ep_return(f, H, E, 2, 0, f, f, 32, 64, peers(2, 0), None) == _INVALID   # NULL peer
    assert L.moe_ep_return(f, H, E, 2, 0, f + 4, f, 32, 64, ok2, None) == _INVALID       # meta alignment
    assert L.moe_ep_return(f, H, E, 2, 0, f, f, 32, 0, ok2, None) == _OK                 # nothing received
    assert L.moe_ipc_handle_bytes() == 64
    assert L.moe_ipc_open(None, None) == _INVALID
    assert L.moe_device_alloc(0, C.byref(C.c_void_p())) == _INVALID


def test_decode_session_argument_checks():
    from quantized_moe_bit_b200 import _lib
    L = _lib.lib()
    f = _FAKE
    H, I, Is, E, k = 2816, 704, 2112, 128, 8
    r = _q(E, H, 8)
    routers = (_lib.moe_qmat * 1)(r)
    sh = (_lib.moe_qmat * 3)(_q(Is, H, 4), _q(Is, H, 4), _q(H, Is, 4))
    blobs = (C.c_void_p * 1)(f)
    out = C.c_void_p()
    dws = L.moe_decode_workspace_size(1, H, I, Is, E, k)
    args = [f, H, I, Is, E, k, 1, routers, None, 0, blobs, sh, f, dws, 0]
    assert L.moe_decode_session_create(*args, None) == _INVALID                          # no out
    assert L.moe_decode_session_create(*args[:6], 0, *args[7:], C.byref(out)) == _INVALID  # L = 0
    assert L.moe_decode_session_create(*args[:13], dws - 1, 0, C.byref(out)) == _INVALID  # workspace
    assert L.moe_decode_session_create(f + 4, *args[1:], C.byref(out)) == _INVALID        # misaligned h
    bad = (_lib.moe_qmat * 1)(_q(E, H, 4))
    assert L.moe_decode_session_create(*args[:7], bad, *args[8:], C.byref(out)) == _INVALID  # 4-bit router
    assert out.value is None
    assert L.moe_decode_session_step(None, f, f) == _INVALID
    assert L.moe_decode_session_destroy(None) == _OK


def test_header_is_plain_c(tmp_path):
    """include/moe.h compiles as C99 with warnings as errors (the boundary
    carries no C++ or torch types)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        import pytest
        pytest.skip("no C compiler")
    src = tmp_path / "use_header.c"
    src.write_text('#include "moe.h"\nint main(void) { return moe_version() > 0 ? 0 : 1; }\n')
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-I",
                        os.path.join(ROOT, "include"), str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
