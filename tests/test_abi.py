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
    assert L.moe_set_gemv_max_rows(-1) == 1
    assert L.moe_blob_bytes(100, 64, None) == 0
