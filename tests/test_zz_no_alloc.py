"""moe_expert_forward_noalloc: the routed-expert forward for callers that
cannot allocate device memory (no workspace argument; its scratch is a static
array inside the library).

Checked through the C-ABI against moe_expert_forward with a caller workspace,
on two calls in a row with different inputs, and for the size limit.  Both
calls run the same kernels on the same inputs and differ only in where the
scratch lives, and every kernel on the path is deterministic, so the outputs
must be equal bit for bit.  This file is collected last so that a run
stopping at the first failure has already run every other test.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import gen
from gen import tiny_config, CONFIGS
from tests._support import HostLayer

pytestmark = pytest.mark.gpu


def _buckets(M, hl, dl, z):
    c = hl.cfg
    T = z.shape[0]
    h = torch.from_numpy(z).cuda()
    x = torch.empty((T, c.H), dtype=torch.int16, device="cuda")
    M.moe_rmsnorm(h, x)
    idx = torch.empty((T, c.k), dtype=torch.int32, device="cuda")
    gates = torch.empty((T, c.k), dtype=torch.float32, device="cuda")
    M.moe_router_topk(x, dl.router.c, dl.bias, 0, c.E, c.k, idx, gates)
    offs = torch.empty(c.E + 1, dtype=torch.int32, device="cuda")
    pairs = torch.empty(T * c.k, dtype=torch.int32, device="cuda")
    active = torch.empty(c.E, dtype=torch.int32, device="cuda")
    n_active = torch.empty(1, dtype=torch.int32, device="cuda")
    M.moe_bucket(idx, c.E, offs, pairs, active, n_active)
    return x, offs, pairs, active, n_active


@pytest.mark.parametrize("which,T", [("tiny", 37), ("full", 16), ("full", 70)])
def test_noalloc_matches_workspace_entry_on_two_calls(which, T):
    import quantized_moe_bit_b200 as M
    cfg = tiny_config("prefill_1L_128tok", T=T) if which == "tiny" else replace(CONFIGS["prefill_1L_128tok"], T=T)
    c = cfg
    hl = HostLayer(cfg, 0)
    dl = hl.upload()
    for call, stream in enumerate((1000, 1001)):      # two calls in a row, different inputs
        z = gen.rows(c.seed, stream, T, c.H)
        x, offs, pairs, active, n_active = _buckets(M, hl, dl, z)
        y_ref = torch.full((T * c.k, c.H), float("nan"), dtype=torch.float32, device="cuda")
        ws = torch.empty(M.moe_expert_workspace_size(T, c.H, c.I, c.k), dtype=torch.uint8, device="cuda")
        M.moe_expert_forward(x, c.I, c.E, c.k, dl.blob_ptrs, offs, pairs, active, n_active, y_ref, ws)
        y = torch.full((T * c.k, c.H), float("nan"), dtype=torch.float32, device="cuda")
        M.moe_expert_forward_noalloc(x, c.I, c.E, c.k, dl.blob_ptrs, offs, pairs, active, n_active, y)
        M.moe_sync()
        assert torch.isfinite(y).all(), f"call {call}: unwritten rows"
        assert torch.equal(y, y_ref), f"call {call}: differs from the workspace entry point"


def test_noalloc_rejects_requests_beyond_the_static_scratch():
    import quantized_moe_bit_b200 as M
    c = CONFIGS["prefill_1L_128tok"]
    T = 71                                   # 71 rows need more than the 4 MiB scratch
    x = torch.empty((T, c.H), dtype=torch.int16, device="cuda")
    dummy = torch.empty(1024, dtype=torch.int32, device="cuda")
    y = torch.empty((1,), dtype=torch.float32, device="cuda")
    with pytest.raises(M.MoeError) as ei:
        M.moe_expert_forward_noalloc(x, c.I, c.E, c.k, dummy, dummy, dummy, dummy, dummy, y)
    assert ei.value.status == 1 and "static scratch" in str(ei.value)
    M.moe_sync()
