"""GPU parity of each C-ABI call and of a whole layer against the fp64 oracle.

Inputs: seeded generator rows; candidate rows whose oracle logits have a gap
below 1e-3 among the k+1 largest are redrawn (so routing is decided by the
data, not by rounding) unless a test says otherwise.
"""
import numpy as np
import pytest
import torch

import gen
from dataclasses import replace

from gen import tiny_config, CONFIGS
from oracle import moe_oracle as O
from tests._support import HostLayer, check_close, check_output, check_routing, gap_ok_predicate

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    import quantized_moe_bit_b200 as M
    return M


def _np(t):
    return t.detach().cpu().numpy()


def _bits(t):
    return _np(t.view(torch.int16)).view(np.uint16)


def _run_calls(M, hl, dl, z, flags=0):
    """Run A0..A7 through the separate calls (expert path per `flags`);
    return every intermediate."""
    c = hl.cfg
    T = z.shape[0]
    dev = "cuda"
    h = torch.from_numpy(z).to(dev)
    x = torch.empty((T, c.H), dtype=torch.int16, device=dev)
    M.moe_rmsnorm(h, x)
    idx = torch.empty((T, c.k), dtype=torch.int32, device=dev)
    gates = torch.empty((T, c.k), dtype=torch.float32, device=dev)
    logits = torch.empty((T, c.E), dtype=torch.float32, device=dev)
    M.moe_router_topk(x, dl.router.c, dl.bias, 0, c.E, c.k, idx, gates, logits)
    offs = torch.empty(c.E + 1, dtype=torch.int32, device=dev)
    pairs = torch.empty(T * c.k, dtype=torch.int32, device=dev)
    active = torch.empty(c.E, dtype=torch.int32, device=dev)
    n_active = torch.empty(1, dtype=torch.int32, device=dev)
    M.moe_bucket(idx, c.E, offs, pairs, active, n_active)
    yp = torch.empty((T * c.k, c.H), dtype=torch.float32, device=dev)
    ws = torch.empty(M.moe_expert_workspace_size(T, c.H, c.I, c.k), dtype=torch.uint8, device=dev)
    M.moe_expert_forward(x, c.I, c.E, c.k, dl.blob_ptrs, offs, pairs, active, n_active, yp, ws, flags=flags)
    ysh = torch.empty((T, c.H), dtype=torch.float32, device=dev)
    wss = torch.empty(M.moe_shared_workspace_size(T, c.H, c.Is), dtype=torch.uint8, device=dev)
    M.moe_shared_forward(x, c.Is, dl.shared_c, ysh, wss, flags=flags)
    y = torch.empty((T, c.H), dtype=torch.int16, device=dev)
    resid = h.clone()
    M.moe_combine(yp, gates, ysh, y, resid)
    M.moe_sync()
    return dict(x=_bits(x), idx=_np(idx), gates=_np(gates), logits=_np(logits), offsets=_np(offs),
                pairs=_np(pairs), active=_np(active), n_active=int(_np(n_active)[0]), y_pairs=_np(yp),
                ysh=_np(ysh), y=_bits(y), resid=_np(resid))


def _check_all(hl, z, g):
    c = hl.cfg
    T = z.shape[0]
    # A0: bf16 x equals the oracle's except where the fp64 value sits within
    # fp32 rounding of a bf16 midpoint (then they differ by one unit)
    xb_o, _ = O.rmsnorm(z.astype(np.float64))
    diff = np.abs(g["x"].astype(np.int32) - xb_o.astype(np.int32))
    assert diff.max() <= 1 and (diff > 0).mean() < 1e-3
    x = O.bf16_to_f64(g["x"])               # teacher forcing: the GPU's layer input
    lg = O.router_logits(x, hl.router, hl.bias)
    check_close(g["logits"], lg, 1e-5, 1e-6, "logits")
    check_routing(g["idx"], lg, c.k)
    g_o = O.softmax_gates(lg, g["idx"])
    assert np.abs(g["gates"] - g_o).max() < 2e-6
    off, pairs, active = O.buckets(g["idx"], c.E)
    assert np.array_equal(g["offsets"], off) and np.array_equal(g["pairs"], pairs)
    assert g["n_active"] == len(active) and np.array_equal(g["active"][:len(active)], active)
    r = O.layer_forward(x, hl.router, hl.bias, hl.expert, hl.shared, c.k, c.E, idx=g["idx"])
    check_close(g["y_pairs"], r["y_pairs"], 2e-3, 2e-4, "y_pairs")
    check_close(g["ysh"], r["ysh"], 2e-3, 2e-4, "ysh")
    check_output(g["y"], r["out"], "y")
    check_close(g["resid"], z.astype(np.float64) + r["out"], 2e-3, 2e-4, "h + y")


@pytest.mark.parametrize("T", [1, 3, 37])
def test_calls_tiny(M, T):
    cfg = tiny_config("prefill_1L_128tok", T=T)
    hl = HostLayer(cfg, 0)
    z = gen.rows(cfg.seed, 1000, T, cfg.H, accept=gap_ok_predicate(hl))
    g = _run_calls(M, hl, hl.upload(), z)
    _check_all(hl, z, g)


def test_calls_single_layer_full(M):
    cfg = CONFIGS["single_layer_1tok"]
    hl = HostLayer(cfg, 0)
    z = gen.rows(cfg.seed, 1000, 1, cfg.H, accept=gap_ok_predicate(hl))
    g = _run_calls(M, hl, hl.upload(), z)
    _check_all(hl, z, g)


@pytest.mark.parametrize("T", [2, 19, 150])
def test_layer_forward_matches_calls_and_is_deterministic(M, T):
    """The whole-layer call (routed buckets and shared expert in one grouped
    launch per projection when T > 2) equals the separate calls bit for bit,
    and repeats bit for bit."""
    cfg = tiny_config("prefill_1L_128tok", T=T)
    hl = HostLayer(cfg, 0)
    dl = hl.upload()
    z = gen.rows(cfg.seed, 1000, cfg.T, cfg.H)
    g = _run_calls(M, hl, dl, z)
    c = cfg
    outs = []
    for _ in range(2):
        h = torch.from_numpy(z).cuda()
        ho = torch.empty_like(h)
        y = torch.empty((c.T, c.H), dtype=torch.int16, device="cuda")
        idx = torch.empty((c.T, c.k), dtype=torch.int32, device="cuda")
        ws = torch.empty(M.moe_layer_workspace_size(c.T, c.H, c.I, c.Is, c.E, c.k), dtype=torch.uint8, device="cuda")
        M.moe_layer_forward(c.T, c.H, c.I, c.Is, c.E, c.k, dl.router.c, dl.bias, 0, dl.blob_ptrs, dl.shared_c, ws,
                            h_in=h, h_out=ho, y=y, idx=idx)
        M.moe_sync()
        outs.append((_bits(y), _np(ho), _np(idx)))
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
    assert np.array_equal(outs[0][0], g["y"]) and np.array_equal(outs[0][2], g["idx"])
    assert np.array_equal(outs[0][1], g["resid"])


def test_empty_and_invalid(M):
    cfg = tiny_config("prefill_1L_128tok", T=0)
    hl = HostLayer(cfg, 0)
    dl = hl.upload()
    c = cfg
    x = torch.empty((0, c.H), dtype=torch.int16, device="cuda")
    idx = torch.empty((0, c.k), dtype=torch.int32, device="cuda")
    gates = torch.empty((0, c.k), dtype=torch.float32, device="cuda")
    M.moe_router_topk(x, dl.router.c, None, 0, c.E, c.k, idx, gates)      # T = 0 is a no-op
    with pytest.raises(M.MoeError) as ei:
        M.moe_router_topk(x, dl.router.c, None, 0, c.E, 9, idx, gates)   # k > 8
    assert ei.value.status == 1
    bad = torch.empty((1, 100), dtype=torch.int16, device="cuda")       # H not a multiple of 64
    with pytest.raises(M.MoeError):
        M.moe_rmsnorm(torch.empty((1, 100), device="cuda"), bad)
    M.moe_sync()


@pytest.mark.parametrize("flags", [0, 1, 2])
@pytest.mark.parametrize("T", [1, 3, 37, 130])
def test_expert_paths_tiny(M, T, flags):
    """GEMV (flag 1), grouped tensor-core GEMM (flag 2) and the library's
    choice (0) against the oracle.  T = 1 on the GEMM pads one-row buckets to
    16 MMA columns; T = 130 gives buckets above 128 rows (several chunks)."""
    cfg = tiny_config("prefill_1L_128tok", T=T)
    hl = HostLayer(cfg, 0)
    z = gen.rows(cfg.seed, 1000, T, cfg.H, accept=gap_ok_predicate(hl))
    g = _run_calls(M, hl, hl.upload(), z, flags=flags)
    _check_all(hl, z, g)


@pytest.mark.parametrize("flags", [0, 1])
def test_prefill_128_full(M, flags):
    """The 128-row prefill chunk at full size (H=2816, E=128, I=704) on the
    grouped GEMM (0) and on the GEMV kernels (1)."""
    cfg = CONFIGS["prefill_1L_128tok"]
    hl = HostLayer(cfg, 0)
    z = gen.rows(cfg.seed, 1000, cfg.T, cfg.H, accept=gap_ok_predicate(hl))
    g = _run_calls(M, hl, hl.upload(), z, flags=flags)
    _check_all(hl, z, g)


def test_prefill_large_chunk_full(M):
    """Large prefill chunk (512 rows of the prefill workload's shapes and
    routing skew) through the whole-layer call: routing, buckets and every
    output row against the oracle; the largest buckets span several
    128-row chunks of the grouped GEMM."""
    cfg = replace(CONFIGS["prefill_1L_128tok"], T=512)
    c = cfg
    hl = HostLayer(cfg, 0)
    dl = hl.upload()
    z = gen.rows(c.seed, 2000, c.T, c.H, accept=gap_ok_predicate(hl))
    h = torch.from_numpy(z).cuda()
    ho = torch.empty_like(h)
    x = torch.empty((c.T, c.H), dtype=torch.int16, device="cuda")
    y = torch.empty((c.T, c.H), dtype=torch.int16, device="cuda")
    idx = torch.empty((c.T, c.k), dtype=torch.int32, device="cuda")
    gates = torch.empty((c.T, c.k), dtype=torch.float32, device="cuda")
    ws = torch.empty(M.moe_layer_workspace_size(c.T, c.H, c.I, c.Is, c.E, c.k), dtype=torch.uint8, device="cuda")
    M.moe_layer_forward(c.T, c.H, c.I, c.Is, c.E, c.k, dl.router.c, dl.bias, 0, dl.blob_ptrs, dl.shared_c, ws,
                        h_in=h, h_out=ho, x_out=x, y=y, idx=idx, gates=gates)
    M.moe_sync()
    xg = O.bf16_to_f64(_bits(x))
    lg = O.router_logits(xg, hl.router, hl.bias)
    gi = _np(idx)
    check_routing(gi, lg, c.k)
    off, _, active = O.buckets(gi, c.E)
    assert int(np.diff(off).max()) > 128                       # several chunks for the top expert
    assert np.abs(_np(gates) - O.softmax_gates(lg, gi)).max() < 2e-6
    r = O.layer_forward(xg, hl.router, hl.bias, hl.expert, hl.shared, c.k, c.E, idx=gi)
    check_output(_bits(y), r["out"], "y (512 rows)")
    check_close(_np(ho), z.astype(np.float64) + r["out"], 2e-3, 2e-4, "h + y (512 rows)")
