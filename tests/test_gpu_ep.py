"""GPU parity of the expert-parallel layer (quantized_moe_bit_b200.ep).

G ranks run in this process on one GPU (`LocalRanks`): the dispatch and
return kernels store into the ranks' own buffers through the same peer
tables and receiver layout they use across GPUs.  Per layer and rank, the
oracle recomputes the layer from the rank's own GPU layer input and routing
(teacher forcing), and the bf16 output and the residual update are checked
against it.  The process-group path (`EpComm` over NCCL) runs with one rank.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

import gen
from gen import CONFIGS, tiny_config
from dataclasses import replace
from oracle import moe_oracle as O
from tests._support import HostLayer, check_close, check_output, check_routing

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    import quantized_moe_bit_b200 as M
    return M


def _np(t):
    return t.detach().cpu().numpy()


def _bits(t):
    return _np(t.view(torch.int16)).view(np.uint16)


def _run_layers(M, cfg, G, layers, z_by_rank, bias_override=None):
    """Run `layers` layers of the EP path over G local ranks; check every rank
    and layer against the oracle; return per-rank received row counts."""
    from quantized_moe_bit_b200 import ep
    c = cfg
    hls = [HostLayer(cfg, l) for l in range(layers)]
    dls = [hl.upload() for hl in hls]
    if bias_override is not None:
        for hl, dl in zip(hls, dls):
            hl.bias = bias_override
            dl.bias = torch.from_numpy(bias_override.astype(np.float32)).cuda()
    ranks = [ep.EpRank(G, r, c.T, c.H, c.I, c.Is, c.E, c.k, dls[0]) for r in range(G)]
    comm = ep.LocalRanks(ranks)
    hs = [torch.from_numpy(z).cuda() for z in z_by_rank]
    received = []
    for l in range(layers):
        for r in ranks:
            r.set_layer(dls[l])
        before = [_np(h).astype(np.float64) for h in hs]
        ep.ep_layer_forward(ranks, comm, hs)
        M.moe_sync()
        received.append([int(_np(r.loff)[-1]) for r in ranks])
        for g, r in enumerate(ranks):
            x = O.bf16_to_f64(_bits(r.x))
            idx = _np(r.idx)
            lg = O.router_logits(x, hls[l].router, hls[l].bias)
            check_routing(idx, lg, c.k)
            ref = O.layer_forward(x, hls[l].router, hls[l].bias, hls[l].expert, hls[l].shared, c.k, c.E, idx=idx)
            assert np.abs(_np(r.gates) - ref["gates"]).max() < 2e-6, f"gates l{l} r{g}"
            check_output(_bits(r.y), ref["out"], f"y l{l} r{g}")
            check_close(_np(hs[g]), before[g] + ref["out"], 2e-3, 2e-4, f"h l{l} r{g}")
        # every pair of every rank was received exactly once
        assert sum(received[-1]) == G * c.T * c.k
    for r in ranks:
        r.close()
    return received


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_ep_local_ranks_tiny(M, G):
    cfg = tiny_config("prefill_1L_128tok", T=5, E=64)
    zs = [gen.rows(cfg.seed, 1000 + g, cfg.T, cfg.H) for g in range(G)]
    rec = _run_layers(M, cfg, G, 2, zs)
    if G > 1:
        # several owners received rows (with the Zipf routing skew some of
        # the 8-expert ranges may stay empty)
        assert sum(n > 0 for n in rec[0]) >= 2


@pytest.mark.parametrize("G,T", [(4, 16), (8, 16)])
def test_ep_local_ranks_full_size(M, G, T):
    cfg = replace(CONFIGS["prefill_1L_128tok"], T=T)
    zs = [gen.rows(cfg.seed, 1000 + g, cfg.T, cfg.H) for g in range(G)]
    _run_layers(M, cfg, G, 1, zs)


def test_ep_all_pairs_to_one_rank(M):
    """Every pair of every rank routed to rank 0's experts: rank 0 receives
    its full capacity, the others nothing (empty receivers)."""
    G = 4
    cfg = tiny_config("prefill_1L_128tok", T=7, E=64)
    El = cfg.E // G
    bias = gen.forced_bias(np.arange(cfg.k, dtype=np.int32)[None, :], cfg.E)[0].astype(np.float64)
    assert set(np.argsort(-bias)[:cfg.k]) <= set(range(El))
    zs = [gen.rows(cfg.seed, 1000 + g, cfg.T, cfg.H) for g in range(G)]
    rec = _run_layers(M, cfg, G, 1, zs, bias_override=bias)
    assert rec[0] == [G * cfg.T * cfg.k, 0, 0, 0]


def test_ep_process_group_one_rank(M):
    """EpComm over NCCL (one rank): the collectives, the peer tables of a
    process-per-rank run and the layer against the oracle."""
    import torch.distributed as dist
    from quantized_moe_bit_b200 import ep
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    store = dist.TCPStore("127.0.0.1", port, 1, True, timeout=datetime.timedelta(seconds=30))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        cfg = tiny_config("prefill_1L_128tok", T=9, E=64)
        hl = HostLayer(cfg, 0)
        dl = hl.upload()
        r = ep.EpRank(1, 0, cfg.T, cfg.H, cfg.I, cfg.Is, cfg.E, cfg.k, dl)
        comm = ep.EpComm(device="cuda")
        ep.connect(r, comm)
        z = gen.rows(cfg.seed, 1000, cfg.T, cfg.H)
        h = torch.from_numpy(z).cuda()
        ep.ep_layer_forward([r], comm, [h])
        M.moe_sync()
        x = O.bf16_to_f64(_bits(r.x))
        ref = O.layer_forward(x, hl.router, hl.bias, hl.expert, hl.shared, cfg.k, cfg.E, idx=_np(r.idx))
        check_output(_bits(r.y), ref["out"], "y")
        check_close(_np(h), z.astype(np.float64) + ref["out"], 2e-3, 2e-4, "h")
        assert np.array_equal(_np(r.all_off)[0], _np(r.offsets))
        r.close()
    finally:
        dist.destroy_process_group()


def test_ep_layer_replays_from_a_cuda_graph(M):
    """The whole expert-parallel layer of 2 local ranks captured in one CUDA
    graph (no host synchronisation inside) replays bit for bit like the
    eager calls."""
    from quantized_moe_bit_b200 import ep
    G = 2
    cfg = tiny_config("prefill_1L_128tok", T=6)
    hl = HostLayer(cfg, 0)
    dl = hl.upload()
    ranks = [ep.EpRank(G, r, cfg.T, cfg.H, cfg.I, cfg.Is, cfg.E, cfg.k, dl) for r in range(G)]
    comm = ep.LocalRanks(ranks)
    zs = [torch.from_numpy(gen.rows(cfg.seed, 1000 + g, cfg.T, cfg.H)).cuda() for g in range(G)]
    hs = [z.clone() for z in zs]
    ep.ep_layer_forward(ranks, comm, hs)
    M.moe_sync()
    want = [(_np(h), _bits(r.y)) for h, r in zip(hs, ranks)]
    hs_g = [z.clone() for z in zs]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):                       # warm-up outside the capture
        ep.ep_layer_forward(ranks, comm, hs_g)
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        ep.ep_layer_forward(ranks, comm, hs_g)
    for _ in range(2):
        for h, z in zip(hs_g, zs):
            h.copy_(z)
        graph.replay()
        torch.cuda.synchronize()
        M.moe_sync()
        for (h_w, y_w), h, r in zip(want, hs_g, ranks):
            assert np.array_equal(_np(h), h_w) and np.array_equal(_bits(r.y), y_w)
    del graph
    for r in ranks:
        r.close()


def test_ep_exportable_buffers_one_rank(M):
    """A rank whose receive buffers are whole device allocations exportable
    by CUDA IPC (moe_device_alloc): the layer runs on them, their IPC
    handles are produced, and close() frees them."""
    from quantized_moe_bit_b200 import ep
    cfg = tiny_config("prefill_1L_128tok", T=4, E=64)
    hl = HostLayer(cfg, 0)
    dl = hl.upload()
    r = ep.EpRank(1, 0, cfg.T, cfg.H, cfg.I, cfg.Is, cfg.E, cfg.k, dl, exportable=True)
    handles = r.ipc_handles()
    assert len(handles) == 3 and all(len(h) == 64 for h in handles)
    comm = ep.LocalRanks([r])
    z = gen.rows(cfg.seed, 1000, cfg.T, cfg.H)
    h = torch.from_numpy(z).cuda()
    ep.ep_layer_forward([r], comm, [h])
    M.moe_sync()
    x = O.bf16_to_f64(_bits(r.x))
    ref = O.layer_forward(x, hl.router, hl.bias, hl.expert, hl.shared, cfg.k, cfg.E, idx=_np(r.idx))
    check_output(_bits(r.y), ref["out"], "y")
    r.close()
    assert r._raw == []
