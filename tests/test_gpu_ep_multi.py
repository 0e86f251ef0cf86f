"""The expert-parallel layer across two processes on two GPUs: NCCL
collectives (offsets all-gather, stream-ordered barriers), receive buffers
exported by CUDA IPC and mapped by the peer, the exchange kernels storing
over NVLink.  Each rank's output against the oracle on its own tokens.

Needs two GPUs: skipped where fewer are visible.  No rank waits inside a
kernel for another (the exchanges are stores; the waits are NCCL
collectives between kernels), and nothing uses NVLink multicast.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

WORLD = 2


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, port, q):
    import torch.distributed as dist
    import gen
    from gen import tiny_config
    from oracle import moe_oracle as O
    from tests._support import HostLayer, check_close, check_output
    import quantized_moe_bit_b200 as M
    from quantized_moe_bit_b200 import ep
    os.environ["NCCL_NVLS_ENABLE"] = "0"
    dev = torch.device("cuda", rank)
    torch.cuda.set_device(dev)
    store = dist.TCPStore("127.0.0.1", port, WORLD, rank == 0, timeout=datetime.timedelta(seconds=60))
    dist.init_process_group("nccl", store=store, rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=60), device_id=dev)
    r = None
    try:
        cfg = tiny_config("prefill_1L_128tok", T=6)
        hl = HostLayer(cfg, 0)
        dl = hl.upload(dev)
        r = ep.EpRank(WORLD, rank, cfg.T, cfg.H, cfg.I, cfg.Is, cfg.E, cfg.k, dl, device=dev, exportable=True)
        comm = ep.EpComm(device=dev)
        ep.connect(r, comm)
        z = gen.rows(cfg.seed, 1000 + rank, cfg.T, cfg.H)
        h = torch.from_numpy(z).to(dev)
        ep.ep_layer_forward([r], comm, [h])
        torch.cuda.synchronize(dev)
        M.moe_sync()
        x = O.bf16_to_f64(r.x.cpu().numpy().view(np.uint16))
        ref = O.layer_forward(x, hl.router, hl.bias, hl.expert, hl.shared, cfg.k, cfg.E, idx=r.idx.cpu().numpy())
        check_output(r.y.cpu().numpy().view(np.uint16), ref["out"], f"rank {rank} y")
        check_close(h.cpu().numpy(), z.astype(np.float64) + ref["out"], 2e-3, 2e-4, f"rank {rank} h")
        # rows of this rank crossed to the other rank's experts
        idx = r.idx.cpu().numpy()
        q.put((rank, "ok", int((idx // (cfg.E // WORLD) != rank).sum())))
    except Exception as exc:       # reported to the parent, which fails the test
        q.put((rank, repr(exc), 0))
    finally:
        dist.barrier()             # no peer writes into the buffers after this
        if r is not None:
            r.close()
        dist.destroy_process_group()


@pytest.mark.skipif(torch.cuda.device_count() < WORLD, reason="needs two GPUs")
def test_ep_two_gpus_nccl_ipc():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(rk, port, q)) for rk in range(WORLD)]
    for p in ps:
        p.start()
    res = [q.get(timeout=300) for _ in range(WORLD)]
    for p in ps:
        p.join(timeout=120)
        assert p.exitcode == 0
    for rank, status, crossed in res:
        assert status == "ok", (rank, status)
        assert crossed > 0, rank
