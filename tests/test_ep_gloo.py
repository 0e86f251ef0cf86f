"""The expert-parallel layer schedule (quantized_moe_bit_b200.ep) across two
gloo ranks on the CPU.

The product's schedule (`ep_layer_forward`) and collectives (`EpComm`) run
unchanged; each rank's steps are host stand-ins computed with the oracle, and
the peers' buffers are shared-memory CPU tensors that the ranks store into
directly, as the kernels store into peer GPU memory.  The stand-ins place rows
by the receiver layout as the C-ABI header defines it.  Two layers in a row
(buffers reused across layers), and the result of every rank equals the
one-process oracle layer on that rank's tokens.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import gen
from gen import tiny_config
from oracle import moe_oracle as O

CFG = tiny_config("prefill_1L_128tok", T=5)
WORLD = 2


def _cfg(world):
    # E/world experts per rank, a multiple of 8
    return CFG if world == 2 else tiny_config("prefill_1L_128tok", T=5, E=8 * world)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


class HostEpRank:
    """Oracle stand-in of EpRank's steps on host buffers."""

    def __init__(self, G, rank, cfg, recv_x, recv_meta, y_pairs):
        self.G, self.rank, self.c = G, rank, cfg
        self.El = cfg.E // G
        self.recv_x, self.recv_meta, self.y_pairs = recv_x, recv_meta, y_pairs
        self.offsets = torch.zeros(cfg.E + 1, dtype=torch.int32)
        self.all_off = torch.zeros((G, cfg.E + 1), dtype=torch.int32)
        self.layer = None

    def set_layer(self, l):
        c = self.c
        self.layer = l
        self.router = gen.router_weights(c.seed, l, c.E, c.H)
        self.bias = gen.zipf_bias(c.seed, l, c.E) if c.zipf else None
        self.shared_w = gen.shared_weights(c.seed, l, c.H, c.Is)

    def front(self, h, flags=0):
        c = self.c
        _, self.x = O.rmsnorm(h.numpy())
        lg = O.router_logits(self.x, self.router, self.bias)
        self.idx = O.top_k(lg, c.k)
        self.gates = O.softmax_gates(lg, self.idx)
        off, self.pairs, _ = O.buckets(self.idx, c.E)
        self.offsets.copy_(torch.from_numpy(off))

    def shared(self, flags=0):
        self.ysh = O.mlp(self.x, *self.shared_w)

    def _row(self, s, e, i):
        """Receiver row of slot i of source s's bucket e (the header's layout)."""
        return _layout_rows(self.all_off.numpy().astype(np.int64), self.El, s, e, i)

    def dispatch(self):
        c = self.c
        n = int(self.offsets[c.E])
        for i in range(n):
            p = int(self.pairs[i])
            e = int(self.idx.reshape(-1)[p])
            d = e // self.El
            r = self._row(self.rank, e, i)
            self.recv_x[d][r] = torch.from_numpy(self.x[p // c.k])
            self.recv_meta[d][r] = torch.tensor([self.rank, p], dtype=torch.int32)

    def experts(self, flags=0):
        c = self.c
        A = self.all_off.numpy().astype(np.int64)
        cnt = A[:, 1:] - A[:, :-1]
        d = self.rank
        mine = cnt[:, d * self.El:(d + 1) * self.El].sum(axis=0)
        loff = np.concatenate([[0], np.cumsum(mine)])
        rx = self.recv_x[d].numpy()
        meta = self.recv_meta[d].numpy()
        for j in range(self.El):
            a, b = int(loff[j]), int(loff[j + 1])
            if a == b:
                continue
            e = d * self.El + j
            # every row of the expert's range came from a pair routed to e
            for r in range(a, b):
                s, p = meta[r]
                assert s in range(self.G)
            y = O.mlp(rx[a:b], *gen.expert_weights(c.seed, self.layer, e, c.H, c.I))
            for r in range(a, b):
                s, p = meta[r]
                self.y_pairs[s][p] = torch.from_numpy(y[r - a])

    def combine(self, h):
        out = O.combine(self.y_pairs[self.rank].numpy(), self.gates, self.ysh)
        h += torch.from_numpy(out)


def _worker(rank, world, port, recv_x, recv_meta, y_pairs, q):
    global CFG
    CFG = _cfg(world)
    import datetime
    import torch.distributed as dist
    from quantized_moe_bit_b200 import ep
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        c = CFG
        comm = ep.EpComm()
        r = HostEpRank(world, rank, c, recv_x, recv_meta, y_pairs)
        z = gen.rows(c.seed, 1000 + rank, c.T, c.H).astype(np.float64)
        h = torch.from_numpy(z.copy())
        want = z.copy()
        for l in range(2):
            r.set_layer(l)
            ep.ep_layer_forward([r], comm, [h])
            _, x = O.rmsnorm(want)
            res = O.layer_forward(x, r.router, r.bias, lambda e, l=l: gen.expert_weights(c.seed, l, e, c.H, c.I),
                                  r.shared_w, c.k, c.E)
            want = want + res["out"]
        q.put((rank, float(np.abs(h.numpy() - want).max()), float(np.abs(want).max())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_ranks_two_layers_match_oracle(world):
    WORLD = world
    c = _cfg(world)
    cap = WORLD * c.T * c.k
    recv_x = [torch.zeros((cap, c.H), dtype=torch.float64).share_memory_() for _ in range(WORLD)]
    recv_meta = [torch.full((cap, 2), -1, dtype=torch.int32).share_memory_() for _ in range(WORLD)]
    y_pairs = [torch.zeros((c.T * c.k, c.H), dtype=torch.float64).share_memory_() for _ in range(WORLD)]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, WORLD, port, recv_x, recv_meta, y_pairs, q)) for r in range(WORLD)]
    for p in ps:
        p.start()
    got = {}
    for _ in range(WORLD):
        rank, err, scale = q.get(timeout=180)
        got[rank] = (err, scale)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, (err, scale) in got.items():
        assert err <= 1e-12 * scale, (rank, err, scale)
    # rows crossed between ranks (the exchange was exercised)
    crossed = sum(len((set(recv_meta[d][:, 0].tolist()) - {-1}) - {d}) for d in range(WORLD))
    assert crossed >= WORLD, crossed


def test_rank_shapes_rejected_before_any_allocation():
    from quantized_moe_bit_b200 import ep
    with pytest.raises(ValueError):
        ep.EpRank(3, 0, 4, 256, 128, 192, 16, 4, layer=None)      # 16 experts do not split over 3 ranks
    with pytest.raises(ValueError):
        ep.EpRank(4, 0, 4, 256, 128, 192, 16, 4, layer=None)      # 4 experts per rank: not a multiple of 8


def _layout_rows(A, El, s, e, i):
    """Receiver row of slot i of source s's bucket e, as the C-ABI header
    defines it (A: every rank's bucket offsets)."""
    cnt = A[:, 1:] - A[:, :-1]
    d0 = (e // El) * El
    return int(cnt[:, d0:e].sum()) + int(cnt[:s, e].sum()) + (i - int(A[s, e]))


@pytest.mark.parametrize("G,E", [(1, 8), (2, 16), (4, 32), (8, 64)])
def test_receiver_layout_is_an_ordered_bijection(G, E):
    """The receiver layout over random buckets: every (source, slot) lands on
    a distinct row of its expert's owner, the rows of each owner are exactly
    0 .. R-1, and they run by expert, then by source, then by slot."""
    rng = np.random.default_rng(G * 100 + E)
    El = E // G
    T, k = 7, 4
    A = np.zeros((G, E + 1), dtype=np.int64)
    for s_ in range(G):
        ids = rng.choice(E, size=(T, k), p=rng.dirichlet(np.full(E, 0.3)))
        A[s_, 1:] = np.cumsum(np.bincount(ids.reshape(-1), minlength=E))
    for d in range(G):
        keys, rows = [], []
        for s_ in range(G):
            for e in range(d * El, (d + 1) * El):
                for i in range(int(A[s_, e]), int(A[s_, e + 1])):
                    keys.append((e, s_, i))
                    rows.append(_layout_rows(A, El, s_, e, i))
        assert sorted(rows) == list(range(len(rows)))
        order = [key for _, key in sorted(zip(rows, keys))]
        assert order == sorted(keys)
