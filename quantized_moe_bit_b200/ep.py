"""Expert-parallel routed-MoE layer over G ranks (plumbing around libmoe).

Rank d owns routed experts [d E/G, (d+1) E/G); every rank keeps its own
tokens and runs its own norm, router, bucketing, shared expert and combine.
Per layer (`ep_layer_forward`):

    front      moe_rmsnorm, moe_router_topk, moe_bucket
    gather     every rank's bucket offsets into all_offsets [G, E+1]
    dispatch   moe_ep_dispatch: input rows stored into the owners' recv_x
               (and the rank's own receiver plan written)
    shared     moe_shared_forward (before the barrier: a rank's shared expert
               runs while slower ranks still dispatch)
    barrier
    experts    moe_expert_forward (k = 1, E/G experts) over the received rows,
               moe_ep_return: output rows stored into the sources' y_pairs
    barrier
    combine    moe_combine into the rank's residual stream

Every step is a libmoe kernel; Python only orders the calls and the
collectives.  The exchanges are the kernels' own stores into peer memory, so
the collectives are an all-gather of G x (E+1) integers and two barriers,
all stream-ordered: no host synchronisation inside a layer.

`EpComm` runs the collectives over torch.distributed (NCCL between GPUs; the
same code drives gloo on CPU).  `LocalRanks` holds all G ranks in one process
on one GPU (the exchanges are then stores into this GPU's own buffers): the
same kernels and layout, for testing the path where only one GPU exists.
"""
from __future__ import annotations

from typing import List, Optional, Sequence

import torch
import torch.distributed as dist

from . import binding as B


class _RawDeviceArray:
    """A whole cudaMalloc allocation seen as a torch tensor (exportable by
    CUDA IPC, unlike a slice of torch's caching allocator)."""

    def __init__(self, nbytes: int):
        self.addr = B.moe_device_alloc(nbytes)
        self.__cuda_array_interface__ = {"shape": (nbytes,), "typestr": "|u1", "data": (self.addr, False),
                                         "version": 3, "strides": None}

    def free(self):
        if self.addr:
            B.moe_device_free(self.addr)
            self.addr = 0


class EpRank:
    """One rank's state for one layer shape: its routing buffers, the
    receive buffers other ranks store into, and the peer tables."""

    def __init__(self, G: int, rank: int, T: int, H: int, I: int, Is: int, E: int, k: int, layer,
                 device="cuda", exportable: bool = False):
        if E % G or (E // G) % 8:
            raise ValueError(f"E/G must be a whole multiple of 8 (E={E}, G={G})")
        self.G, self.rank, self.T, self.H, self.I, self.Is, self.E, self.k = G, rank, T, H, I, Is, E, k
        self.El = E // G
        self.cap = G * T * k                     # worst case: every pair of every rank to this one
        self.device = device
        self._raw: List[_RawDeviceArray] = []
        self._opened: List[int] = []
        self.set_layer(layer)
        i32, f32, bf = torch.int32, torch.float32, torch.int16
        z = lambda shape, dt: torch.empty(shape, dtype=dt, device=device)  # noqa: E731
        self.x = z((T, H), bf)
        self.idx, self.gates = z((T, k), i32), z((T, k), f32)
        self.offsets, self.pairs = z(E + 1, i32), z(T * k, i32)
        self.active, self.n_active = z(E, i32), z(1, i32)
        self.all_off = z((G, E + 1), i32)
        self.loff, self.rpairs = z(self.El + 1, i32), z(max(self.cap, 1), i32)
        self.ractive, self.rn = z(self.El, i32), z(1, i32)
        self.y_rows = z((max(self.cap, 1), H), f32)
        self.ysh, self.y = z((T, H), f32), z((T, H), bf)
        # buffers the other ranks store into
        self.recv_x = self._shared_buf((max(self.cap, 1), H), bf, exportable)
        self.recv_meta = self._shared_buf((max(self.cap, 1), 2), i32, exportable)
        self.y_pairs = self._shared_buf((max(T * k, 1), H), f32, exportable)
        self.ws_e = z(B.moe_expert_workspace_size(self.cap, H, I, 1), torch.uint8)
        self.ws_s = z(B.moe_shared_workspace_size(T, H, Is), torch.uint8)
        self.peer_recv_x: Optional[list] = None
        self.peer_recv_meta: Optional[list] = None
        self.peer_y_pairs: Optional[list] = None

    def set_layer(self, layer):
        """The layer's weights (a DeviceLayer): router, bias, shared expert
        and this rank's slice of the routed blob table."""
        self.layer = layer
        self.local_blobs = layer.blob_ptrs[self.rank * self.El:(self.rank + 1) * self.El]

    def _shared_buf(self, shape, dtype, exportable: bool) -> torch.Tensor:
        if not exportable:
            return torch.empty(shape, dtype=dtype, device=self.device)
        nbytes = torch.Size(shape).numel() * torch.empty((), dtype=dtype).element_size()
        raw = _RawDeviceArray(max(nbytes, 16))
        self._raw.append(raw)
        return torch.as_tensor(raw, device=self.device)[:nbytes].view(dtype).view(shape)

    # -- peers
    def own_buffers(self):
        return self.recv_x.data_ptr(), self.recv_meta.data_ptr(), self.y_pairs.data_ptr()

    def set_peers(self, recv_x: Sequence[int], recv_meta: Sequence[int], y_pairs: Sequence[int]):
        assert len(recv_x) == len(recv_meta) == len(y_pairs) == self.G
        self.peer_recv_x, self.peer_recv_meta, self.peer_y_pairs = list(recv_x), list(recv_meta), list(y_pairs)

    def ipc_handles(self):
        return [B.moe_ipc_get_handle(p) for p in self.own_buffers()]

    def open_peers(self, handles_by_rank):
        """handles_by_rank[r] = rank r's ipc_handles(); maps every other rank's
        buffers into this process."""
        tables = ([], [], [])
        for r, hs in enumerate(handles_by_rank):
            for j, h in enumerate(hs):
                if r == self.rank:
                    tables[j].append(self.own_buffers()[j])
                else:
                    p = B.moe_ipc_open(h)
                    self._opened.append(p)
                    tables[j].append(p)
        self.set_peers(*tables)

    def close(self):
        for p in self._opened:
            B.moe_ipc_close(p)
        self._opened = []
        for raw in self._raw:
            raw.free()
        self._raw = []

    # -- the layer's steps on this rank
    def front(self, h: torch.Tensor, flags: int = 0):
        L = self.layer
        B.moe_rmsnorm(h, self.x)
        B.moe_router_topk(self.x, L.router.c, L.bias, 0, self.E, self.k, self.idx, self.gates)
        B.moe_bucket(self.idx, self.E, self.offsets, self.pairs, self.active, self.n_active)

    def shared(self, flags: int = 0):
        B.moe_shared_forward(self.x, self.Is, self.layer.shared_c, self.ysh, self.ws_s, flags=flags)

    def dispatch(self):
        B.moe_ep_dispatch(self.x, self.k, self.E, self.G, self.rank, self.idx, self.pairs, self.all_off,
                          self.peer_recv_x, self.peer_recv_meta, self.cap, self.loff, self.rpairs, self.ractive,
                          self.rn)

    def experts(self, flags: int = 0):
        B.moe_expert_forward(self.recv_x[:self.cap], self.I, self.El, 1, self.local_blobs, self.loff, self.rpairs,
                             self.ractive, self.rn, self.y_rows, self.ws_e, flags=flags)
        B.moe_ep_return(self.y_rows[:self.cap], self.E, self.G, self.rank, self.recv_meta, self.loff, self.T * self.k,
                        self.peer_y_pairs)

    def combine(self, h: torch.Tensor):
        B.moe_combine(self.y_pairs, self.gates, self.ysh, self.y, residual=h)


class EpComm:
    """Collectives between processes (one rank each) over torch.distributed."""

    def __init__(self, group=None, device=None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.nccl = dist.get_backend(group) == "nccl"
        self._one = torch.ones(1, dtype=torch.int32, device=device)

    def gather_offsets(self, ranks):
        (r,) = ranks
        if self.nccl:
            dist.all_gather_into_tensor(r.all_off.view(-1), r.offsets, group=self.group)
        else:
            dist.all_gather(list(r.all_off.unbind(0)), r.offsets, group=self.group)

    def barrier(self):
        # stream-ordered on NCCL: later kernels on the stream start after
        # every rank's earlier ones have finished (MAX keeps the word at 1)
        dist.all_reduce(self._one, op=dist.ReduceOp.MAX, group=self.group)

    def exchange_handles(self, rank: EpRank):
        out = [None] * self.world
        dist.all_gather_object(out, rank.ipc_handles(), group=self.group)
        return out


class LocalRanks:
    """All G ranks in this process on one device: the offsets gather is a
    copy per rank pair, and the barriers are the stream order itself."""

    def __init__(self, ranks: Sequence[EpRank]):
        self.ranks = list(ranks)
        bufs = [r.own_buffers() for r in self.ranks]
        for r in self.ranks:
            r.set_peers([b[0] for b in bufs], [b[1] for b in bufs], [b[2] for b in bufs])

    def gather_offsets(self, ranks):
        for r in ranks:
            for s, src in enumerate(self.ranks):
                r.all_off[s].copy_(src.offsets)

    def barrier(self):
        pass


def connect(rank: EpRank, comm: EpComm):
    """Peer tables of a process-per-rank run: this rank's own buffers, the
    others' mapped by CUDA IPC (G = 1 maps nothing)."""
    if comm.world == 1:
        p = rank.own_buffers()
        rank.set_peers([p[0]], [p[1]], [p[2]])
    else:
        rank.open_peers(comm.exchange_handles(rank))


def ep_layer_forward(ranks: Sequence[EpRank], comm, hs: Sequence[torch.Tensor], flags: int = 0):
    """One layer on the ranks this process holds (one per process, or all G
    under LocalRanks); hs[i] is rank i's residual stream fp32 [T, H], updated
    in place.  Returns nothing; each rank's y, idx and gates hold the layer's
    output and routing."""
    for r, h in zip(ranks, hs):
        r.front(h, flags)
    comm.gather_offsets(ranks)
    for r in ranks:
        r.dispatch()
    for r in ranks:
        r.shared(flags)
    comm.barrier()
    for r in ranks:
        r.experts(flags)
    comm.barrier()
    for r, h in zip(ranks, hs):
        r.combine(h)
