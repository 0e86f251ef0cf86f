"""Routed experts streamed through the per-layer LFU slot cache.

The streamed run must equal the all-resident run bit for bit, the LFU access
log must equal the reference simulator's on the same routing stream, the
layer outputs must match the oracle (teacher-forced samples), and host-side
faults must surface as errors without touching the GPU's health.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import gen
from gen import CONFIGS, tiny_config
from oracle import moe_oracle as O
from oracle.lfu_sim import LFUSim
from tests._support import HostLayer, check_output, check_routing

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    import quantized_moe_bit_b200 as M
    return M


class Streamed:
    """Weights of a streamed workload: pinned host blobs, device copies for the
    resident reference, LFU slot pool and per-layer device pointer tables."""

    def __init__(self, M, cfg):
        from quantized_moe_bit_b200.weights import blob_table, upload_qmat
        c = cfg
        self.cfg = c
        self.stride = gen.synth.default_blob_stride(c.H, c.I)
        self.host = torch.empty((c.layers, c.E, self.stride), dtype=torch.uint8, pin_memory=True)
        hv = self.host.numpy()
        self.routers, self.shared = [], []
        for l in range(c.layers):
            gen.layer_blobs(c.seed, l, c.E, c.H, c.I, self.stride, out=hv[l], threads=16)
            self.routers.append(upload_qmat(gen.router_weights(c.seed, l, c.E, c.H)))
            self.shared.append([upload_qmat(m) for m in gen.shared_weights(c.seed, l, c.H, c.Is)])
        self.dev = self.host.cuda()                                   # resident copy
        self.dev_tables = [blob_table(self.dev[l]) for l in range(c.layers)]
        self.pool = torch.empty((c.layers, c.n_slots, self.stride), dtype=torch.uint8, device="cuda")
        self.slot_tables = torch.zeros((c.layers, c.E), dtype=torch.int64, device="cuda")
        base = self.host.data_ptr()
        self.host_ptrs = [base + (l * c.E + e) * self.stride for l in range(c.layers) for e in range(c.E)]
        n_tok = c.prompt_tokens + c.decode_steps
        self.sets = [gen.forced_routing(c.seed, l, n_tok, c.E, c.k) for l in range(c.layers)]

    def inputs(self):
        c = self.cfg
        prompt = gen.rows(c.seed, 3000, c.prompt_tokens, c.H)
        dec = [gen.rows(c.seed, 4000 + d, 1, c.H) for d in range(c.decode_steps)]
        units = [(prompt[i:i + c.T], i) for i in range(0, c.prompt_tokens, c.T)]
        units += [(dec[d], c.prompt_tokens + d) for d in range(c.decode_steps)]
        return units

    def bias(self, l, t0, T):
        return torch.from_numpy(gen.forced_bias(self.sets[l][t0:t0 + T], self.cfg.E)).cuda()


def run_resident(M, S, units):
    c = S.cfg
    outs = []
    for z, t0 in units:
        T = z.shape[0]
        h = torch.from_numpy(z).cuda()
        ws = torch.empty(M.moe_layer_workspace_size(T, c.H, c.I, c.Is, c.E, c.k), dtype=torch.uint8, device="cuda")
        ys, idxs, xs = [], [], []
        for l in range(c.layers):
            y = torch.empty((T, c.H), dtype=torch.int16, device="cuda")
            x = torch.empty((T, c.H), dtype=torch.int16, device="cuda")
            idx = torch.empty((T, c.k), dtype=torch.int32, device="cuda")
            M.moe_layer_forward(T, c.H, c.I, c.Is, c.E, c.k, S.routers[l].c, S.bias(l, t0, T), 1, S.dev_tables[l],
                                [m.c for m in S.shared[l]], ws, h_in=h, h_out=h, x_out=x, y=y, idx=idx)
            ys.append(y); idxs.append(idx); xs.append(x)
        M.moe_sync()
        outs.append(dict(h=h.cpu().numpy(), y=[t.cpu().numpy() for t in ys], idx=[t.cpu().numpy() for t in idxs],
                         x=[t.cpu().numpy() for t in xs]))
    return outs


def run_streamed(M, S, units, lfu, side, on_error=None):
    """Streamed run; on_error(unit, layer, exc) may clear an injected fault
    and return True to repeat the failed layer call."""
    c = S.cfg
    outs = []
    main = torch.cuda.current_stream()
    for u, (z, t0) in enumerate(units):
        T = z.shape[0]
        h = torch.from_numpy(z).cuda()
        ws = torch.empty(M.moe_streamed_workspace_size(T, c.H, c.I, c.Is, c.E, c.k), dtype=torch.uint8, device="cuda")
        ys, idxs, xs = [], [], []
        for l in range(c.layers):
            y = torch.empty((T, c.H), dtype=torch.int16, device="cuda")
            x = torch.empty((T, c.H), dtype=torch.int16, device="cuda")
            idx = torch.empty((T, c.k), dtype=torch.int32, device="cuda")
            while True:
                try:
                    M.moe_streamed_layer_forward(lfu, l, h, c.I, c.Is, c.E, c.k, S.routers[l].c, S.bias(l, t0, T),
                                                 1, [m.c for m in S.shared[l]], S.slot_tables[l], ws, x_out=x,
                                                 y_out=y, idx_out=idx, main_stream=main, side_stream=side)
                    break
                except M.MoeError as exc:
                    if on_error is None or not on_error(u, l, exc):
                        raise
            ys.append(y); idxs.append(idx); xs.append(x)
        M.moe_sync()
        outs.append(dict(h=h.cpu().numpy(), y=[t.cpu().numpy() for t in ys], idx=[t.cpu().numpy() for t in idxs],
                         x=[t.cpu().numpy() for t in xs]))
    return outs


def simulate(S, outs, prefetch: int = 0):
    c = S.cfg
    sim = LFUSim(c.layers, c.n_slots)
    for o in outs:
        for l in range(c.layers):
            idx = o["idx"][l]
            if idx.shape[0] == 1:
                sim.step(l, [int(e) for e in idx[0]])
            else:
                for ids in sim.chunk_steps(l, np.unique(idx).tolist(), c.k):
                    sim.step(l, ids)
            sim.prefetch(l, prefetch)            # after every layer call (nothing at 0)
    return sim


def check_against_oracle(S, outs, units, samples):
    c = S.cfg
    for (u, l) in samples:
        z, t0 = units[u]
        T = z.shape[0]
        hl = HostLayer(c, l, with_blobs=False)
        x = O.bf16_to_f64(outs[u]["x"][l].view(np.uint16))
        b = gen.forced_bias(S.sets[l][t0:t0 + T], c.E).astype(np.float64)
        lg = O.router_logits(x, hl.router, b)
        check_routing(outs[u]["idx"][l], lg, c.k)
        assert all(set(outs[u]["idx"][l][t]) == set(S.sets[l][t0 + t]) for t in range(T))   # forced sets
        r = O.layer_forward(x, hl.router, b, hl.expert, hl.shared, c.k, c.E, idx=outs[u]["idx"][l])
        check_output(outs[u]["y"][l].view(np.uint16), r["out"], f"unit {u} layer {l}")


def _run_all(M, cfg, samples, prefetch: int = 0):
    S = Streamed(M, cfg)
    units = S.inputs()
    ref = run_resident(M, S, units)
    lfu = M.MoeLfu(cfg.layers, cfg.E, cfg.n_slots, gen.blob_bytes(cfg.H, cfg.I), S.host_ptrs, S.pool,
                   S.stride)
    lfu.set_prefetch(prefetch)
    side = torch.cuda.Stream()
    got = run_streamed(M, S, units, lfu, side)
    for a, b in zip(ref, got):
        assert np.array_equal(a["h"], b["h"])
        for l in range(cfg.layers):
            assert np.array_equal(a["y"][l], b["y"][l]) and np.array_equal(a["idx"][l], b["idx"][l])
    sim = simulate(S, got, prefetch)
    assert lfu.log() == sim.log
    hits, misses, nbytes = lfu.stats()
    staged = sum(1 for r in sim.log if r[3] == 2)
    assert (misses + staged) * gen.blob_bytes(cfg.H, cfg.I) == nbytes and hits > 0
    assert (staged > 0) == (prefetch > 0)
    check_against_oracle(S, got, units, samples)
    lfu.close()
    return hits, misses


@pytest.mark.parametrize("prefetch", [0, 2])
def test_streamed_tiny(M, prefetch):
    cfg = replace(tiny_config("streamed_30L_lfu"), layers=4, T=24, prompt_tokens=48, decode_steps=6, n_slots=6)
    _run_all(M, cfg, samples=[(0, 0), (1, 3), (2, 1), (7, 2)], prefetch=prefetch)


@pytest.mark.parametrize("prefetch", [0, 2])
def test_streamed_full(M, prefetch):
    """1024-token prompt in chunks of 128 through 30 layers, then 128 decode
    steps, routed experts in pinned host memory, 16 slots per layer (with and
    without the lookahead prefetch of 2 experts per layer call)."""
    cfg = CONFIGS["streamed_30L_lfu"]
    hits, misses = _run_all(M, cfg, samples=[(0, 0), (3, 17), (7, 29), (8, 5), (100, 12), (135, 29)],
                            prefetch=prefetch)
    print(f"streamed_30L_lfu prefetch {prefetch}: hits {hits} misses {misses}")


def test_streamed_layer_major_tiny(M):
    """The whole prompt through each layer in one call (layer-major): equal
    to the all-resident run of the same units bit for bit, the log equal to
    the simulator's, and fewer misses than the same prompt in chunks."""
    chunked = replace(tiny_config("streamed_30L_lfu"), layers=4, T=12, prompt_tokens=48, decode_steps=6, n_slots=6)
    _, miss_chunked = _run_all(M, chunked, samples=[(0, 0)])
    cfg = replace(chunked, T=48)
    hits, misses = _run_all(M, cfg, samples=[(0, 0), (0, 3), (1, 2), (6, 1)])
    assert misses < miss_chunked


def test_streamed_layer_major_full(M):
    """The full streamed workload with its 1024-token prompt through each of
    the 30 layers in one call, then the 128 decode steps."""
    cfg = replace(CONFIGS["streamed_30L_lfu"], T=1024)
    hits, misses = _run_all(M, cfg, samples=[(1, 0), (60, 17), (128, 29)])
    print(f"streamed_30L_lfu layer-major prompt: hits {hits} misses {misses}")


def test_lfu_host_faults(M):
    cfg = replace(tiny_config("streamed_30L_lfu"), layers=2, T=8, prompt_tokens=8, decode_steps=0, n_slots=4)
    S = Streamed(M, cfg)
    (z, t0), = S.inputs()
    lfu = M.MoeLfu(cfg.layers, cfg.E, cfg.n_slots, gen.blob_bytes(cfg.H, cfg.I), S.host_ptrs, S.pool, S.stride)
    lfu.set_fault(1, 2)                         # the third copy fails
    h = torch.from_numpy(z).cuda()
    ws = torch.empty(M.moe_streamed_workspace_size(8, cfg.H, cfg.I, cfg.Is, cfg.E, cfg.k), dtype=torch.uint8,
                     device="cuda")
    with pytest.raises(M.MoeError) as ei:
        for l in range(cfg.layers):
            M.moe_streamed_layer_forward(lfu, l, h, cfg.I, cfg.Is, cfg.E, cfg.k, S.routers[l].c, S.bias(l, t0, 8), 1,
                                         [m.c for m in S.shared[l]], S.slot_tables[l], ws,
                                         side_stream=torch.cuda.Stream())
    assert ei.value.status == 2 and "injected" in str(ei.value)
    torch.cuda.synchronize()
    lfu.close()
    # a bounded host wait that runs out: a stream held by a host function
    import time
    s = torch.cuda.Stream()
    ev = torch.cuda.Event()
    with torch.cuda.stream(s):
        torch.cuda._sleep(200 * 1000 * 1000)    # ~0.1-0.2 s of device-side spinning on this stream
        ev.record(s)
    with pytest.raises(M.MoeError) as ei:
        M.moe_lfu_wait(ev, 5)
    assert ei.value.status == 3
    s.synchronize()
    M.moe_lfu_wait(ev, 1000)
    M.moe_sync()


def test_lfu_copy_failure_mid_chunk_then_retry(M):
    """A copy that fails in the middle of a prefill chunk's layer call rolls
    the layer's cache state back; repeating the call and carrying on gives
    output bitwise equal to the all-resident run and an access log equal to
    the simulator's (the failed attempt leaves no record)."""
    cfg = replace(tiny_config("streamed_30L_lfu"), layers=3, T=24, prompt_tokens=72, decode_steps=4, n_slots=6)
    S = Streamed(M, cfg)
    units = S.inputs()
    ref = run_resident(M, S, units)
    # misses per (unit, layer) of the policy on this routing, from the simulator
    sim = LFUSim(cfg.layers, cfg.n_slots)
    misses = {}
    for u, o in enumerate(ref):
        for l in range(cfg.layers):
            n0 = len(sim.log)
            idx = o["idx"][l]
            steps = [[int(e) for e in idx[0]]] if idx.shape[0] == 1 else \
                sim.chunk_steps(l, np.unique(idx).tolist(), cfg.k)
            for ids in steps:
                sim.step(l, ids)
            misses[(u, l)] = sum(1 for r in sim.log[n0:] if r[3] == 0)
    # fail the 3rd miss of unit 1 (a prefill chunk), layer 1
    before = sum(misses[(u, l)] for u in range(1) for l in range(cfg.layers)) + misses[(1, 0)]
    assert misses[(1, 1)] >= 4
    lfu = M.MoeLfu(cfg.layers, cfg.E, cfg.n_slots, gen.blob_bytes(cfg.H, cfg.I), S.host_ptrs, S.pool, S.stride)
    lfu.set_fault(1, before + 2)
    failures = []

    def on_error(u, l, exc):
        assert exc.status == 2 and "injected" in str(exc)
        failures.append((u, l))
        lfu.set_fault(0, 0)
        return True
    got = run_streamed(M, S, units, lfu, torch.cuda.Stream(), on_error=on_error)
    assert failures == [(1, 1)]
    for a, b in zip(ref, got):
        assert np.array_equal(a["h"], b["h"])
        for l in range(cfg.layers):
            assert np.array_equal(a["y"][l], b["y"][l]) and np.array_equal(a["idx"][l], b["idx"][l])
    assert lfu.log() == simulate(S, got).log
    hits, n_miss, nbytes = lfu.stats()
    assert n_miss * gen.blob_bytes(cfg.H, cfg.I) <= nbytes      # the failed attempt's copies are extra
    lfu.close()
