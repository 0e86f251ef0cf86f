#!/usr/bin/env python
"""Benchmark of the routed-MoE layer stack: 30-layer batch-1 decode.

Workload (decode_30L_b1): 30 independent layers of H=2816, E=128 routed
experts (top 8), expert I=704, shared expert Is=2112; MLX-style affine 4-bit
group-64 experts (12.85 GB of routed weights resident in HBM), 8-bit router,
Zipf(1.1) per-layer routing skew.  One step = one fresh token through all 30
layers (RMS norm, router + top-8, routed experts, shared expert, combine,
residual add).  Synthetic seeded weights and inputs.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs one process per GPU (torchrun), each an independent replica on its
own token stream (no collective on the data path); `value` sums all ranks.
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import gen  # noqa: E402

CFG = gen.CONFIGS["decode_30L_b1"]
METRIC = "MoE tokens/s (30-layer decode b=1; 128-tok prefill) and % of HBM/TC roofline"
FALLBACK_HBM = 6650.0


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM, "fallback"


# DRAM read + write of the decode kernel measured by ncu on 3 full-size
# layers of this workload, per layer; valid only for the kernel source the
# capture was taken on (sha256 prefix of decode_fused.cu).
DECODE_TRAFFIC = {"source_sha256_prefix": "0b3e112df90c7b80", "bytes_per_layer": 38.7517e6}


def decode_traffic(layers: int):
    src = os.path.join(ROOT, "quantized_moe_bit_b200", "csrc", "decode_fused.cu")
    try:
        with open(src, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()[:16]
    except OSError:
        return None
    if sha != DECODE_TRAFFIC["source_sha256_prefix"]:
        return None
    return DECODE_TRAFFIC["bytes_per_layer"] * layers


def step_bytes(cfg, distinct_per_layer: float) -> float:
    """Algorithmic weight bytes of one step: per layer the router, the shared
    expert and every distinct routed expert touched, read once."""
    router = cfg.E * cfg.H + 2 * 2 * cfg.E * (cfg.H // 64)
    blob = gen.blob_bytes(cfg.H, cfg.I)
    shared = sum(gen.qmat_bytes(o, i) for o, i in ((cfg.Is, cfg.H), (cfg.Is, cfg.H), (cfg.H, cfg.Is)))
    return cfg.layers * (router + shared) + distinct_per_layer * cfg.layers * blob


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None
        time.sleep(0.3)

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except Exception:
            self.p.kill()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm = [float(r[1]) for r in rows if len(r) >= 9 and r[1].strip().replace(".", "").isdigit()]
        if not sm:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.strip() == "Active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]), "samples": len(sm),
                "reasons": sorted(reasons)}


def load_stack(cfg, device, rank):
    import torch
    from quantized_moe_bit_b200.weights import upload_layer
    layers = []
    t0 = time.time()
    stride = gen.synth.default_blob_stride(cfg.H, cfg.I)
    host = np.empty((cfg.E, stride), dtype=np.uint8)
    for l in range(cfg.layers):
        router = gen.router_weights(cfg.seed, l, cfg.E, cfg.H)
        bias = gen.zipf_bias(cfg.seed, l, cfg.E) if cfg.zipf else None
        shared = gen.shared_weights(cfg.seed, l, cfg.H, cfg.Is)
        gen.layer_blobs(cfg.seed, l, cfg.E, cfg.H, cfg.I, stride, out=host, threads=16)
        layers.append(upload_layer(router, bias, shared, host, device))
    torch.cuda.synchronize()
    log(f"[rank {rank}] weights: {cfg.layers} layers in {time.time() - t0:.1f}s")
    return layers


def peaks_tc():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def layer_flops(cfg, T: int) -> float:
    """Dense FLOPs of one layer on T rows: routed experts (T*k pairs, gate, up
    and down), shared expert, router."""
    routed = 2.0 * T * cfg.k * 3 * cfg.I * cfg.H
    shared = 2.0 * T * 3 * cfg.Is * cfg.H
    router = 2.0 * T * cfg.E * cfg.H
    return routed + shared + router


def layer_bytes(cfg, distinct: float) -> float:
    """Weight bytes of one layer touched once: router, shared expert, the distinct routed experts."""
    router = cfg.E * cfg.H + 2 * 2 * cfg.E * (cfg.H // 64)
    shared = sum(gen.qmat_bytes(o, i) for o, i in ((cfg.Is, cfg.H), (cfg.Is, cfg.H), (cfg.H, cfg.Is)))
    return router + shared + distinct * gen.blob_bytes(cfg.H, cfg.I)


def run_prefill(M, layers, device, reps: int, T: int = 128):
    """T-row prefill chunks through one layer (the prefill workload's shapes,
    input stream and routing skew); chunk i runs on layer i mod 30 so that
    weights come from HBM.  One graph replay = one chunk per layer."""
    import torch
    from dataclasses import replace
    cfg = replace(gen.CONFIGS["prefill_1L_128tok"], T=T)
    H = cfg.H
    z = torch.from_numpy(gen.rows(cfg.seed, cfg.row_stream, T, H)).to(device)
    ws = torch.empty(M.moe_layer_workspace_size(T, H, cfg.I, cfg.Is, cfg.E, cfg.k), dtype=torch.uint8, device=device)
    ho = torch.empty_like(z)
    idx = torch.empty((len(layers), T, cfg.k), dtype=torch.int32, device=device)

    def chunk(l):
        dl = layers[l]
        M.moe_layer_forward(T, H, cfg.I, cfg.Is, cfg.E, cfg.k, dl.router.c, dl.bias, 0, dl.blob_ptrs, dl.shared_c,
                            ws, h_in=z, h_out=ho, idx=idx[l])
    for l in range(len(layers)):
        chunk(l)
    torch.cuda.synchronize()
    M.moe_sync()
    g = torch.cuda.CUDAGraph()
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        with torch.cuda.graph(g, stream=st):
            for l in range(len(layers)):
                chunk(l)
    torch.cuda.current_stream().wait_stream(st)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    M.moe_sync()
    n_chunks = reps * len(layers)
    t = e0.elapsed_time(e1) / 1e3 / n_chunks
    ids = idx.cpu().numpy()
    distinct = float(np.mean([len(np.unique(ids[l])) for l in range(len(layers))]))
    flops, byts = layer_flops(cfg, T), layer_bytes(cfg, distinct)
    gemm_flops = 2.0 * T * (cfg.k * 3 * cfg.I * cfg.H + 3 * cfg.Is * cfg.H)
    tc, tc_src = peaks_tc()
    hbm, hbm_src = peaks()
    del g
    t_hbm, t_tc = byts / (hbm * 1e9), gemm_flops / (tc * 1e12)
    return {"workload": f"prefill_1L_{T}tok", "value": T / t, "unit": "tokens/s", "us_per_chunk": t * 1e6,
            "rows_per_chunk": T, "chunks": n_chunks, "distinct_experts_per_chunk": distinct,
            "tensor": {"achieved_tflops": flops / t / 1e12, "peak": tc, "frac": flops / t / 1e12 / tc,
                       "peak_source": tc_src, "flops_per_chunk": flops},
            "hbm": {"achieved_gbs": byts / t / 1e9, "peak": hbm, "frac": byts / t / 1e9 / hbm,
                    "peak_source": hbm_src, "bytes_per_chunk": byts},
            "binding_roofline": {"bound": "hbm" if t_hbm >= t_tc else "tensor",
                                 "frac": max(t_hbm, t_tc) / t, "ideal_us": max(t_hbm, t_tc) * 1e6},
            "l2": "each chunk on another of 30 layers (weights of 30 layers per graph replay)"}


def run_decode_b64(M, stack, device, reps: int):
    """64 independent rows per step through the 30 layers (batched-decode
    workload): one graph replay = one step."""
    import torch
    cfg = gen.CONFIGS["decode_30L_b64"]
    T, H = cfg.T, cfg.H
    z = torch.from_numpy(gen.rows(cfg.seed, cfg.row_stream, T, H)).to(device)
    h = torch.empty_like(z)
    ws = torch.empty(M.moe_decode_workspace_size(T, H, cfg.I, cfg.Is, cfg.E, cfg.k), dtype=torch.uint8, device=device)
    idx = torch.empty((cfg.layers, T, cfg.k), dtype=torch.int32, device=device)

    def step():
        h.copy_(z)
        M.moe_decode_forward(h, cfg.I, cfg.Is, cfg.E, cfg.k, stack, ws, idx_trace=idx)
    step()
    torch.cuda.synchronize()
    M.moe_sync()
    g = torch.cuda.CUDAGraph()
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        with torch.cuda.graph(g, stream=st):
            step()
    torch.cuda.current_stream().wait_stream(st)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    M.moe_sync()
    t = e0.elapsed_time(e1) / 1e3 / reps
    ids = idx.cpu().numpy()
    distinct = float(np.mean([len(np.unique(ids[l])) for l in range(cfg.layers)]))
    byts = cfg.layers * layer_bytes(cfg, distinct)
    hbm, hbm_src = peaks()
    del g
    return {"workload": "decode_30L_b64", "value": T / t, "unit": "tokens/s", "ms_per_step": t * 1e3, "steps": reps,
            "distinct_experts_per_layer": distinct,
            "hbm": {"achieved_gbs": byts / t / 1e9, "peak": hbm, "frac": byts / t / 1e9 / hbm, "peak_source": hbm_src,
                    "bytes_per_step": byts},
            "l2": "inputs larger than L2 (every step touches all 30 layers)"}


def run_streamed_lfu(M, device):
    """Streamed workload: 1024-token prompt in chunks of 128 through 30 layers,
    then 128 decode steps, routed experts in pinned host memory, 16 HBM slots
    per layer (misses copied host -> device on a side stream while the shared
    expert runs).  Prefill and decode timed separately (CUDA events; the LFU
    plan of every layer step needs the routing on the host).  A/B of the
    lookahead prefetch: off and on (2 experts per layer call), each on a fresh
    cache, alternately twice; the top-level figures are the first run with
    the prefetch off."""
    import torch
    from quantized_moe_bit_b200.weights import blob_table, upload_qmat
    c = gen.CONFIGS["streamed_30L_lfu"]
    stride = gen.synth.default_blob_stride(c.H, c.I)
    host = torch.empty((c.layers, c.E, stride), dtype=torch.uint8, pin_memory=True)
    hv = host.numpy()
    routers, shared = [], []
    for l in range(c.layers):
        gen.layer_blobs(c.seed, l, c.E, c.H, c.I, stride, out=hv[l], threads=16)
        routers.append(upload_qmat(gen.router_weights(c.seed, l, c.E, c.H), device))
        shared.append([upload_qmat(m, device) for m in gen.shared_weights(c.seed, l, c.H, c.Is)])
    pool = torch.empty((c.layers, c.n_slots, stride), dtype=torch.uint8, device=device)
    tables = torch.zeros((c.layers, c.E), dtype=torch.int64, device=device)
    base = host.data_ptr()
    host_ptrs = [base + (l * c.E + e) * stride for l in range(c.layers) for e in range(c.E)]
    n_tok = c.prompt_tokens + c.decode_steps
    sets = [gen.forced_routing(c.seed, l, n_tok, c.E, c.k) for l in range(c.layers)]
    biases = {}

    def bias(l, t0, T):
        key = (l, t0, T)
        if key not in biases:
            biases[key] = torch.from_numpy(gen.forced_bias(sets[l][t0:t0 + T], c.E)).to(device)
        return biases[key]
    prompt = gen.rows(c.seed, 3000, c.prompt_tokens, c.H)
    dec = [gen.rows(c.seed, 4000 + d, 1, c.H) for d in range(c.decode_steps)]
    units = [(torch.from_numpy(prompt[i:i + c.T]).to(device), i) for i in range(0, c.prompt_tokens, c.T)]
    dec_units = [(torch.from_numpy(dec[d]).to(device), c.prompt_tokens + d) for d in range(c.decode_steps)]
    units += dec_units
    # layer-major prompt: the whole prompt as one call per layer (each layer's
    # distinct experts staged about once), the same decode steps after it
    units_lm = [(torch.from_numpy(prompt).to(device), 0)] + dec_units
    for l in range(c.layers):                   # biases built before the timed region
        for z, t0 in units + units_lm[:1]:
            bias(l, t0, z.shape[0])
    side = torch.cuda.Stream(device=device)
    main = torch.cuda.current_stream()
    ws = {T: torch.empty(M.moe_streamed_workspace_size(T, c.H, c.I, c.Is, c.E, c.k), dtype=torch.uint8,
                         device=device) for T in (c.T, 1, c.prompt_tokens)}

    def arm(prefetch: int, layer_major: bool = False):
        """One run of the workload on a fresh cache (lookahead prefetch of
        `prefetch` experts per layer call, 0: off; the prompt in chunks of
        128 rows, each through all layers, or layer-major: the whole prompt
        through each layer in one call)."""
        us_all = units_lm if layer_major else units
        n_pre = 1 if layer_major else c.prompt_tokens // c.T
        lfu = M.MoeLfu(c.layers, c.E, c.n_slots, gen.blob_bytes(c.H, c.I), host_ptrs, pool, stride)
        lfu.set_prefetch(prefetch)

        def run(us):
            for z, t0 in us:
                T = z.shape[0]
                h = z.clone()
                for l in range(c.layers):
                    M.moe_streamed_layer_forward(lfu, l, h, c.I, c.Is, c.E, c.k, routers[l].c, bias(l, t0, T), 1,
                                                 [m.c for m in shared[l]], tables[l], ws[T], main_stream=main,
                                                 side_stream=side)
        torch.cuda.synchronize()
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record()
        run(us_all[:n_pre])
        e1.record()
        run(us_all[n_pre:])
        e2.record()
        torch.cuda.synchronize()
        M.moe_sync()
        t_pre, t_dec = e0.elapsed_time(e1) / 1e3, e1.elapsed_time(e2) / 1e3
        hits, misses, nbytes = lfu.stats()
        staged = sum(1 for r in lfu.log() if r[3] == 2)
        lfu.close()
        return {"prefetch_per_call": prefetch, "prompt": "layer-major" if layer_major else f"chunks of {c.T}",
                "prefill_tokens_per_s": c.prompt_tokens / t_pre,
                "decode_tokens_per_s": c.decode_steps / t_dec, "prefill_s": t_pre, "decode_s": t_dec,
                "hits": hits, "misses": misses, "prefetched": staged, "h2d_bytes": nbytes,
                "h2d_gbs_while_streaming": nbytes / (t_pre + t_dec) / 1e9}
    runs = [arm(p) for p in (0, 2, 0, 2)]           # the two arms alternately, twice
    lm = [arm(0, True), arm(0, True)]
    base = runs[0]
    # pinned host -> device copy bandwidth of this machine, for context
    buf = host.view(-1)[: 256 << 20]
    dst = torch.empty(buf.numel(), dtype=torch.uint8, device=device)
    dst.copy_(buf, non_blocking=True)
    torch.cuda.synchronize()
    e3, e4 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e3.record()
    dst.copy_(buf, non_blocking=True)
    e4.record()
    torch.cuda.synchronize()
    h2d = buf.numel() / (e3.elapsed_time(e4) / 1e3) / 1e9
    return {"workload": "streamed_30L_lfu", **{k: base[k] for k in base if k != "prefetch_per_call"},
            "pinned_h2d_copy_gbs": h2d, "slots_per_layer": c.n_slots,
            "prefetch_ab": {"arms": "lookahead prefetch off (0) and on (2 experts per layer call), run alternately",
                            "runs": runs},
            "layer_major": {"prompt": f"all {c.prompt_tokens} prompt rows through each layer in one call "
                                      "(layer-major), then the same decode steps; prefetch off",
                            "runs": lm},
            "note": "bitwise equality with the all-resident run and the LFU log are checked by the GPU tests"}


class OracleLayers:
    """Host weights of the first layers of a workload for the oracle, built
    before any timer starts; a routed expert's weights are generated the
    first time it is asked for and kept (a warm-up pass asks for them)."""

    def __init__(self, cfg, n_layers: int):
        self.cfg, self.cache = cfg, {}
        self.layers = []
        for l in range(n_layers):
            self.layers.append((gen.router_weights(cfg.seed, l, cfg.E, cfg.H),
                                gen.zipf_bias(cfg.seed, l, cfg.E) if cfg.zipf else None,
                                self._expert_fn(l), gen.shared_weights(cfg.seed, l, cfg.H, cfg.Is)))

    def _expert_fn(self, l):
        def f(e):
            if (l, e) not in self.cache:
                self.cache[(l, e)] = gen.expert_weights(self.cfg.seed, l, e, self.cfg.H, self.cfg.I)
            return self.cache[(l, e)]
        return f

    def generate_all(self):
        for l, (_, _, f, _) in enumerate(self.layers):
            for e in range(self.cfg.E):
                f(e)


def oracle_cores():
    try:
        from threadpoolctl import threadpool_info
        return max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count()


def time_oracle(fn, one_core: bool):
    """Wall time of fn() on the host: all cores (numpy's BLAS threads) or one."""
    if one_core:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(1):
            t0 = time.perf_counter()
            fn()
            return time.perf_counter() - t0
    t0 = time.perf_counter()
    fn()
    return time.perf_counter() - t0


def cpu_baseline_oracle(n_layers: int = 3):
    """The fp64 oracle on the host cores, weights generated before the timer:
    one token of the 30-layer batch-1 workload through its first n_layers
    layers (scaled to tokens/s of the 30-layer step), the single-layer token
    and the 128-row prefill chunk; each on all cores and on one core."""
    from oracle import moe_oracle as O
    cfg = CFG
    ol = OracleLayers(cfg, n_layers)
    z = gen.rows(cfg.seed, 999, 1, cfg.H).astype(np.float64)
    run = lambda: O.stack_forward(z, ol.layers, cfg.k, cfg.E)
    run()                                   # warm-up: generates the routed experts this token touches
    t_all = time_oracle(run, False)
    t_one = time_oracle(run, True)
    c0 = gen.CONFIGS["single_layer_1tok"]
    o0 = OracleLayers(c0, 1)
    z0 = gen.rows(c0.seed, 1000, 1, c0.H).astype(np.float64)
    r0 = lambda: O.stack_forward(z0, o0.layers, c0.k, c0.E)
    r0()
    c2 = gen.CONFIGS["prefill_1L_128tok"]
    o2 = OracleLayers(c2, 1)
    z2 = gen.rows(c2.seed, c2.row_stream, c2.T, c2.H).astype(np.float64)
    r2 = lambda: O.stack_forward(z2, o2.layers, c2.k, c2.E)
    r2()
    t0a, t0o = time_oracle(r0, False), time_oracle(r0, True)
    t2a, t2o = time_oracle(r2, False), time_oracle(r2, True)
    scale = cfg.layers / n_layers
    return {"value": 1.0 / (t_all * scale), "unit": "tokens/s", "cores": oracle_cores(), "kind": "oracle",
            "one_core": {"value": 1.0 / (t_one * scale), "cores": 1},
            "sample": (f"one token of decode_30L_b1 through its first {n_layers} of 30 layers ({t_all:.2f} s on "
                       f"all cores, {t_one:.2f} s on one), scaled by 30/{n_layers}; weights generated before the "
                       f"timer (a warm-up pass generates the experts the token routes to)"),
            "single_layer_1tok": {"s_all_cores": t0a, "s_one_core": t0o, "tokens_per_s": 1.0 / t0a},
            "prefill_1L_128tok": {"s_all_cores": t2a, "s_one_core": t2o, "tokens_per_s": c2.T / t2a}}


def replica_streams(rank: int, n: int) -> list:
    """Generator stream ids of the n input tokens of replica `rank`: disjoint
    across ranks (each replica decodes its own token stream)."""
    base = 1000 + rank * 100000
    return [base + s for s in range(n)]


def max_over_ranks(values, world: int, device):
    """Element-wise max over ranks of a list of floats (timings): every rank
    takes part, every rank gets the result."""
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def whole_job_rate(ms: float, steps: int, world: int) -> float:
    """Tokens per second of the whole job: every replica decodes `steps`
    tokens; the job takes the slowest rank's time."""
    return steps * world / (ms / 1e3)


def run_reference(args, rank, world):
    """The oracle as it stands, on the host cores (rank 0 only): each step is
    one fresh token of the 30-layer batch-1 workload through its first
    layers (3, or fewer for long runs); every routed expert of those layers
    is generated before the first timed step.  value = tokens/s of the whole
    30-layer step (the sample's layers / 30 tokens per step time)."""
    if rank != 0:
        return
    from oracle import moe_oracle as O
    cfg = CFG
    # layers per step: 3, fewer when many steps are asked for, so that the
    # whole run stays near two minutes (about 0.6 s of oracle per layer)
    n_layers = max(1, min(3, int(120.0 / (0.6 * max(1, args.steps + args.warmup)))))
    ol = OracleLayers(cfg, n_layers)
    ol.generate_all()
    times = []
    for i in range(args.warmup + args.steps):
        z = gen.rows(cfg.seed, 1000 + i, 1, cfg.H).astype(np.float64)
        dt = time_oracle(lambda: O.stack_forward(z, ol.layers, cfg.k, cfg.E), False)
        if i >= args.warmup:
            times.append(dt)
    ms = 1e3 * sum(times) / args.steps
    value = (n_layers / cfg.layers) / (ms / 1e3)
    sample = (f"each step: one token through the first {n_layers} of the 30 layers (fp64 numpy oracle, all its "
              f"experts generated before the first step), i.e. {n_layers}/30 of a token")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "decode_30L_b1", "layers": 30, "batch": 1, "H": cfg.H, "E": cfg.E, "k": cfg.k,
                       "I": cfg.I, "Is": cfg.Is},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle_cores(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import quantized_moe_bit_b200 as M

    cfg = CFG
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    layers = load_stack(cfg, device, rank)
    stack = M.DecodeStack(layers)
    H = cfg.H
    n_in = args.warmup + args.steps
    z = np.concatenate([gen.rows(cfg.seed, s, 1, H) for s in replica_streams(rank, n_in)])  # [n_in, H]
    z_dev = torch.from_numpy(z).to(device).view(n_in, 1, H)
    ws = torch.empty(M.moe_decode_workspace_size(1, H, cfg.I, cfg.Is, cfg.E, cfg.k), dtype=torch.uint8,
                     device=device)
    h = torch.empty((1, H), dtype=torch.float32, device=device)
    idx_tr = torch.empty((cfg.layers, 1, cfg.k), dtype=torch.int32, device=device)

    def step():
        M.moe_decode_forward(h, cfg.I, cfg.Is, cfg.E, cfg.k, stack, ws, idx_trace=idx_tr)

    # eager warm-up (sets kernel attributes), then capture one step in a graph
    h.copy_(z_dev[0])
    step()
    torch.cuda.synchronize()
    M.moe_sync()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            step()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()

    distinct = []
    for i in range(args.warmup):
        h.copy_(z_dev[i])
        g.replay()
    torch.cuda.synchronize()
    M.moe_sync()

    def barrier():
        if world > 1:
            dist.barrier()

    sampler = ClockSampler(local_rank)
    sampler.start()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        h.copy_(z_dev[args.warmup + i])
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1)
    idx_last = idx_tr.cpu().numpy()
    distinct = float(np.mean([len(set(idx_last[l, 0].tolist())) for l in range(cfg.layers)]))

    # end to end through the public C-ABI, one token at a time from host
    # memory to host memory: moe_decode_session_step copies the row in, runs
    # the 30 layers, copies the row out and waits for it (one C call per
    # token; events on the session's stream bracket the whole loop)
    zh = torch.from_numpy(z[args.warmup:]).pin_memory().view(args.steps, 1, H)
    out_h = torch.empty((args.steps, 1, H), dtype=torch.float32).pin_memory()
    h_sess = torch.empty((1, H), dtype=torch.float32, device=device)
    sess = M.DecodeSession(h_sess, cfg.I, cfg.Is, cfg.E, cfg.k, stack, ws)
    sstream = torch.cuda.ExternalStream(sess.stream, device=device)
    for i in range(3):
        sess.step(zh[i].data_ptr(), out_h[i].data_ptr())
    torch.cuda.synchronize()
    barrier()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(sstream)
    for i in range(args.steps):
        sess.step(zh[i].data_ptr(), out_h[i].data_ptr())
    e3.record(sstream)
    torch.cuda.synchronize()
    barrier()
    ms_e2e = e2.elapsed_time(e3)
    sess.close()
    # the same through the eager moe_decode_forward call with torch copies of
    # the row and a host wait per token (argument checks and launch inside)
    cur = torch.cuda.current_stream()
    torch.cuda.synchronize()
    barrier()
    e6, e7 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e6.record()
    for i in range(args.steps):
        h.copy_(zh[i], non_blocking=True)
        step()
        out_h[i].copy_(h, non_blocking=True)
        cur.synchronize()
    e7.record()
    torch.cuda.synchronize()
    barrier()
    ms_eager = e6.elapsed_time(e7)
    # the same with the step replayed from a CUDA graph and no host wait
    # between tokens (copies and steps queued back to back)
    e4, e5 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e4.record()
    for i in range(args.steps):
        h.copy_(zh[i], non_blocking=True)
        g.replay()
        out_h[i].copy_(h, non_blocking=True)
    e5.record()
    torch.cuda.synchronize()
    barrier()
    ms_pipe = e4.elapsed_time(e5)
    M.moe_sync()

    ms, ms_e2e, ms_pipe, ms_eager = max_over_ranks([ms, ms_e2e, ms_pipe, ms_eager], world, device)
    del g
    if rank != 0:
        return
    extra = {}
    if not args.no_extra:
        extra["prefill_128"] = run_prefill(M, layers, device, reps=3, T=128)
        sweep = [run_prefill(M, layers, device, reps=2, T=T) for T in (256, 512, 1024)]
        extra["prefill_1L_1024tok"] = sweep[-1]
        extra["prefill_chunk_sweep"] = [{"rows": r["rows_per_chunk"], "us_per_chunk": r["us_per_chunk"],
                                         "tokens_per_s": r["value"], "tensor_frac": r["tensor"]["frac"],
                                         "hbm_frac": r["hbm"]["frac"]}
                                        for r in [extra["prefill_128"]] + sweep]
        extra["decode_b64"] = run_decode_b64(M, stack, device, reps=5)
        extra["streamed_lfu"] = run_streamed_lfu(M, device)
    value = whole_job_rate(ms, args.steps, world)
    e2e_val = whole_job_rate(ms_e2e, args.steps, world)
    hbm, src = peaks()
    bytes_step = step_bytes(cfg, distinct)
    achieved = bytes_step / (ms / args.steps / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u4xs16->s32,f32", "data": "synthetic",
        "config": {"workload": "decode_30L_b1", "layers": cfg.layers, "batch": 1, "H": cfg.H, "E": cfg.E,
                   "k": cfg.k, "I": cfg.I, "Is": cfg.Is, "weights": "4-bit affine g64 experts, 8-bit router",
                   "routing": "Zipf(1.1) per-layer bias", "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (1.1 GB of weights per step)"},
        "roofline": {"bound": "hbm", "kernel": "k_decode_b1 (one persistent launch per step)",
                     "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "peak_source": src, "traffic": decode_traffic(cfg.layers), "bytes_per_step": bytes_step,
                     "distinct_experts_per_layer": distinct},
        "e2e": {"value": e2e_val, "unit": "tokens/s", "h2d_bytes_per_step": H * 4, "d2h_bytes_per_step": H * 4,
                "mode": "one token per C-ABI call (moe_decode_session_step): host row copied in, 30 layers, row "
                        "copied out, host waits for it"},
        "e2e_eager": {"value": whole_job_rate(ms_eager, args.steps, world), "unit": "tokens/s",
                      "h2d_bytes_per_step": H * 4, "d2h_bytes_per_step": H * 4,
                      "mode": "one token per eager moe_decode_forward call with torch copies of the row in and "
                              "out and a host wait"},
        "e2e_pipelined": {"value": whole_job_rate(ms_pipe, args.steps, world), "unit": "tokens/s",
                          "h2d_bytes_per_step": H * 4, "d2h_bytes_per_step": H * 4,
                          "mode": "graph replay per token, copies in and out queued, no host wait between tokens"},
        "gpu_launches": M.moe_decode_launches(1, cfg.layers) * args.steps,
        "clocks": clocks,
        **extra,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_oracle()
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the prefill and batched-decode lines")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
