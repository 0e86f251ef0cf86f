"""Host timing of the fp64 oracle on the five workloads (a profiling driver,
not a test; collected by no test runner).

    python -m tests.time_oracle [--out FILE] [--one-core-only | --all-cores-only]

Times the oracle as it stands on all host cores (numpy's BLAS threads) and
on one core: single_layer_1tok and prefill_1L_128tok in full, the first 8
steps of decode_30L_b1 and decode_30L_b64 (every step one fresh input
through all 30 layers), and the first 128-row prompt chunk plus the first 8
decode tokens of streamed_30L_lfu (through all 30 layers, its forced
routing).  Generating a routed expert's weights is not oracle work: the
time spent inside the weight generator is measured and subtracted from
every step.  Prints one JSON object (tokens/s per workload and mode)."""
import argparse
import json
import os
import sys
import time

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import numpy as np  # noqa: E402

import gen  # noqa: E402
from oracle import moe_oracle as O  # noqa: E402


class Layers:
    """The oracle's per-layer tuples of a workload; routed experts come from
    the generator on demand, and the time spent generating is accumulated."""

    def __init__(self, cfg):
        self.cfg = cfg
        self.gen_s = 0.0
        self.routers = [gen.router_weights(cfg.seed, l, cfg.E, cfg.H) for l in range(cfg.layers)]
        self.shared = [gen.shared_weights(cfg.seed, l, cfg.H, cfg.Is) for l in range(cfg.layers)]
        self.zipf = [gen.zipf_bias(cfg.seed, l, cfg.E) if cfg.zipf else None for l in range(cfg.layers)]

    def expert_fn(self, l):
        def f(e):
            t0 = time.perf_counter()
            w = gen.expert_weights(self.cfg.seed, l, e, self.cfg.H, self.cfg.I)
            self.gen_s += time.perf_counter() - t0
            return w
        return f

    def tuples(self, biases=None):
        return [(self.routers[l], self.zipf[l] if biases is None else biases[l], self.expert_fn(l), self.shared[l])
                for l in range(self.cfg.layers)]


def timed(L, fn):
    """Wall time of fn() minus the weight generation inside it."""
    g0 = L.gen_s
    t0 = time.perf_counter()
    fn()
    return time.perf_counter() - t0 - (L.gen_s - g0)


def run_mode(one_core: bool):
    from threadpoolctl import threadpool_limits
    ctx = threadpool_limits(1) if one_core else None
    out = {}
    try:
        if ctx is not None:
            ctx.__enter__()
        for name in ("single_layer_1tok", "prefill_1L_128tok"):
            c = gen.CONFIGS[name]
            L = Layers(c)
            z = gen.rows(c.seed, c.row_stream, c.T, c.H).astype(np.float64)
            s = timed(L, lambda: O.stack_forward(z, L.tuples(), c.k, c.E))
            out[name] = {"s": s, "tokens": c.T, "tokens_per_s": c.T / s, "scope": "in full"}
        for name in ("decode_30L_b1", "decode_30L_b64"):
            c = gen.CONFIGS[name]
            L = Layers(c)
            ts = []
            for st in range(8):
                z = gen.rows(c.seed, c.row_stream + st, c.T, c.H).astype(np.float64)
                ts.append(timed(L, lambda: O.stack_forward(z, L.tuples(), c.k, c.E)))
            out[name] = {"s": sum(ts), "tokens": 8 * c.T, "tokens_per_s": 8 * c.T / sum(ts),
                         "s_per_step": [round(t, 3) for t in ts], "scope": "first 8 steps, 30 layers each"}
        c = gen.CONFIGS["streamed_30L_lfu"]
        L = Layers(c)
        n_tok = c.prompt_tokens + c.decode_steps
        sets = [gen.forced_routing(c.seed, l, n_tok, c.E, c.k) for l in range(c.layers)]
        prompt = gen.rows(c.seed, 3000, c.prompt_tokens, c.H).astype(np.float64)
        units = [(prompt[:c.T], 0)] + [(gen.rows(c.seed, 4000 + d, 1, c.H).astype(np.float64), c.prompt_tokens + d)
                                       for d in range(8)]
        ts = []
        for z, t0 in units:
            T = z.shape[0]
            biases = [gen.forced_bias(sets[l][t0:t0 + T], c.E).astype(np.float64) for l in range(c.layers)]
            ts.append(timed(L, lambda: O.stack_forward(z, L.tuples(biases), c.k, c.E)))
        out["streamed_30L_lfu"] = {"s": sum(ts), "tokens": c.T + 8, "tokens_per_s": (c.T + 8) / sum(ts),
                                   "chunk_s": round(ts[0], 3), "decode_s_per_token": [round(t, 3) for t in ts[1:]],
                                   "scope": "first 128-row prompt chunk and first 8 decode tokens, 30 layers each"}
    finally:
        if ctx is not None:
            ctx.__exit__(None, None, None)
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--out", default=None)
    g = ap.add_mutually_exclusive_group()
    g.add_argument("--one-core-only", action="store_true")
    g.add_argument("--all-cores-only", action="store_true")
    args = ap.parse_args()
    res = {"host_cores": os.cpu_count()}
    if not args.one_core_only:
        res["all_cores"] = run_mode(False)
    if not args.all_cores_only:
        res["one_core"] = run_mode(True)
    txt = json.dumps(res, indent=1)
    if args.out:
        with open(args.out, "w") as f:
            f.write(txt)
    print(txt)


if __name__ == "__main__":
    main()
