"""Event timings of the expert-parallel layer's steps with G ranks held in
one process on one GPU (a profiling driver, not a test; collected by no test
runner).

    python -m tests.profile_ep [--ranks 8] [--tokens 128] [--reps 10]

Layer 0 of the prefill workload; every rank holds `tokens` rows of its own
input stream.  Each repetition queues the whole layer of every rank behind a
GPU sleep (so host launch costs do not enter the events) and brackets each
rank's steps with CUDA events: front (norm, router, bucketing, shared
expert), dispatch (with the receiver plan), the expert GEMM over the received
rows, return, combine.  Then each exchange kernel of the rank with the most
received rows runs 20 times back to back.  Prints one JSON object (medians
over ranks and repetitions, microseconds).  With one GPU the exchanges are
stores into this GPU's own memory: the kernels' cost without the links."""
import argparse
import json
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))


def main():
    import numpy as np
    import torch
    from dataclasses import replace
    import gen
    import quantized_moe_bit_b200 as M
    from quantized_moe_bit_b200 import binding as B, ep
    from tests._support import HostLayer
    ap = argparse.ArgumentParser()
    ap.add_argument("--ranks", type=int, default=8)
    ap.add_argument("--tokens", type=int, default=128)
    ap.add_argument("--reps", type=int, default=10)
    a = ap.parse_args()
    G, T = a.ranks, a.tokens
    cfg = replace(gen.CONFIGS["prefill_1L_128tok"], T=T)
    dl = HostLayer(cfg, 0).upload()
    ranks = [ep.EpRank(G, r, T, cfg.H, cfg.I, cfg.Is, cfg.E, cfg.k, dl) for r in range(G)]
    comm = ep.LocalRanks(ranks)
    hs = [torch.from_numpy(gen.rows(cfg.seed, cfg.row_stream + g, T, cfg.H)).cuda() for g in range(G)]
    for _ in range(3):
        ep.ep_layer_forward(ranks, comm, [h.clone() for h in hs])
    M.moe_sync()

    def ev():
        return torch.cuda.Event(enable_timing=True)

    spans = {k: [] for k in ("front", "dispatch", "experts", "return", "combine")}
    for _ in range(a.reps):
        hh = [h.clone() for h in hs]
        torch.cuda._sleep(20_000_000)
        for r, h in zip(ranks, hh):
            e0, e1 = ev(), ev()
            e0.record(); r.front(h); r.shared(); e1.record()
            spans["front"].append((e0, e1))
        comm.gather_offsets(ranks)
        for r in ranks:
            e0, e1 = ev(), ev()
            e0.record(); r.dispatch(); e1.record()
            spans["dispatch"].append((e0, e1))
        for r in ranks:
            e0, e1, e2 = ev(), ev(), ev()
            e0.record()
            B.moe_expert_forward(r.recv_x[:r.cap], r.I, r.El, 1, r.local_blobs, r.loff, r.rpairs, r.ractive, r.rn,
                                 r.y_rows, r.ws_e)
            e1.record()
            B.moe_ep_return(r.y_rows[:r.cap], r.E, r.G, r.rank, r.recv_meta, r.loff, r.T * r.k, r.peer_y_pairs)
            e2.record()
            spans["experts"].append((e0, e1))
            spans["return"].append((e1, e2))
        for r, h in zip(ranks, hh):
            e0, e1 = ev(), ev()
            e0.record(); r.combine(h); e1.record()
            spans["combine"].append((e0, e1))
    M.moe_sync()
    rows = [int(r.loff[-1].item()) for r in ranks]
    out = {"ranks": G, "tokens_per_rank": T, "rows_received": rows}
    for k, v in spans.items():
        out[k + "_us"] = round(float(np.median([x.elapsed_time(y) * 1e3 for x, y in v])), 2)
    r0 = ranks[int(np.argmax(rows))]
    for name, fn in (("dispatch", r0.dispatch),
                     ("return", lambda: B.moe_ep_return(r0.y_rows[:r0.cap], r0.E, r0.G, r0.rank, r0.recv_meta,
                                                       r0.loff, r0.T * r0.k, r0.peer_y_pairs))):
        torch.cuda._sleep(20_000_000)
        e0, e1 = ev(), ev()
        e0.record()
        for _ in range(20):
            fn()
        e1.record()
        M.moe_sync()
        out[name + "_back_to_back_us"] = round(e0.elapsed_time(e1) * 1e3 / 20, 2)
    # bytes each exchange kernel moves (read + write)
    out["dispatch_bytes_rank_of_most_rows"] = T * cfg.k * cfg.H * 2 * 2
    out["return_bytes_rank_of_most_rows"] = max(rows) * cfg.H * 4 * 2
    out["rank_of_most_rows"] = r0.rank
    for r in ranks:
        r.close()
    print(json.dumps(out, indent=1))


if __name__ == "__main__":
    main()
