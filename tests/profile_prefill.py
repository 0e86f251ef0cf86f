"""Prefill chunks through one layer, for profiling the grouped expert GEMM
on the tensor cores.

    python -m tests.profile_prefill --reps 3 [--rows 128]

Uploads layer 0 of the prefill workload and runs the layer call `reps` times
on `rows` rows of the prefill workload's input stream (not a test; collected
by no test runner)."""
import argparse
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))


def main():
    import torch
    import gen
    import quantized_moe_bit_b200 as M
    from tests._support import HostLayer
    ap = argparse.ArgumentParser()
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--rows", type=int, default=128)
    args = ap.parse_args()
    from dataclasses import replace
    cfg = replace(gen.CONFIGS["prefill_1L_128tok"], T=args.rows)
    dl = HostLayer(cfg, 0).upload()
    T, H = cfg.T, cfg.H
    z = torch.from_numpy(gen.rows(cfg.seed, cfg.row_stream, T, H)).cuda()
    ho = torch.empty_like(z)
    ws = torch.empty(M.moe_layer_workspace_size(T, H, cfg.I, cfg.Is, cfg.E, cfg.k), dtype=torch.uint8, device="cuda")
    for _ in range(args.reps):
        M.moe_layer_forward(T, H, cfg.I, cfg.Is, cfg.E, cfg.k, dl.router.c, dl.bias, 0, dl.blob_ptrs, dl.shared_c, ws,
                            h_in=z, h_out=ho)
    torch.cuda.synchronize()
    M.moe_sync()
    print("ok")


if __name__ == "__main__":
    main()
