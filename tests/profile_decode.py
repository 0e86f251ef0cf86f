"""Small full-shape decode case for profiling the fused batch-1 kernel.

    python -m tests.profile_decode --layers 3

Uploads the first N layers of the 30-layer batch-1 workload and runs four
fused decode steps (not a test; collected by no test runner)."""
import argparse
import os
import sys
from dataclasses import replace

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))


def main():
    import torch
    import gen
    import quantized_moe_bit_b200 as M
    from tests._support import upload_stack
    ap = argparse.ArgumentParser()
    ap.add_argument("--layers", type=int, default=3)
    ap.add_argument("--steps", type=int, default=4)
    args = ap.parse_args()
    cfg = replace(gen.CONFIGS["decode_30L_b1"], layers=args.layers)
    layers = upload_stack(cfg)
    stack = M.DecodeStack(layers)
    ws = torch.empty(M.moe_decode_workspace_size(1, cfg.H, cfg.I, cfg.Is, cfg.E, cfg.k), dtype=torch.uint8,
                     device="cuda")
    for i in range(args.steps):
        h = torch.from_numpy(gen.rows(cfg.seed, cfg.row_stream + i, 1, cfg.H)).cuda()
        M.moe_decode_forward(h, cfg.I, cfg.Is, cfg.E, cfg.k, stack, ws)
    torch.cuda.synchronize()
    M.moe_sync()
    print("ok")


if __name__ == "__main__":
    main()
