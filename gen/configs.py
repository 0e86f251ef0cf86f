"""The five synthetic workloads of the routed-MoE layer and a tiny test shape.

  single_layer_1tok    1 layer, 1 token (no routing skew)
  decode_30L_b1        30 layers, batch 1, 256 steps, residual stream, Zipf(1.1) skew
  prefill_1L_128tok    1 layer, 128 rows, Zipf(1.1) skew
  decode_30L_b64       30 layers, 64 rows per step, 64 steps, Zipf(1.1) skew
  streamed_30L_lfu     30 layers, 1024-token prompt in chunks of 128, then 128
                       decode steps; routed experts in pinned host memory,
                       16-slot LFU per layer; temporally forced routing
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Config:
    name: str
    H: int = 2816
    I: int = 704
    Is: int = 2112
    E: int = 128
    k: int = 8
    layers: int = 1
    T: int = 1            # rows per step (per chunk for the streamed workload)
    steps: int = 1
    zipf: bool = False
    seed: int = 0
    # streamed workload only
    prompt_tokens: int = 0
    decode_steps: int = 0
    n_slots: int = 16
    # input row streams
    row_stream: int = 1000

    @property
    def tokens_per_step(self) -> int:
        return self.T


CONFIGS = {
    "single_layer_1tok": Config("single_layer_1tok", layers=1, T=1, steps=1),
    "decode_30L_b1": Config("decode_30L_b1", layers=30, T=1, steps=256, zipf=True),
    "prefill_1L_128tok": Config("prefill_1L_128tok", layers=1, T=128, steps=1, zipf=True),
    "decode_30L_b64": Config("decode_30L_b64", layers=30, T=64, steps=64, zipf=True),
    "streamed_30L_lfu": Config("streamed_30L_lfu", layers=30, T=128, steps=8, zipf=False,
                               prompt_tokens=1024, decode_steps=128, n_slots=16),
}


def tiny_config(base: str = "single_layer_1tok", **kw) -> Config:
    """Small shapes (H=256, I=128, Is=192, E=16, k=4) for fast tests."""
    c = replace(CONFIGS[base], H=256, I=128, Is=192, E=16, k=4, name=base + "_tiny")
    return replace(c, **kw)
