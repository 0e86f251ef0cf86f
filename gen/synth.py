"""Seeded synthetic weights and inputs for the routed-MoE layer.

Only random draws and byte layout live here.  Every stream is a numpy
PCG64 ``default_rng`` keyed by a tuple, so any single expert, layer or row
block can be regenerated on its own:

  expert e of layer l       default_rng([seed, l, 100 + e])
  shared expert of layer l  default_rng([seed, l, 2])
  router of layer l         default_rng([seed, l, 1])
  Zipf permutation, layer l default_rng([seed, l, 3])
  layer-input rows          default_rng([seed, stream])   (stream >= 1000)
  forced routing, layer l   default_rng([seed, 2000 + l])

Distributions (the 4-bit experts follow the single-layer workload of the
routed-MoE description; the router and the Zipf skew follow the readings
listed in the design notes):

  4-bit q-matrix [o, i]: Q uint32 [o, i/8] uniform words (so every nibble is
      uniform in 0..15, element c at bits 4*(c%8) of word c/8),
      S = bf16(U(0.004, 0.02)), B = bf16(-8*S + N(0, 1e-3^2)) per group of 64.
  8-bit router [E, H]: Q uint32 [E, H/4] uniform words (byte c%4 of word c/4),
      S = bf16(U(2.0e-4, 4.4e-4)), B = bf16(-128*S + N(0, (0.1*S)^2)).
  layer input z: N(0, 1) rows, fp32.
"""
from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass
from typing import Callable, Optional

import numpy as np

__all__ = [
    "QMat", "bf16_bits", "bf16_bits_to_f32", "expert_weights", "shared_weights",
    "router_weights", "zipf_permutation", "zipf_probs", "zipf_bias", "rows",
    "qmat_bytes", "blob_layout", "blob_bytes", "pack_blob", "layer_blobs",
    "forced_routing", "forced_bias", "BLOB_STRIDE_ALIGN",
]

# Expert blobs are padded to whole 16 KiB pages (page-aligned, fixed-size
# blobs in one file per layer, as the streamed runtime stores them).
BLOB_STRIDE_ALIGN = 16384


@dataclass
class QMat:
    """An affine-quantised matrix [out, inn]: w = S*q + B per group of 64 inputs."""
    q: np.ndarray      # uint32 [out, inn*bits/32]
    s: np.ndarray      # uint16 (bf16 bits) [out, inn/64]
    b: np.ndarray      # uint16 (bf16 bits) [out, inn/64]
    out: int
    inn: int
    bits: int


def bf16_bits(a) -> np.ndarray:
    """Round to float32, then to bfloat16 (round to nearest even); return the bits."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _words(rng, shape) -> np.ndarray:
    return rng.integers(0, 2 ** 32, size=shape, dtype=np.uint32)


def _qmat4(rng, out: int, inn: int) -> QMat:
    assert inn % 64 == 0
    q = _words(rng, (out, inn // 8))
    s = bf16_bits(rng.uniform(0.004, 0.02, size=(out, inn // 64)))
    s64 = bf16_bits_to_f32(s).astype(np.float64)
    b = bf16_bits(-8.0 * s64 + 1e-3 * rng.standard_normal((out, inn // 64)))
    return QMat(q, s, b, out, inn, 4)


def expert_weights(seed: int, layer: int, e: int, H: int, I: int):
    """(gate [I,H], up [I,H], down [H,I]) of routed expert e in layer `layer`."""
    rng = np.random.default_rng([seed, layer, 100 + e])
    return _qmat4(rng, I, H), _qmat4(rng, I, H), _qmat4(rng, H, I)


def shared_weights(seed: int, layer: int, H: int, Is: int):
    """(gate [Is,H], up [Is,H], down [H,Is]) of the always-on shared expert."""
    rng = np.random.default_rng([seed, layer, 2])
    return _qmat4(rng, Is, H), _qmat4(rng, Is, H), _qmat4(rng, H, Is)


def router_weights(seed: int, layer: int, E: int, H: int) -> QMat:
    """8-bit affine group-64 router projection [E, H]."""
    assert H % 64 == 0
    rng = np.random.default_rng([seed, layer, 1])
    q = _words(rng, (E, H // 4))
    s = bf16_bits(rng.uniform(2.0e-4, 4.4e-4, size=(E, H // 64)))
    s64 = bf16_bits_to_f32(s).astype(np.float64)
    b = bf16_bits(-128.0 * s64 + 0.1 * s64 * rng.standard_normal((E, H // 64)))
    return QMat(q, s, b, E, H, 8)


def zipf_permutation(seed: int, layer: int, E: int) -> np.ndarray:
    """pi[e] = popularity rank (0 = most popular) of expert e in this layer."""
    return np.random.default_rng([seed, layer, 3]).permutation(E)


def zipf_probs(E: int, s: float = 1.1) -> np.ndarray:
    """p_r proportional to r^-s for ranks r = 1..E."""
    w = np.arange(1, E + 1, dtype=np.float64) ** (-s)
    return w / w.sum()


def zipf_bias(seed: int, layer: int, E: int, s: float = 1.1) -> np.ndarray:
    """Per-layer router logit bias beta[e] = ln p_{pi(e)} (fp32 [E])."""
    pi = zipf_permutation(seed, layer, E)
    return np.log(zipf_probs(E, s))[pi].astype(np.float32)


def rows(seed: int, stream: int, T: int, H: int,
         accept: Optional[Callable[[np.ndarray], bool]] = None) -> np.ndarray:
    """T rows of N(0,1) fp32 drawn in order from stream `stream`.

    With `accept`, a rejected row is replaced by the next draw of the same
    stream (the predicate is supplied by the caller; nothing here decides).
    """
    rng = np.random.default_rng([seed, stream])
    if accept is None:
        return rng.standard_normal((T, H)).astype(np.float32)
    out = np.empty((T, H), dtype=np.float32)
    n = 0
    while n < T:
        r = rng.standard_normal(H).astype(np.float32)
        if accept(r):
            out[n] = r
            n += 1
    return out


# ----------------------------------------------------------------- blob layout
def qmat_bytes(out: int, inn: int, bits: int = 4) -> int:
    return out * inn * bits // 8 + 2 * 2 * out * (inn // 64)


def blob_layout(H: int, I: int):
    """Byte offsets of the nine arrays in one expert blob, in storage order:
    gate.Q gate.S gate.B up.Q up.S up.B down.Q down.S down.B."""
    offs, o = [], 0
    for (out, inn) in ((I, H), (I, H), (H, I)):
        for nbytes in (out * inn // 2, out * (inn // 64) * 2, out * (inn // 64) * 2):
            offs.append(o)
            o += nbytes
    return offs, o


def blob_bytes(H: int, I: int) -> int:
    return blob_layout(H, I)[1]


def default_blob_stride(H: int, I: int) -> int:
    n = blob_bytes(H, I)
    return (n + BLOB_STRIDE_ALIGN - 1) // BLOB_STRIDE_ALIGN * BLOB_STRIDE_ALIGN


def pack_blob(w, stride: int, out: Optional[np.ndarray] = None) -> np.ndarray:
    """Concatenate an expert's (gate, up, down) arrays into one zero-padded blob."""
    gate, up, down = w
    if out is None:
        out = np.zeros(stride, dtype=np.uint8)
    o = 0
    for m in (gate, up, down):
        for a in (m.q, m.s, m.b):
            raw = np.ascontiguousarray(a).view(np.uint8).reshape(-1)
            out[o:o + raw.size] = raw
            o += raw.size
    assert o <= stride
    out[o:stride] = 0
    return out


def layer_blobs(seed: int, layer: int, E: int, H: int, I: int, stride: int,
                out: Optional[np.ndarray] = None, threads: int = 8) -> np.ndarray:
    """All E expert blobs of one layer as uint8 [E, stride]."""
    if out is None:
        out = np.empty((E, stride), dtype=np.uint8)

    def one(e):
        pack_blob(expert_weights(seed, layer, e, H, I), stride, out[e])

    if threads > 1:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(one, range(E)))
    else:
        for e in range(E):
            one(e)
    return out


# ------------------------------------------------------ temporally forced routing
def forced_routing(seed: int, layer: int, n_tokens: int, E: int, k: int,
                   s: float = 1.1, carry: int = 2) -> np.ndarray:
    """Expert sets for a token sequence at one layer, temporally correlated.

    Token 0 takes k distinct Zipf(s) draws.  Each later token takes `carry`
    experts drawn uniformly from the previous token's set, then k - carry
    distinct Zipf(s) draws that exclude those.  Zipf ranks map to experts
    through the layer's permutation.  Returns int32 [n_tokens, k] (sets, in
    draw order; the order carries no meaning).
    """
    rng = np.random.default_rng([seed, 2000 + layer])
    pi = zipf_permutation(seed, layer, E)
    p_e = zipf_probs(E, s)[pi]                 # probability of each expert
    sets = np.empty((n_tokens, k), dtype=np.int32)
    prev = None
    for t in range(n_tokens):
        mask = np.ones(E, dtype=bool)
        chosen = []
        if prev is not None and carry > 0:
            keep = rng.choice(prev, size=carry, replace=False)
            chosen.extend(int(e) for e in keep)
            mask[keep] = False
        p = np.where(mask, p_e, 0.0)
        p = p / p.sum()
        fresh = rng.choice(E, size=k - len(chosen), replace=False, p=p)
        chosen.extend(int(e) for e in fresh)
        sets[t] = chosen
        prev = sets[t]
    return sets


def forced_bias(sets: np.ndarray, E: int, value: float = 32.0) -> np.ndarray:
    """Per-row router bias fp32 [T, E]: +value on each row's set, 0 elsewhere."""
    T = sets.shape[0]
    b = np.zeros((T, E), dtype=np.float32)
    b[np.arange(T)[:, None], sets] = value
    return b
