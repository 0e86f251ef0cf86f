"""Plain fp64 CPU oracle of the routed Mixture-of-Experts layer.

TEST INFRASTRUCTURE.  Only the tests, the package smoke check and the
benchmark's CPU-baseline leg may import this module.  The CUDA library never
does, and this module imports nothing from it.

What it computes, step by step, for rows x of one layer (numpy, float64
throughout; a matmul is the only library primitive used):

  A0  x = bf16( h / sqrt(mean(h^2) + 1e-6) )                (multi-layer input)
  A1  logits[t, e] = sum_c w_r[e, c] * x[t, c] + beta[e]    (8-bit affine router)
  A2  idx[t] = the k largest logits, descending, ties to the lower expert id;
      gates[t] = softmax over those k logits
  A3  per expert, ascending: the pairs p = t*k + j with idx[t, j] = e, t ascending
  A4  a = W_g x, u = W_u x, act = gelu_tanh(a) * u           (per pair)
  A5  y_pair = W_d act
  A6  ysh = W_sd (gelu_tanh(W_sg x) * W_su x)               (every row)
  A7  out[t] = sum_j gates[t, j] * y_pair[t*k + j] + ysh[t]

Sources:
  * "TurboFieldfare: Gemma 4 26B on an 8 GB MacBook, in ~2 GB of RAM"
    (blog-mushroom.pages.dev), section "Why 26B Fits in 2 GB": the router
    picks 8 of 128 experts per token in each of 30 layers; the shared-expert
    branch runs beside the routed experts and the two outputs are merged;
    prefill chunks of up to 128 rows let one expert's weights serve the chunk.
  * "TurboFieldfareとは｜26BのGemma 4を約2GBのRAMで動かすSwift製ランタイムの実像"
    (ai-heartland.com), section "TurboFieldfareとは": MLX affine 4-bit, group 64,
    bf16 scale and bias; the router projection alone is 8-bit; shared and routed
    experts are 4-bit.
  * The layer definition of this library's workloads (the pages do not give
    it): softmax over the top-8 logits, gelu_tanh(gate) * up, an ungated
    shared expert added to the gate-weighted sum, an eps = 1e-6 RMS norm with
    no learned weight on the layer input, and a residual add between layers.

Readings where the pages are silent: low nibble (low byte) first inside a
word; scale and bias per output row per group of 64 inputs; gelu_tanh is the
tanh approximation 0.5 z (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3))).
"""
from __future__ import annotations

import math

import numpy as np

# ----------------------------------------------------------------------------- bf16


def bf16_to_f64(bits) -> np.ndarray:
    """bfloat16 bit patterns -> float64 (exact: bf16 is the top half of fp32)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16(x) -> np.ndarray:
    """float64 -> bfloat16 bits, one rounding to nearest, ties to even.

    Done on the float64 value directly (not via float32) by locating the two
    neighbouring bf16 values with math.frexp; only finite normal inputs occur.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    flat, oflat = x.reshape(-1), out.reshape(-1)
    for n in range(flat.size):
        v = float(flat[n])
        if v == 0.0:
            oflat[n] = 0x8000 if math.copysign(1.0, v) < 0 else 0
            continue
        m, e = math.frexp(abs(v))          # |v| = m * 2^e, m in [0.5, 1)
        scaled = m * 256.0                 # 8 significant bits -> [128, 256)
        lo = math.floor(scaled)
        rem = scaled - lo
        if rem > 0.5 or (rem == 0.5 and lo % 2 == 1):
            lo += 1
        val = math.ldexp(lo, e - 8)
        bits = np.array([math.copysign(val, v)], dtype=np.float32).view(np.uint32)[0] >> 16
        oflat[n] = bits
    return out


# ------------------------------------------------------------------------ dequant
def unpack_codes(q_words: np.ndarray, inn: int, bits: int) -> np.ndarray:
    """Integer codes [o, inn] from packed words: element c sits at bit
    bits*(c % per) of word c // per (per = 32 / bits), low bits first."""
    per = 32 // bits
    w = np.asarray(q_words, dtype=np.uint32)
    shifts = (bits * np.arange(per, dtype=np.uint32))
    codes = (w[:, :, None] >> shifts[None, None, :]) & np.uint32((1 << bits) - 1)
    return codes.reshape(w.shape[0], -1)[:, :inn].astype(np.int64)


def dequant(m) -> np.ndarray:
    """w[r, c] = S[r, c//64] * q[r, c] + B[r, c//64]   (float64 [out, inn])."""
    q = unpack_codes(m.q, m.inn, m.bits).astype(np.float64)
    s = np.repeat(bf16_to_f64(m.s), 64, axis=1)
    b = np.repeat(bf16_to_f64(m.b), 64, axis=1)
    return s * q + b


# --------------------------------------------------------------------------- A0
def rmsnorm(h: np.ndarray, eps: float = 1e-6):
    """x = bf16(h / sqrt(mean(h^2) + eps)) per row; returns (bits, float64 value)."""
    h = np.asarray(h, dtype=np.float64)
    r = np.sqrt(np.mean(h * h, axis=1, keepdims=True) + eps)
    bits = f64_to_bf16(h / r)
    return bits, bf16_to_f64(bits)


# ------------------------------------------------------------------------ A1, A2
def router_logits(x: np.ndarray, router, bias=None) -> np.ndarray:
    """logits [T, E] = x @ W_r^T (+ bias [E] or [T, E])."""
    W = dequant(router)
    lg = np.asarray(x, dtype=np.float64) @ W.T
    if bias is not None:
        lg = lg + np.asarray(bias, dtype=np.float64)
    return lg


def top_k(logits: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest logits per row, in descending logit order,
    an exact tie going to the lower expert id (sort on (-logit, id))."""
    T, E = logits.shape
    idx = np.empty((T, k), dtype=np.int32)
    ids = np.arange(E)
    for t in range(T):
        order = np.lexsort((ids, -logits[t]))
        idx[t] = order[:k]
    return idx


def softmax_gates(logits: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """g_j = exp(l_j - l_0) / sum_i exp(l_i - l_0) over the selected logits."""
    sel = np.take_along_axis(logits, idx.astype(np.int64), axis=1)
    z = np.exp(sel - sel[:, :1])
    return z / z.sum(axis=1, keepdims=True)


def near_tie_rows(logits: np.ndarray, k: int, min_gap: float = 1e-3) -> np.ndarray:
    """True where two of the k+1 largest logits of a row are closer than
    min_gap (the selection there is decided by rounding, not by the data)."""
    s = -np.sort(-logits, axis=1)[:, :k + 1]
    return (np.diff(-s, axis=1) < min_gap).any(axis=1)


# --------------------------------------------------------------------------- A3
def buckets(idx: np.ndarray, E: int):
    """Group the (t, j) pairs by expert: returns offsets [E+1], pairs [T*k]
    (value t*k + j, experts ascending, t then j ascending inside one expert),
    and the ascending list of experts that received at least one pair."""
    T, k = idx.shape
    lists = [[] for _ in range(E)]
    for t in range(T):
        for j in range(k):
            lists[int(idx[t, j])].append(t * k + j)
    offsets = np.zeros(E + 1, dtype=np.int32)
    pairs = np.empty(T * k, dtype=np.int32)
    n = 0
    for e in range(E):
        offsets[e] = n
        for p in lists[e]:
            pairs[n] = p
            n += 1
    offsets[E] = n
    active = np.array([e for e in range(E) if lists[e]], dtype=np.int32)
    return offsets, pairs, active


# ---------------------------------------------------------------------- A4 - A6
def gelu_tanh(z):
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * z * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (z + 0.044715 * z ** 3)))


def mlp(x: np.ndarray, gate, up, down, dense=None) -> np.ndarray:
    """GeGLU MLP from affine-quantised weights: W_d (gelu_tanh(W_g x) * (W_u x)).
    x is [n, inn]; `dense` may carry already dequantised (Wg, Wu, Wd)."""
    Wg, Wu, Wd = dense if dense is not None else (dequant(gate), dequant(up), dequant(down))
    x = np.asarray(x, dtype=np.float64)
    act = gelu_tanh(x @ Wg.T) * (x @ Wu.T)
    return act @ Wd.T


# --------------------------------------------------------------------------- A7
def combine(y_pairs: np.ndarray, gates: np.ndarray, ysh: np.ndarray) -> np.ndarray:
    """out[t] = sum_j gates[t, j] * y_pairs[t*k + j] + ysh[t]."""
    T, k = gates.shape
    yp = y_pairs.reshape(T, k, -1)
    return np.einsum("tj,tjh->th", gates, yp) + ysh


# ------------------------------------------------------------------ whole layer
def layer_forward(x: np.ndarray, router, bias, expert_fn, shared, k: int, E: int,
                  idx: np.ndarray | None = None):
    """One routed-MoE layer on rows x (float64 [T, H]).

    expert_fn(e) -> (gate, up, down) q-matrices of routed expert e.
    If `idx` is given, that selection is used (gates still come from the
    logits); otherwise the oracle's own top-k is used.
    Returns a dict with logits, idx, gates, offsets, pairs, active, y_pairs,
    ysh and out.
    """
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[0]
    lg = router_logits(x, router, bias)
    if idx is None:
        idx = top_k(lg, k)
    g = softmax_gates(lg, idx)
    offsets, pairs, active = buckets(idx, E)
    H = x.shape[1]
    y_pairs = np.zeros((T * k, H))
    for e in active:
        plist = pairs[offsets[e]:offsets[e + 1]]
        gate, up, down = expert_fn(int(e))
        y_pairs[plist] = mlp(x[plist // k], gate, up, down)
    ysh = mlp(x, *shared)
    out = combine(y_pairs, g, ysh)
    return dict(logits=lg, idx=idx, gates=g, offsets=offsets, pairs=pairs,
                active=active, y_pairs=y_pairs, ysh=ysh, out=out)


def stack_forward(h0: np.ndarray, layers, k: int, E: int, eps: float = 1e-6):
    """Several layers with A0 before each and a residual add after each:
    x_l = rmsnorm(h_l); h_{l+1} = h_l + out_l.  `layers` yields tuples
    (router, bias, expert_fn, shared).  Returns per-layer results and h."""
    h = np.asarray(h0, dtype=np.float64)
    res = []
    for (router, bias, expert_fn, shared) in layers:
        xb, x = rmsnorm(h, eps)
        r = layer_forward(x, router, bias, expert_fn, shared, k, E)
        r["x_bits"] = xb
        res.append(r)
        h = h + r["out"]
    return res, h
