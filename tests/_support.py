"""Test support: building seeded layers on both sides and the comparison rules.

Inputs come from the generator; expected values come from the oracle only.
"""
from __future__ import annotations

import numpy as np

import gen
from oracle import moe_oracle as O

# Output tolerance of the bf16 layer output against the fp64 oracle, per
# compared tensor: max |err| <= 2e-2 * rms and mean |err| <= 2e-3 * rms, rms
# taken over the oracle's values.
MAX_TOL = 2e-2
MEAN_TOL = 2e-3
GAP = 1e-3


class HostLayer:
    """Host-side weights of one layer from the generator."""

    def __init__(self, cfg, layer: int, with_blobs: bool = True):
        self.cfg, self.layer = cfg, layer
        c = cfg
        self.router = gen.router_weights(c.seed, layer, c.E, c.H)
        self.bias = gen.zipf_bias(c.seed, layer, c.E) if c.zipf else None
        self.shared = gen.shared_weights(c.seed, layer, c.H, c.Is)
        self.stride = gen.synth.default_blob_stride(c.H, c.I)
        self.blobs = gen.layer_blobs(c.seed, layer, c.E, c.H, c.I, self.stride) if with_blobs else None
        self._cache = {}

    def expert(self, e: int):
        if e not in self._cache:
            self._cache[e] = gen.expert_weights(self.cfg.seed, self.layer, e, self.cfg.H, self.cfg.I)
        return self._cache[e]

    def upload(self, device="cuda"):
        from quantized_moe_bit_b200.weights import upload_layer
        return upload_layer(self.router, self.bias, self.shared, self.blobs, device)


def gap_ok_predicate(hl: HostLayer, bias_row=None):
    """Accept a candidate input row only if the oracle's logits of its
    normalised bf16 form keep every gap among the k+1 largest >= GAP."""
    k = hl.cfg.k

    def ok(z):
        _, x = O.rmsnorm(z[None, :].astype(np.float64))
        b = hl.bias if bias_row is None else bias_row
        lg = O.router_logits(x, hl.router, b)
        return not bool(O.near_tie_rows(lg, k, GAP)[0])
    return ok


def check_routing(gpu_idx: np.ndarray, logits: np.ndarray, k: int):
    """Selection parity.  Rows without a near tie must match the oracle's
    top-k exactly (ids and order).  At a near tie the GPU's list must still be
    a valid top-k within GAP: distinct, descending within GAP, and no excluded
    expert above the smallest selected one by more than GAP.  Returns the
    number of near-tie rows."""
    want = O.top_k(logits, k)
    ties = O.near_tie_rows(logits, k, GAP)
    for t in range(logits.shape[0]):
        if not ties[t]:
            assert np.array_equal(gpu_idx[t], want[t]), (t, gpu_idx[t], want[t])
        else:
            sel = [int(e) for e in gpu_idx[t]]
            assert len(set(sel)) == k
            v = logits[t, sel]
            assert np.all(np.diff(v) <= GAP), (t, v)
            rest = np.delete(logits[t], sel)
            assert rest.max() <= v.min() + GAP
    return int(ties.sum())


def bf16_half_ulp(ref: np.ndarray) -> np.ndarray:
    """Half the bf16 spacing at |ref| (8 significant bits)."""
    a = np.maximum(np.abs(ref), np.finfo(np.float64).tiny)
    return 0.5 * np.exp2(np.floor(np.log2(a)) - 7)


def check_output(y_gpu_bits: np.ndarray, ref: np.ndarray, what: str = "y"):
    """bf16 output against the fp64 oracle.  The output is bf16, so rounding
    the exact value to bf16 is not an error of the computation: the max bound
    is applied on top of half a bf16 unit of the exact value (an element at 6
    rms already carries up to 2.3e-2 rms of pure rounding); the mean bound
    includes the rounding.  The plain max |err| / rms is reported beside the
    excess over the rounding so the margin against the stated bound stays
    visible.  Returns (plain max, excess over rounding, mean), each / rms."""
    y = O.bf16_to_f64(y_gpu_bits)
    err = np.abs(y - ref)
    rms = float(np.sqrt(np.mean(ref * ref)))
    plain = float(err.max()) / rms
    excess = float(np.max(err - bf16_half_ulp(ref))) / rms
    mean = float(err.mean()) / rms
    assert excess <= MAX_TOL and mean <= MEAN_TOL, \
        f"{what}: max {plain:.3e} (beyond bf16 rounding {excess:.3e}), mean {mean:.3e} (x rms)"
    return plain, excess, mean


def check_close(a: np.ndarray, ref: np.ndarray, max_rel: float, mean_rel: float, what: str):
    err = np.abs(np.asarray(a, dtype=np.float64) - ref)
    rms = float(np.sqrt(np.mean(ref * ref))) or 1.0
    mx, mean = float(err.max()) / rms, float(err.mean()) / rms
    assert mx <= max_rel and mean <= mean_rel, f"{what}: max {mx:.3e} mean {mean:.3e} (x rms)"
    return mx, mean


class HostStack:
    """Per-layer host weights of a multi-layer workload, generated on demand
    (router, bias, shared expert, expert lookup) for the oracle side."""

    def __init__(self, cfg):
        self.cfg = cfg
        self._layers = {}

    def layer(self, l: int) -> HostLayer:
        if l not in self._layers:
            self._layers[l] = HostLayer(self.cfg, l, with_blobs=False)
        return self._layers[l]


def upload_stack(cfg, device="cuda"):
    """All layers of a workload on the device (one layer of host blobs at a time)."""
    import gen as G
    from quantized_moe_bit_b200.weights import upload_layer
    stride = G.synth.default_blob_stride(cfg.H, cfg.I)
    host = np.empty((cfg.E, stride), dtype=np.uint8)
    out = []
    for l in range(cfg.layers):
        router = G.router_weights(cfg.seed, l, cfg.E, cfg.H)
        bias = G.zipf_bias(cfg.seed, l, cfg.E) if cfg.zipf else None
        shared = G.shared_weights(cfg.seed, l, cfg.H, cfg.Is)
        G.layer_blobs(cfg.seed, l, cfg.E, cfg.H, cfg.I, stride, out=host, threads=16)
        out.append(upload_layer(router, bias, shared, host, device))
    return out
