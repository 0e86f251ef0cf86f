"""Pins for the fp64 oracle: closed forms, invariants and brute force.

Each test checks the oracle against something other than itself, chosen so
that a plausible slip (wrong nibble order, wrong group axis, dropped bias,
wrong sign or constant, transposed operand, unstable ordering) fails.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import gen
from gen.synth import QMat
from oracle import moe_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def bf(v):
    """bf16 bits of a value that is exactly representable in bf16."""
    b = np.array([v], dtype=np.float32).view(np.uint32)[0]
    assert b & 0xFFFF == 0
    return np.uint16(b >> 16)


def qm(words, s, b, out, inn, bits=4):
    return QMat(np.asarray(words, dtype=np.uint32).reshape(out, -1),
                np.asarray(s, dtype=np.uint16).reshape(out, -1),
                np.asarray(b, dtype=np.uint16).reshape(out, -1), out, inn, bits)


# ------------------------------------------------------------------ bf16 helpers
def test_bf16_round_trip_and_ties():
    assert O.f64_to_bf16(1.0)[()] == 0x3F80
    assert O.f64_to_bf16(-2.0)[()] == 0xC000
    # 1 + 2^-8 is the midpoint of 1 and 1 + 2^-7: ties go to the even code 0x3F80
    assert O.f64_to_bf16(1.0 + 2 ** -8)[()] == 0x3F80
    # 1 + 3*2^-8 is the midpoint of 0x3F81 and 0x3F82: even is 0x3F82
    assert O.f64_to_bf16(1.0 + 3 * 2 ** -8)[()] == 0x3F82
    # just above a midpoint rounds up
    assert O.f64_to_bf16(1.0 + 2 ** -8 + 2 ** -30)[()] == 0x3F81
    assert O.bf16_to_f64(np.uint16(0x3F81))[()] == 1.0 + 2 ** -7


def test_bf16_is_nearest():
    rng = np.random.default_rng(5)
    v = rng.standard_normal(2000) * np.exp(rng.uniform(-20, 20, 2000))
    bits = O.f64_to_bf16(v).astype(np.int64)
    got = O.bf16_to_f64(bits.astype(np.uint16))
    for d in (-1, 1):
        nb = O.bf16_to_f64((bits + d).astype(np.uint16))
        assert np.all(np.abs(v - got) <= np.abs(v - nb))


# ---------------------------------------------------------------------- dequant
def test_dequant_nibble_order_closed_form():
    # word 0x76543210 holds codes 0..7, low nibble first; S = 1, B = -8
    m = qm([0x76543210] * 8, [bf(1.0)], [bf(-8.0)], 1, 64)
    w = O.dequant(m)
    assert np.array_equal(w[0], np.tile(np.arange(-8.0, 0.0), 8))


def test_dequant_all_fifteen():
    m = qm([0xFFFFFFFF] * 16, [bf(2 ** -4)] * 2, [bf(0.0)] * 2, 2, 64)
    assert np.all(O.dequant(m) == 0.9375)


def test_dequant_group_axis_is_input_dim():
    # 2 rows x 128 inputs = 2 groups per row, different per row and per group
    words = [0x11111111] * 32
    s = [bf(1.0), bf(2.0), bf(4.0), bf(8.0)]
    b = [bf(0.0), bf(0.5), bf(-1.0), bf(0.25)]
    w = O.dequant(qm(words, s, b, 2, 128))
    assert np.all(w[0, :64] == 1.0) and np.all(w[0, 64:] == 2.5)
    assert np.all(w[1, :64] == 3.0) and np.all(w[1, 64:] == 8.25)


def test_dequant_8bit_byte_order():
    m = qm([0x03020100, 0xFF80FE01] * 16, [bf(0.5)] * 2, [bf(-1.0)] * 2, 1, 128, bits=8)
    w = O.dequant(m)[0]
    codes = np.tile([0, 1, 2, 3, 1, 254, 128, 255], 16)
    assert np.array_equal(w, 0.5 * codes - 1.0)


def naive_dequant(m):
    """Independent element-by-element dequant using integer division."""
    per = 32 // m.bits
    base = 1 << m.bits
    w = np.zeros((m.out, m.inn))
    for r in range(m.out):
        for c in range(m.inn):
            word = int(m.q[r, c // per])
            code = (word // (base ** (c % per))) % base
            s = float(O.bf16_to_f64(m.s[r, c // 64]))
            b = float(O.bf16_to_f64(m.b[r, c // 64]))
            w[r, c] = s * code + b
    return w


def test_dequant_matches_naive_on_random():
    rng = np.random.default_rng(1)
    for bits in (4, 8):
        out, inn = 3, 128
        m = qm(rng.integers(0, 2 ** 32, out * inn * bits // 32, dtype=np.uint32),
               gen.bf16_bits(rng.uniform(0.01, 0.1, out * 2)),
               gen.bf16_bits(rng.uniform(-1, 1, out * 2)), out, inn, bits)
        assert np.array_equal(O.dequant(m), naive_dequant(m))


# --------------------------------------------------------------------------- A0
def test_rmsnorm_closed_forms():
    b, x = O.rmsnorm(np.ones((1, 64)))
    assert np.all(b == 0x3F80)            # 1/sqrt(1 + 1e-6) rounds to 1.0
    b, x = O.rmsnorm(np.full((1, 64), 1e-3))
    # 1e-3 / sqrt(1e-6 + 1e-6) = 1/sqrt(2) -> bf16 0x3F35
    assert np.all(b == 0x3F35)
    h = np.array([[3.0, -4.0] * 32])      # rms = sqrt(12.5)
    b, x = O.rmsnorm(h)
    r = math.sqrt(12.5 + 1e-6)
    assert np.allclose(x[0, :2], [3 / r, -4 / r], rtol=2 ** -8)


# -------------------------------------------------------------------------- A1
def _tiny_router(seed=3, E=16, H=128):
    rng = np.random.default_rng(seed)
    return qm(rng.integers(0, 2 ** 32, E * H // 4, dtype=np.uint32),
              gen.bf16_bits(rng.uniform(2e-4, 4.4e-4, E * H // 64)),
              gen.bf16_bits(rng.uniform(-0.06, -0.05, E * H // 64)), E, H, 8)


def test_router_one_hot_gives_column():
    R = _tiny_router()
    bias = np.linspace(-1, 1, 16)
    for c in (0, 5, 64, 127):
        x = np.zeros((1, 128))
        x[0, c] = 1.0
        lg = O.router_logits(x, R, bias)[0]
        for e in range(16):
            code = (int(R.q[e, c // 4]) // 256 ** (c % 4)) % 256
            s = float(O.bf16_to_f64(R.s[e, c // 64]))
            b = float(O.bf16_to_f64(R.b[e, c // 64]))
            assert lg[e] == pytest.approx(s * code + b + bias[e], abs=1e-15)


def test_router_matches_naive_loops():
    R = _tiny_router(seed=4)
    W = naive_dequant(R)
    rng = np.random.default_rng(7)
    x = rng.standard_normal((3, 128))
    bias = rng.standard_normal((3, 16))   # per-row bias
    lg = O.router_logits(x, R, bias)
    for t in range(3):
        for e in range(16):
            acc = sum(W[e, c] * x[t, c] for c in range(128)) + bias[t, e]
            assert lg[t, e] == pytest.approx(acc, rel=1e-12, abs=1e-12)


# -------------------------------------------------------------------------- A2
def test_topk_is_max_sum_subset_bruteforce():
    rng = np.random.default_rng(11)
    for _ in range(20):
        lg = rng.standard_normal((1, 16))
        idx = O.top_k(lg, 4)[0]
        best = max(itertools.combinations(range(16), 4), key=lambda s: sum(lg[0, list(s)]))
        assert set(idx) == set(best)
        assert all(lg[0, idx[j]] > lg[0, idx[j + 1]] for j in range(3))


def test_topk_ties_go_to_lower_id():
    lg = np.array([[0.0, 2.0, 1.0, 2.0, 1.0, 1.0]])
    assert list(O.top_k(lg, 4)[0]) == [1, 3, 2, 4]
    assert list(O.top_k(np.zeros((1, 8)), 3)[0]) == [0, 1, 2]


def test_topk_permutation_invariance():
    rng = np.random.default_rng(12)
    R = _tiny_router(seed=9)
    x = rng.standard_normal((4, 128))
    bias = rng.standard_normal(16)
    lg = O.router_logits(x, R, bias)
    idx = O.top_k(lg, 4)
    g = O.softmax_gates(lg, idx)
    perm = rng.permutation(16)            # new row p holds old expert perm[p]
    Rp = QMat(R.q[perm], R.s[perm], R.b[perm], 16, 128, 8)
    lgp = O.router_logits(x, Rp, bias[perm])
    idxp = O.top_k(lgp, 4)
    assert np.array_equal(perm[idxp], idx)
    assert np.allclose(O.softmax_gates(lgp, idxp), g, rtol=0, atol=1e-15)


def test_gates_closed_forms():
    lg = np.random.default_rng(2).standard_normal((5, 16))
    idx = O.top_k(lg, 8)
    g = O.softmax_gates(lg, idx)
    assert np.allclose(g.sum(1), 1.0, atol=1e-15)
    assert np.all(np.diff(g, axis=1) <= 0)              # descending with the logits
    assert np.allclose(O.softmax_gates(np.zeros((1, 16)), O.top_k(np.zeros((1, 16)), 8)), 1 / 8)
    lg2 = np.array([[0.3, -1.2, 5.0]])
    g2 = O.softmax_gates(lg2, np.array([[2, 0]]))
    assert g2[0, 0] == pytest.approx(1 / (1 + math.exp(0.3 - 5.0)), rel=1e-14)


def test_near_tie_detection():
    lg = np.array([[5.0, 4.0, 3.0, 2.0, 1.9995, 0.0],
                   [5.0, 4.0, 3.0, 2.0, 1.0, 0.0]])
    assert list(O.near_tie_rows(lg, 4)) == [True, False]   # gap at the k/k+1 boundary
    assert list(O.near_tie_rows(lg, 3)) == [False, False]  # below the k+1 largest
    assert list(O.near_tie_rows(lg, 2)) == [False, False]


# -------------------------------------------------------------------------- A3
def test_buckets_bruteforce():
    rng = np.random.default_rng(13)
    T, k, E = 9, 4, 16
    idx = np.array([rng.choice(E, k, replace=False) for _ in range(T)], dtype=np.int32)
    off, pairs, active = O.buckets(idx, E)
    assert off[E] == T * k and np.all(np.diff(off) >= 0)
    for e in range(E):
        want = [t * k + j for t in range(T) for j in range(k) if idx[t, j] == e]
        assert list(pairs[off[e]:off[e + 1]]) == want
    assert list(active) == sorted(set(idx.reshape(-1).tolist()))


# ------------------------------------------------------------------------ GeGLU
def test_gelu_tanh_against_erf_gelu():
    z = np.linspace(-12, 12, 48001)
    exact = 0.5 * z * (1 + np.array([math.erf(v / math.sqrt(2)) for v in z]))
    assert np.max(np.abs(O.gelu_tanh(z) - exact)) < 5e-4
    assert O.gelu_tanh(0.0) == 0.0
    assert O.gelu_tanh(30.0) == pytest.approx(30.0, rel=1e-15)
    assert abs(O.gelu_tanh(-30.0)) < 1e-100


# ------------------------------------------------------------------ A4 - A7
def _rand_q4(rng, out, inn, zero=False):
    if zero:
        return qm(np.zeros(out * inn // 8, np.uint32), np.zeros(out * inn // 64, np.uint16),
                  np.zeros(out * inn // 64, np.uint16), out, inn)
    s = gen.bf16_bits(rng.uniform(0.004, 0.02, out * inn // 64))
    b = gen.bf16_bits(-8 * gen.bf16_bits_to_f32(s) + 1e-3 * rng.standard_normal(out * inn // 64))
    return qm(rng.integers(0, 2 ** 32, out * inn // 8, dtype=np.uint32), s, b, out, inn)


def _tiny_expert(rng, H=128, I=64, zero=False):
    return (_rand_q4(rng, I, H, zero), _rand_q4(rng, I, H, zero), _rand_q4(rng, H, I, zero))


def test_mlp_matches_naive_loops():
    rng = np.random.default_rng(21)
    g, u, d = _tiny_expert(rng)
    Wg, Wu, Wd = naive_dequant(g), naive_dequant(u), naive_dequant(d)
    x = rng.standard_normal((2, 128))
    y = O.mlp(x, g, u, d)
    for t in range(2):
        act = []
        for i in range(64):
            a = sum(Wg[i, c] * x[t, c] for c in range(128))
            b = sum(Wu[i, c] * x[t, c] for c in range(128))
            act.append(0.5 * a * (1 + math.tanh(math.sqrt(2 / math.pi) * (a + 0.044715 * a ** 3))) * b)
        for o in range(128):
            ref = sum(Wd[o, i] * act[i] for i in range(64))
            assert y[t, o] == pytest.approx(ref, rel=1e-10, abs=1e-12)


def test_mlp_zero_and_linearity_in_down():
    rng = np.random.default_rng(22)
    g, u, d = _tiny_expert(rng)
    x = rng.standard_normal((3, 128))
    z = _tiny_expert(rng, zero=True)
    assert np.all(O.mlp(x, *z) == 0.0)
    # doubling S_d and B_d (bf16 exponent + 1) doubles the output exactly
    d2 = QMat(d.q, (d.s.astype(np.uint32) + 0x80).astype(np.uint16),
              (d.b.astype(np.uint32) + 0x80).astype(np.uint16), d.out, d.inn, 4)
    assert np.allclose(O.mlp(x, g, u, d2), 2 * O.mlp(x, g, u, d), rtol=1e-13, atol=1e-13)


def _tiny_layer(seed=31, E=6, k=2, H=128, I=64, Is=64):
    rng = np.random.default_rng(seed)
    R = _tiny_router(seed=seed, E=E, H=H)
    experts = [_tiny_expert(rng, H, I) for _ in range(E)]
    shared = _tiny_expert(rng, H, Is)
    return R, experts, shared


def test_layer_combine_closed_forms():
    E, k = 6, 2
    R, experts, shared = _tiny_layer()
    rng = np.random.default_rng(32)
    x = rng.standard_normal((4, 128))
    r = O.layer_forward(x, R, None, lambda e: experts[e], shared, k, E)
    # direct definition: sum_j g_j * expert_{idx_j}(x) + shared(x)
    for t in range(4):
        want = O.mlp(x[t:t + 1], *shared)[0]
        for j in range(k):
            want = want + r["gates"][t, j] * O.mlp(x[t:t + 1], *experts[r["idx"][t, j]])[0]
        assert np.allclose(r["out"][t], want, rtol=1e-12, atol=1e-12)
    # zero shared weights leave the routed sum
    z = _tiny_expert(rng, 128, 64, zero=True)
    r0 = O.layer_forward(x, R, None, lambda e: experts[e], z, k, E)
    assert np.allclose(r0["out"], r["out"] - r["ysh"], atol=1e-12)
    # one-hot gates pick out one expert's output
    gh = np.zeros((4, k))
    gh[:, 1] = 1.0
    oh = O.combine(r["y_pairs"], gh, np.zeros_like(r["ysh"]))
    assert np.array_equal(oh, r["y_pairs"].reshape(4, k, -1)[:, 1])
    # a zero-weight expert contributes nothing
    ez = list(experts)
    e0 = int(r["idx"][0, 0])
    ez[e0] = z
    rz = O.layer_forward(x, R, None, lambda e: ez[e], shared, k, E)
    hit = (r["idx"] == e0)
    assert np.all(rz["y_pairs"].reshape(4, k, -1)[hit] == 0.0)


def test_layer_expert_permutation_invariance():
    E, k = 6, 2
    R, experts, shared = _tiny_layer(seed=41)
    x = np.random.default_rng(42).standard_normal((5, 128))
    r = O.layer_forward(x, R, None, lambda e: experts[e], shared, k, E)
    perm = np.array([3, 0, 5, 1, 4, 2])
    Rp = QMat(R.q[perm], R.s[perm], R.b[perm], E, 128, 8)
    rp = O.layer_forward(x, Rp, None, lambda e: experts[perm[e]], shared, k, E)
    assert np.allclose(rp["out"], r["out"], rtol=1e-12, atol=1e-12)


def test_stack_identity_with_zero_weights():
    rng = np.random.default_rng(51)
    R = _tiny_router(seed=5, E=6, H=128)
    z = _tiny_expert(rng, 128, 64, zero=True)
    h0 = rng.standard_normal((2, 128))
    res, h = O.stack_forward(h0, [(R, None, lambda e: z, z)] * 3, 2, 6)
    assert np.array_equal(h, h0)
    xb0, _ = O.rmsnorm(h0)
    for r in res:
        assert np.array_equal(r["x_bits"], xb0)


# --------------------------------------------------------- golden: format sizes
def test_blob_sizes_match_the_pages():
    with open(os.path.join(GOLD, "format_sizes.json")) as f:
        g = json.load(f)
    H, I = g["H"], g["I"]
    blob = gen.blob_bytes(H, I)
    assert blob == g["expert_blob_bytes"]
    assert round(blob / 1e6, 1) == g["expert_blob_MB_printed"]
    stride = gen.synth.default_blob_stride(H, I)
    total = g["layers"] * g["experts"] * stride
    assert round(total / 2 ** 30, 2) == g["routed_total_GB_printed"]
    # the nine arrays tile the blob without gaps or overlap
    offs, end = gen.blob_layout(H, I)
    assert offs[0] == 0 and end == blob and sorted(offs) == offs
