"""The seeded generator: determinism, shapes, ranges and blob layout."""
import numpy as np

import gen


def test_expert_weights_deterministic_and_ranged():
    a = gen.expert_weights(0, 3, 17, 256, 128)
    b = gen.expert_weights(0, 3, 17, 256, 128)
    c = gen.expert_weights(0, 3, 18, 256, 128)
    for x, y in zip(a, b):
        assert np.array_equal(x.q, y.q) and np.array_equal(x.s, y.s) and np.array_equal(x.b, y.b)
    assert not np.array_equal(a[0].q, c[0].q)
    g, u, d = a
    assert g.q.shape == (128, 32) and d.q.shape == (256, 16) and d.s.shape == (256, 2)
    s = gen.bf16_bits_to_f32(np.concatenate([m.s.ravel() for m in a]))
    assert s.min() >= 0.0039 and s.max() <= 0.0201
    bb = gen.bf16_bits_to_f32(np.concatenate([m.b.ravel() for m in a]))
    r = bb / s + 8.0                       # B = -8 S + N(0, 1e-3): r ~ N(0, 1e-3)/S
    assert np.abs(r).max() < 8e-3 / 0.004 + 0.1


def test_router_and_bias():
    R = gen.router_weights(0, 0, 16, 256)
    assert R.q.shape == (16, 64) and R.bits == 8
    z = gen.zipf_bias(0, 0, 128)
    p = np.exp(z.astype(np.float64))
    assert abs(p.sum() - 1) < 1e-5
    assert np.isclose(np.sort(p)[::-1][0] / np.sort(p)[::-1][1], 2 ** 1.1, rtol=1e-4)


def test_rows_accept_replaces_rejected_in_stream_order():
    allr = gen.rows(0, 1000, 40, 64)
    take = gen.rows(0, 1000, 3, 64, accept=lambda r: r[0] > 0)
    want = [r for r in allr if r[0] > 0][:3]
    assert np.array_equal(take, np.array(want))


def test_pack_blob_roundtrip():
    H, I = 256, 128
    w = gen.expert_weights(0, 0, 1, H, I)
    stride = gen.synth.default_blob_stride(H, I)
    blob = gen.pack_blob(w, stride)
    offs, end = gen.blob_layout(H, I)
    arrays = [a for m in w for a in (m.q, m.s, m.b)]
    for o, a in zip(offs, arrays):
        raw = np.ascontiguousarray(a).view(np.uint8).reshape(-1)
        assert np.array_equal(blob[o:o + raw.size], raw)
    assert np.all(blob[end:] == 0) and stride % 16384 == 0


def test_forced_routing_structure():
    sets = gen.forced_routing(0, 2, 50, 128, 8)
    assert sets.shape == (50, 8)
    for t in range(50):
        assert len(set(sets[t].tolist())) == 8
    for t in range(1, 50):
        assert len(set(sets[t].tolist()) & set(sets[t - 1].tolist())) >= 2
    b = gen.forced_bias(sets[:3], 128)
    assert np.all((b > 0).sum(1) == 8)
