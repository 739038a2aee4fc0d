"""The seeded generators: shapes, ranges, distinct picks, determinism, the
block structure that lets any block be regenerated, and the bf16 rounding."""
import numpy as np
import pytest

from synth import WORKLOADS, make_routing, make_gates, make_hidden, f32_to_bf16_bits, bf16_bits_to_f32


@pytest.mark.parametrize("name", ["tiny", "one_node", "ep32", "large_ep64"])
def test_routing_shape_and_sets(name):
    w = WORKLOADS[name]
    T = min(w.T, 70000)
    ids = make_routing(w, T=T)
    assert ids.shape == (w.L, T, w.k) and ids.dtype == np.int32
    assert ids.min() >= 0 and ids.max() < w.E
    s = np.sort(ids, axis=-1)
    assert (np.diff(s, axis=-1) > 0).all()
    assert (make_routing(w, T=T) == ids).all()
    assert not (make_routing(w, T=T, seed=1) == ids).all()


def test_routing_prefix_blocks_are_stable():
    w = WORKLOADS["ep32"]
    a = make_routing(w)
    b = make_routing(w, T=70000)
    assert (a[:, :65536] == b[:, :65536]).all()


def test_routing_is_clustered():
    # the Zipf cluster law makes some pairs far more frequent than uniform
    # routing would (the structure the correlated placement feeds on)
    w = WORKLOADS["one_node"]
    ids = make_routing(w)[0]
    a, b = np.minimum(ids[:, 0], ids[:, 1]), np.maximum(ids[:, 0], ids[:, 1])
    pair_freq = np.bincount(a * w.E + b, minlength=w.E * w.E)
    top = np.sort(pair_freq)[::-1][: int(0.01 * w.E * (w.E - 1) / 2)].sum() / w.T
    assert top > 0.2


def test_gates_softmax():
    w = WORKLOADS["tiny"]
    g = make_gates(w)
    assert g.shape == (w.L, w.T, w.k) and g.dtype == np.float32
    assert (g > 0).all()
    np.testing.assert_allclose(g.sum(-1), 1.0, atol=1e-6)


def test_hidden_blocks_and_dtype():
    w = WORKLOADS["one_node"]
    x = make_hidden(w, T=9000)
    assert x.shape == (9000, w.d) and x.dtype == np.uint16
    assert (make_hidden(w, T=4096) == x[:4096]).all()
    f = bf16_bits_to_f32(x)
    assert abs(float(f.mean())) < 0.01 and abs(float(f.std()) - 1) < 0.01
    xt = make_hidden(WORKLOADS["tiny"])
    assert xt.dtype == np.float32 and xt.shape == (4096, 128)


def test_bf16_rounding_nearest_even():
    one = np.float32(1.0)
    ulp = np.float32(2.0 ** -7)
    vals = np.array([one, one + ulp / 2, one + ulp * 1.5, one + ulp * 0.75, -2.5], np.float32)
    got = bf16_bits_to_f32(f32_to_bf16_bits(vals))
    want = np.array([1.0, 1.0, 1.0 + 2 * ulp, 1.0 + ulp, -2.5], np.float32)
    assert (got == want).all()
    torch = pytest.importorskip("torch")
    r = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 1e3
    ref = torch.from_numpy(r).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (f32_to_bf16_bits(r) == ref).all()
