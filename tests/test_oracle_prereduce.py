"""Pins for the oracle of the receiver-side pre-reduced combine: gates
dispatched with the rows ("Training Communication-Efficient MoE ...",
footnote 3: routed probabilities travel with the hidden states), stand-in
experts applied and gate-weighted at the receiving rank, one row per (token,
rank) summed back at the source.

The whole chain has a closed form that holds whatever the placement: every
pick j of token t contributes w_tj * scale[e_tj] * x_t exactly once, so
out[t] = x_t * sum_j w_tj * scale[e_tj].  With unit scales it reduces to the
direct weighted combine of identity experts."""
from fractions import Fraction

import numpy as np
import pytest


def _setup(seed, T=60, E=16, k=4, G=4, d=5):
    rng = np.random.default_rng(seed)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    z = rng.standard_normal((T, k)).astype(np.float32)
    w = (np.exp(z) / np.exp(z).sum(1, keepdims=True)).astype(np.float32)
    x = rng.standard_normal((T, d)).astype(np.float32)
    scale = rng.uniform(0.5, 2.0, E).astype(np.float32)
    e2r = rng.permutation(np.arange(E, dtype=np.int32) // (E // G)).astype(np.int32)
    return rng, ids, w, x, scale, e2r


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_gate_dispatch_carries_each_pick_once(orc, seed):
    rng, ids, w, x, scale, e2r = _setup(seed)
    p = orc.plan(ids, 16, 4, 2, e2r)
    se, sw = orc.dispatch_gates(ids, w, p["row_token"], p["row_jmask"])
    T, k = ids.shape
    seen = np.zeros((T, k), int)
    for i, t in enumerate(p["row_token"]):
        for j in range(k):
            if se[i, j] >= 0:
                assert se[i, j] == ids[t, j] and sw[i, j] == w[t, j]
                seen[t, j] += 1
            else:
                assert sw[i, j] == 0
    assert (seen == 1).all()
    # the row's gates sum, over a token's rows, to the token's gate total
    tot = np.zeros(T)
    np.add.at(tot, p["row_token"], sw.astype(np.float64).sum(1))
    np.testing.assert_allclose(tot, w.astype(np.float64).sum(1), rtol=1e-12)


@pytest.mark.parametrize("seed,src", [(3, False), (4, True), (5, True)])
def test_chain_closed_form(orc, seed, src):
    rng, ids, w, x, scale, e2r = _setup(seed, T=64)
    s = rng.integers(0, 4, 64).astype(np.int32) if src else None
    p = orc.plan(ids, 16, 4, 2, e2r, src_rank=s)
    send = orc.permute(x, p["row_token"])
    se, sw = orc.dispatch_gates(ids, w, p["row_token"], p["row_jmask"])
    y = orc.expert_reduce(send, se, sw, scale, y_is_bf16=False)
    out = orc.combine_rows(y.astype(np.float32), p["row_of"])
    g = (w.astype(np.float64) * scale.astype(np.float64)[ids]).sum(1)
    ref = x.astype(np.float64) * g[:, None]
    # y was rounded to fp32 before the source sum: allow that rounding
    mag = np.abs(x.astype(np.float64)) * (np.abs(w.astype(np.float64)) * scale[ids]).sum(1)[:, None]
    assert (np.abs(out - ref) <= 2.0 ** -23 * mag * ids.shape[1] + 1e-300).all()
    # fp64 rows summed exactly in fp64: within a few fp64 roundings
    out64 = np.zeros_like(ref)
    for t in range(64):
        for r in sorted(set(p["row_of"][t].tolist())):
            out64[t] += y[r]
    np.testing.assert_allclose(out64, ref, rtol=1e-13, atol=1e-300)


def test_unit_scales_equal_direct_combine(orc):
    rng, ids, w, x, scale, e2r = _setup(6, T=48)
    p = orc.plan(ids, 16, 4, 4, e2r)
    send = orc.permute(x, p["row_token"])
    se, sw = orc.dispatch_gates(ids, w, p["row_token"], p["row_jmask"])
    y = orc.expert_reduce(send, se, sw, np.ones(16, np.float32), y_is_bf16=False)
    out = np.zeros((48, x.shape[1]))
    for t in range(48):
        for r in set(p["row_of"][t].tolist()):
            out[t] += y[r]
    direct = orc.combine(send, p["row_of"], w, y_is_bf16=False)
    np.testing.assert_allclose(out, direct, rtol=1e-13, atol=1e-300)


def test_expert_reduce_exact_small(orc):
    # one row, picks 0 and 2 on it: y = w0*s[e0]*x + w2*s[e2]*x, checked exactly
    send = np.array([[1.5, -2.0, 0.25]], np.float32)
    se = np.array([[3, -1, 1]], np.int32)
    sw = np.array([[0.25, 0.0, 0.5]], np.float32)
    scale = np.array([1.0, 3.0, 1.0, -2.0], np.float32)
    y = orc.expert_reduce(send, se, sw, scale, y_is_bf16=False)
    want = [float(Fraction(0.25) * Fraction(-2.0) * Fraction(v) + Fraction(0.5) * Fraction(3.0) * Fraction(v))
            for v in send[0].tolist()]
    assert y[0].tolist() == want
    with pytest.raises(orc.OracleError):
        orc.expert_reduce(send, np.array([[4, -1, 1]], np.int32), sw, scale, y_is_bf16=False)


def test_combine_rows_counts_each_row_once(orc):
    y = np.array([[1.0, 2.0], [10.0, 20.0], [100.0, 200.0]], np.float32)
    row_of = np.array([[0, 0, 2], [1, 1, 1], [2, 0, 1]], np.int32)
    out = orc.combine_rows(y, row_of)
    assert out.tolist() == [[101.0, 202.0], [10.0, 20.0], [111.0, 222.0]]
    with pytest.raises(orc.OracleError):
        orc.combine_rows(y, np.array([[0, 3, 1]], np.int32))
