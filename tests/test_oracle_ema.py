"""Pins for the oracle of the EMA co-activation statistics ("Cobalt", "Key
Observation": Ochiai on exponential moving averages of co-selection counts and
loads).  Checked against closed forms: the first batch is the counts
themselves, alpha = 1 forgets the past, a constant sequence is a fixed point,
three batches give the geometric weights alpha, alpha(1-alpha), (1-alpha)^2,
and Ochiai on the first batch equals the plain Ochiai."""
import numpy as np
import pytest


def _counts(orc, seed, L=2, T=500, E=12, k=3):
    rng = np.random.default_rng(seed)
    ids = np.stack([np.argsort(rng.random((T, E)), axis=1)[:, :k] for _ in range(L)]).astype(np.int32)
    return orc.coact(ids, E)


def test_first_batch_is_the_counts(orc):
    st = _counts(orc, 0)
    ema, och = orc.coact_ema(st["coact"], 0.3)
    assert (ema == st["coact"].astype(np.float64)).all()
    assert (och.view(np.uint32) == st["ochiai"].view(np.uint32)).all()


def test_alpha_one_forgets(orc):
    a, b = _counts(orc, 1), _counts(orc, 2)
    ema, _ = orc.coact_ema(a["coact"], 1.0)
    ema, och = orc.coact_ema(b["coact"], 1.0, ema)
    assert (ema == b["coact"]).all() and (och.view(np.uint32) == b["ochiai"].view(np.uint32)).all()


def test_constant_sequence_is_a_fixed_point(orc):
    a = _counts(orc, 3)
    ema, _ = orc.coact_ema(a["coact"], 0.25)
    for _ in range(5):
        ema, och = orc.coact_ema(a["coact"], 0.25, ema)
    assert (ema == a["coact"]).all() and (och.view(np.uint32) == a["ochiai"].view(np.uint32)).all()


@pytest.mark.parametrize("alpha", [0.5, 0.25, 0.125])
def test_geometric_weights(orc, alpha):
    c = [_counts(orc, s)["coact"].astype(np.float64) for s in (4, 5, 6)]
    ema, _ = orc.coact_ema(c[0].astype(np.uint32), alpha)
    ema, _ = orc.coact_ema(c[1].astype(np.uint32), alpha, ema)
    ema, och = orc.coact_ema(c[2].astype(np.uint32), alpha, ema)
    want = alpha * c[2] + alpha * (1 - alpha) * c[1] + (1 - alpha) ** 2 * c[0]
    assert (ema == want).all()            # dyadic alpha and small integers: exact
    d = np.einsum("lii->li", want)
    den = d[:, :, None] * d[:, None, :]
    ref = np.where(den > 0, want / np.sqrt(np.where(den > 0, den, 1.0)), 0.0).astype(np.float32)
    assert (och == ref).all()


def test_bad_alpha(orc):
    with pytest.raises(orc.OracleError):
        orc.coact_ema(np.zeros((1, 2, 2), np.uint32), 1.5)
