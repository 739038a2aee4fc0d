"""Seeded random shapes through the whole path against the oracle: T (ragged,
1 to 5000), E, k (1 to 8), G and rpn (divisors), d (row bytes a multiple of
16), f32 or bf16 rows, with or without explicit source ranks.  Counts, plans,
rows and targets bit-exact; combine within the fp32 bound."""
import numpy as np
import pytest
import torch

import oracle as orc
from synth import bf16_bits_to_f32, f32_to_bf16_bits

pytestmark = pytest.mark.gpu
U24 = 2.0 ** -24


@pytest.fixture(scope="module")
def cap():
    from co_activation_placement_b200 import build
    build.build()
    import co_activation_placement_b200 as cap
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    cap.lib()
    return cap


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    torch.cuda.synchronize()
    return t.cpu().numpy()


def _shape(rng):
    G = int(rng.choice([1, 2, 4, 6, 8, 16, 32, 64]))
    rpn = int(rng.choice([r for r in range(1, G + 1) if G % r == 0]))
    E = G * int(rng.integers(1, max(2, 256 // G) + 1))
    k = int(rng.integers(1, min(8, E) + 1))
    with_src = bool(rng.integers(0, 2))
    T = int(rng.integers(1, 5000))
    if not with_src:
        T = max(G, T - T % G)
    bf16 = bool(rng.integers(0, 2))
    d = int(rng.choice([8, 16, 24, 64, 136])) * (1 if bf16 else 1)
    if (d * (2 if bf16 else 4)) % 16:
        d += 8
    L = int(rng.integers(1, 4))
    return T, E, k, G, rpn, with_src, bf16, d, L


@pytest.mark.parametrize("seed", range(24))
def test_fuzz_path(cap, seed):
    rng = np.random.default_rng(1000 + seed)
    T, E, k, G, rpn, with_src, bf16, d, L = _shape(rng)
    ids = np.stack([np.argsort(rng.random((T, E)), axis=1)[:, :k] for _ in range(L)]).astype(np.int32)
    # statistics
    g = cap.coact_stats(dev(ids), E)
    o = orc.coact(ids, E)
    assert int(host(g["err"])[0]) == 0
    assert (host(g["coact"]) == o["coact"]).all()
    assert (host(g["ochiai"]).view(np.uint32) == o["ochiai"].view(np.uint32)).all()
    if L > 1:
        assert (host(g["trans"]) == o["trans"]).all()
    # plan
    e2r = rng.permutation(orc.place_uniform(E, G)).astype(np.int32)
    src = rng.integers(0, G, T).astype(np.int32) if with_src else None
    p = cap.plan_dispatch(dev(ids[0]), E, G, rpn, dev(e2r), src_rank=None if src is None else dev(src))
    op = orc.plan(ids[0], E, G, rpn, e2r, src_rank=src)
    R = op["R"]
    assert int(host(p.err)[0]) == 0
    assert host(p.summary).tolist() == op["summary"].tolist()
    assert (host(p.row_token)[:R] == op["row_token"]).all() and (host(p.row_of)[:T] == op["row_of"]).all()
    assert (host(p.row_jmask)[:R] == op["row_jmask"]).all() and (host(p.offsets) == op["offsets"]).all()
    # rows
    xf = rng.standard_normal((T, d)).astype(np.float32)
    if bf16:
        xh = f32_to_bf16_bits(xf)
        xd = dev(xh.view(np.int16)).view(torch.bfloat16)
        xf = bf16_bits_to_f32(xh)
    else:
        xh, xd = xf, dev(xf)
    send = cap.permute(xd, p.row_of, p.R_max, err=p.err)
    got = host(send.view(torch.int16) if bf16 else send)[:R]
    want = orc.permute(xh, op["row_token"])
    assert (got.view(want.dtype) == want).all()
    w = rng.random((T, k)).astype(np.float32)
    out = host(cap.combine(send, p.row_of, dev(w), out_dtype=torch.float32, err=p.err))
    Yf = orc.permute(xf, op["row_token"])
    ref = orc.combine(Yf, op["row_of"], w, y_is_bf16=False)
    mag = np.einsum("tj,tjc->tc", np.abs(w.astype(np.float64)), np.abs(Yf[op["row_of"]].astype(np.float64)))
    assert (np.abs(out - ref) <= (2 * k - 1) * U24 * mag * 1.0001 + 1e-30).all()
    # shuffle targets
    if L > 1:
        rs = orc.rank_score(o["trans"][0], e2r, G)
        tg = cap.shuffle_targets(dev(ids[0]), E, G, dev(rs))
        assert (host(tg)[:T] == orc.shuffle_targets(ids[0], E, G, rs)).all()
    assert int(host(p.err)[0]) == 0


@pytest.mark.parametrize("E", [6144, 8192, 12288])
def test_plan_many_experts(cap, E):
    # the placement table fills most of the plan kernels' shared memory
    rng = np.random.default_rng(E)
    T, k, G, rpn = 2048, 8, 64, 8
    ids = np.argsort(rng.random((T, 64)), axis=1)[:, :k].astype(np.int32) * (E // 64) + rng.integers(0, E // 64, (T, 1))
    ids = ids.astype(np.int32)
    e2r = rng.permutation(orc.place_uniform(E, G)).astype(np.int32)
    src = rng.integers(0, G, T).astype(np.int32)
    p = cap.plan_dispatch(dev(ids), E, G, rpn, dev(e2r), src_rank=dev(src))
    op = orc.plan(ids, E, G, rpn, e2r, src_rank=src)
    assert int(host(p.err)[0]) == 0
    assert host(p.summary).tolist() == op["summary"].tolist()
    assert (host(p.row_of)[:T] == op["row_of"]).all()
