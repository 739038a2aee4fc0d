"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bit-exact: counts, Ochiai (fp64 math, one rounding on both sides), plans,
permuted rows, rank scores, shuffle targets.  Combine: within the bound that
follows from the arithmetic -- fp32 weight folding and FMA accumulation give
|out - exact| <= (2k-1) 2^-24 sum_j |w_j y_j| (fp32 output; <= 1e-6 relative
for k <= 8), plus half a bf16 ulp for bf16 output.  Full-size cases run the
pipeline exactly as bench.py times it."""
import numpy as np
import pytest
import torch

import oracle as orc
from synth import WORKLOADS, make_routing, make_gates, make_hidden, bf16_bits_to_f32

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


def clustered_ids(rng, L, T, E, k, hot=0.7):
    """k distinct ids per token; most tokens draw from a small hot set."""
    out = np.empty((L, T, k), np.int32)
    hotset = rng.permutation(E)[: min(E, k + 2)]
    for l in range(L):
        u = rng.random(T) < hot
        pick_all = np.argsort(rng.random((T, E)), axis=1)[:, :k]
        pick_hot = hotset[np.argsort(rng.random((T, hotset.size)), axis=1)[:, :k]]
        out[l] = np.where(u[:, None], pick_hot, pick_all)
    return out


def combine_bound(Yf, idx, w, k, out_bf16, ref):
    mag = np.einsum("tj,tjc->tc", np.abs(w.astype(np.float64)), np.abs(Yf[idx].astype(np.float64)))
    b = (2 * k - 1) * U24 * mag * 1.0001 + 1e-30
    if out_bf16:
        b = b + 2.0 ** -8 * (np.abs(ref) + b)
    return b


# --------------------------------------------------------------- statistics

STATS_SHAPES = [  # L, T, k, E
    (1, 1, 1, 4), (2, 1000, 2, 8), (3, 4097, 3, 16), (2, 300, 8, 8), (2, 5000, 6, 64),
    (2, 3333, 8, 128), (3, 2500, 8, 256), (2, 777, 5, 1000), (1, 12345, 4, 32),
    (2, 1500, 8, 1024),                                   # the largest E the call accepts
]


@pytest.mark.parametrize("shape", STATS_SHAPES)
def test_stats_small(cap, shape):
    L, T, k, E = shape
    rng = np.random.default_rng(sum(shape))
    ids = clustered_ids(rng, L, T, E, k)
    g = cap.coact_stats(dev(ids), E)
    o = orc.coact(ids, E)
    assert int(host(g["err"])[0]) == 0
    assert (host(g["coact"]) == o["coact"]).all()
    assert (host(g["ochiai"]).view(np.uint32) == o["ochiai"].view(np.uint32)).all()
    if L > 1:
        assert (host(g["trans"]) == o["trans"]).all()


def test_stats_partial_outputs(cap):
    rng = np.random.default_rng(3)
    ids = clustered_ids(rng, 3, 2000, 64, 4)
    o = orc.coact(ids, 64)
    g = cap.coact_stats(dev(ids), 64, want=("trans",))
    assert g["coact"] is None and (host(g["trans"]) == o["trans"]).all()
    g = cap.coact_stats(dev(ids), 64, want=("ochiai",))
    assert (host(g["ochiai"]).view(np.uint32) == o["ochiai"].view(np.uint32)).all()


@pytest.mark.parametrize("name", ["tiny", "one_node", "ep32", "large_ep64", "stats_sweep"])
def test_stats_workloads_full_size(cap, name):
    w = WORKLOADS[name]
    ids = make_routing(w)
    g = cap.coact_stats(dev(ids), w.E)
    o = orc.coact(ids, w.E)
    assert int(host(g["err"])[0]) == 0
    assert (host(g["coact"]) == o["coact"]).all()
    assert (host(g["ochiai"]).view(np.uint32) == o["ochiai"].view(np.uint32)).all()
    assert (host(g["trans"]) == o["trans"]).all()


# --------------------------------------------------------------- plan

PLAN_SHAPES = [  # T, k, E, G, rpn, src mode
    (64, 1, 4, 4, 2, None), (1000, 2, 8, 4, 2, None), (4096, 2, 8, 4, 2, "rand"),
    (5000, 3, 12, 4, 1, "rand"), (777, 8, 64, 64, 8, "rand"), (1024, 8, 256, 64, 8, None),
    (2048, 6, 64, 32, 8, "skew"), (300, 4, 16, 1, 1, None), (999, 5, 40, 8, 4, "one"),
    (65536, 8, 64, 8, 8, "empty"),
    (3000, 8, 128, 64, 1, "rand"),                        # 64 nodes of one rank: every bit of the node mask
    (2048, 4, 64, 64, 64, None),                          # 64 ranks on one node: V = 0
]


def make_src(rng, mode, T, G):
    if mode is None:
        return None
    if mode == "rand":
        return rng.integers(0, G, T).astype(np.int32)
    if mode == "skew":
        return np.minimum(rng.geometric(0.3, T) - 1, G - 1).astype(np.int32)
    if mode == "one":
        return np.full(T, G - 1, np.int32)
    if mode == "empty":   # every other shard empty
        return (2 * rng.integers(0, G // 2, T)).astype(np.int32)
    raise ValueError(mode)


def check_plan(p, o, T, k):
    R = o["R"]
    assert int(host(p.err)[0]) == 0
    assert host(p.summary).tolist() == o["summary"].tolist()
    assert (host(p.dest_mask)[:T] == o["dest_mask"]).all()
    assert (host(p.counts) == o["counts"]).all()
    assert (host(p.offsets) == o["offsets"]).all()
    assert (host(p.row_token)[:R] == o["row_token"]).all()
    assert (host(p.row_jmask)[:R] == o["row_jmask"]).all()
    assert (host(p.row_of)[:T] == o["row_of"]).all()


@pytest.mark.parametrize("method", [0, 1])
@pytest.mark.parametrize("shape", PLAN_SHAPES)
def test_plan_small(cap, shape, method):
    """Both launch methods: separate kernels (0) and one cooperative launch (1)."""
    T, k, E, G, rpn, mode = shape
    rng = np.random.default_rng(T + k + E + G)
    ids = clustered_ids(rng, 1, T, E, k)[0]
    e2r = rng.permutation(orc.place_uniform(E, G)).astype(np.int32)
    src = make_src(rng, mode, T, G)
    prev = cap.plan_dispatch_method(method)
    try:
        p = cap.plan_dispatch(dev(ids), E, G, rpn, dev(e2r), src_rank=None if src is None else dev(src))
    finally:
        cap.plan_dispatch_method(prev)
    check_plan(p, orc.plan(ids, E, G, rpn, e2r, src_rank=src), T, k)


@pytest.mark.parametrize("shape", [s_ for s_ in PLAN_SHAPES if s_[5] is not None] +
                         [(131072, 8, 256, 64, 8, "rand"), (65536, 6, 64, 32, 8, "skew")])
def test_plan_presorted(cap, shape):
    """The plan in two calls -- the source order first (moe_plan_sources, on a
    second stream ordered by an event), then moe_plan_dispatch_presorted --
    equals the one-call plan and the oracle bit for bit."""
    T, k, E, G, rpn, mode = shape
    rng = np.random.default_rng(T + 3 * k + E + G)
    ids = clustered_ids(rng, 1, T, E, k)[0]
    e2r = rng.permutation(orc.place_uniform(E, G)).astype(np.int32)
    src = make_src(rng, mode, T, G)
    ids_d, e2r_d, src_d = dev(ids), dev(e2r), dev(src)
    ws = torch.empty(cap.plan_dispatch_workspace(T, k, G, True), dtype=torch.uint8, device="cuda")
    p = cap.Plan.empty(T, k, G, ids_d.device)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        cap.plan_sources(src_d, G, ws, p.err)
        ev = torch.cuda.Event()
        ev.record(side)
    torch.cuda.current_stream().wait_event(ev)
    cap.plan_dispatch(ids_d, E, G, rpn, e2r_d, src_rank=src_d, plan=p, ws=ws, presorted=True)
    check_plan(p, orc.plan(ids, E, G, rpn, e2r, src_rank=src), T, k)
    q = cap.plan_dispatch(ids_d, E, G, rpn, e2r_d, src_rank=src_d)
    for a, b in ((p.row_of, q.row_of), (p.offsets, q.offsets), (p.summary, q.summary)):
        assert (host(a) == host(b)).all()


@pytest.mark.parametrize("T,G,mode", [(131072, 64, "rand"), (524288, 64, None), (16384, 8, "skew"), (262144, 32, "rand")])
def test_plan_single_launch_large(cap, T, G, mode):
    """The single-launch plan where blocks loop over several chunks (more
    chunks than resident blocks) and at its chunk limit, against the oracle."""
    k, E = 8, 64
    rng = np.random.default_rng(T + G)
    ids = clustered_ids(rng, 1, T, E, k)[0]
    e2r = rng.permutation(orc.place_uniform(E, G)).astype(np.int32)
    src = make_src(rng, mode, T, G)
    prev = cap.plan_dispatch_method(1)
    try:
        p = cap.plan_dispatch(dev(ids), E, G, 8, dev(e2r), src_rank=None if src is None else dev(src))
    finally:
        cap.plan_dispatch_method(prev)
    check_plan(p, orc.plan(ids, E, G, 8, e2r, src_rank=src), T, k)


@pytest.mark.parametrize("method", [0, 1])
@pytest.mark.parametrize("T,k,G,shift", [(3000, 8, 64, 1), (3000, 8, 64, 2), (2048, 6, 32, 1), (2048, 6, 32, 2),
                                         (999, 5, 8, 1)])
def test_plan_row_of_alignment(cap, T, k, G, shift, method):
    """row_of in a caller's buffer that is not 16-byte (shift 1: not 8-byte)
    aligned: the plan writes a token's entries with narrower stores, same
    values as the oracle."""
    E = 4 * G
    rng = np.random.default_rng(T + 7 * k + shift)
    ids = clustered_ids(rng, 1, T, E, k)[0]
    e2r = rng.permutation(orc.place_uniform(E, G)).astype(np.int32)
    src = make_src(rng, "rand", T, G)
    p = cap.Plan.empty(T, k, G, "cuda")
    buf = torch.full((T * k + 4,), -7, dtype=torch.int32, device="cuda")
    p.row_of = buf[shift:shift + T * k].view(T, k)
    assert p.row_of.data_ptr() % 16 != 0
    prev = cap.plan_dispatch_method(method)
    try:
        cap.plan_dispatch(dev(ids), E, G, 8 if G % 8 == 0 else 1, dev(e2r), src_rank=dev(src), plan=p)
    finally:
        cap.plan_dispatch_method(prev)
    check_plan(p, orc.plan(ids, E, G, 8 if G % 8 == 0 else 1, e2r, src_rank=src), T, k)
    b = host(buf)
    assert (b[:shift] == -7).all() and (b[shift + T * k:] == -7).all()


def test_plan_reuses_workspace_and_buffers(cap):
    # the same Plan and workspace reused across calls of different sizes
    rng = np.random.default_rng(5)
    p = None
    for T, src in [(4096, True), (2048, False), (4096, False), (1000, True)]:
        ids = clustered_ids(rng, 1, T, 16, 3)[0]
        e2r = orc.place_uniform(16, 8)
        s = rng.integers(0, 8, T).astype(np.int32) if src else None
        if not src and T % 8:
            continue
        p = cap.plan_dispatch(dev(ids), 16, 8, 4, dev(e2r), src_rank=None if s is None else dev(s))
        check_plan(p, orc.plan(ids, 16, 8, 4, e2r, src_rank=s), T, 3)


# --------------------------------------------------------------- rows

@pytest.mark.parametrize("dtype,d,k", [("f32", 128, 2), ("bf16", 2048, 2), ("bf16", 96, 8), ("f32", 36, 5),
                                       ("bf16", 7168, 8)])
@pytest.mark.parametrize("out_bf16", [False, True])
def test_permute_combine_small(cap, dtype, d, k, out_bf16):
    rng = np.random.default_rng(d + k)
    T, E, G = 1111 if d < 7168 else 300, 32, 8
    ids = clustered_ids(rng, 1, T, E, k)[0]
    e2r = rng.permutation(orc.place_uniform(E, G)).astype(np.int32)
    src = rng.integers(0, G, T).astype(np.int32)
    xf = rng.standard_normal((T, d)).astype(np.float32)
    if dtype == "bf16":
        from synth import f32_to_bf16_bits
        xh = f32_to_bf16_bits(xf)
        xd = dev(xh.view(np.int16)).view(torch.bfloat16)
        xf = bf16_bits_to_f32(xh)
    else:
        xh, xd = xf, dev(xf)
    p = cap.plan_dispatch(dev(ids), E, G, 4, dev(e2r), src_rank=dev(src))
    o = orc.plan(ids, E, G, 4, e2r, src_rank=src)
    send = cap.permute(xd, p.row_of, p.R_max, err=p.err)
    R = o["R"]
    got = host(send.view(torch.int16) if dtype == "bf16" else send)[:R]
    want = orc.permute(xh, o["row_token"])
    assert (got.view(want.dtype) == want).all()
    # combine with identity experts (Y = send) and with a random Y
    z = rng.standard_normal((T, k)).astype(np.float32)
    wts = (np.exp(z) / np.exp(z).sum(1, keepdims=True)).astype(np.float32)
    out = cap.combine(send, p.row_of, dev(wts), out_dtype=torch.bfloat16 if out_bf16 else torch.float32, err=p.err)
    outf = host(out.float())
    Yf = orc.permute(xf, o["row_token"])
    ref = orc.combine(Yf, o["row_of"], wts, y_is_bf16=False)
    assert (np.abs(outf - ref) <= combine_bound(Yf, o["row_of"], wts, k, out_bf16, ref)).all()
    if out_bf16 and dtype == "bf16":
        assert (host(out.view(torch.int16)).view(np.uint16) == xh).all()   # identity round trip is exact
    idx = rng.integers(0, R, (T, k)).astype(np.int32)
    idx[:, -1] = idx[:, 0]                                                # repeated rows fold their weights
    out2 = cap.combine(send, dev(idx), dev(wts), out_dtype=torch.float32, err=p.err)
    ref2 = orc.combine(Yf, idx, wts, y_is_bf16=False)
    assert (np.abs(host(out2) - ref2) <= combine_bound(Yf, idx, wts, k, False, ref2)).all()
    assert int(host(p.err)[0]) == 0


# --------------------------------------------------------------- shuffle

@pytest.mark.parametrize("T,k,E,G", [(1000, 2, 8, 4), (4097, 8, 256, 64), (3000, 6, 64, 32), (500, 1, 16, 1)])
def test_shuffle_small(cap, T, k, E, G):
    rng = np.random.default_rng(T + G)
    ids = clustered_ids(rng, 2, T, E, k)
    st = orc.coact(ids, E)
    e2r = rng.permutation(orc.place_uniform(E, G)).astype(np.int32)
    rs = cap.rank_score(dev(st["trans"][0]), dev(e2r), G)
    rs_o = orc.rank_score(st["trans"][0], e2r, G)
    assert (host(rs) == rs_o).all()
    tg = cap.shuffle_targets(dev(ids[0]), E, G, rs)
    assert (host(tg)[:T] == orc.shuffle_targets(ids[0], E, G, rs_o)).all()
    # ties: an all-zero table sends every token to rank 0
    z = cap.shuffle_targets(dev(ids[0]), E, G, dev(np.zeros((E, G), np.uint32)))
    assert (host(z)[:T] == 0).all()


@pytest.mark.parametrize("G", [1, 2, 3, 5, 32, 63, 64])
@pytest.mark.parametrize("scale", ["small", "edge_narrow", "edge_wide", "huge"])
def test_shuffle_table_ranges(cap, G, scale):
    """Both scoring paths: 32-bit sums with one redux when G is even and k
    times the table maximum stays below 2^26, 64-bit sums otherwise (odd G,
    the boundary either side, entries up to 2^32 - 1); ties go to the lowest
    rank; an invalid token scores 0 everywhere (rank 0, error recorded)."""
    T, k, E = 3000, 8, 16 * max(1, 64 // max(G, 1))
    rng = np.random.default_rng(G * 7 + len(scale))
    ids = clustered_ids(rng, 1, T, E, k)[0]
    top = {"small": 1000, "edge_narrow": ((1 << 26) - 1) // k, "edge_wide": ((1 << 26) - 1) // k + 1,
           "huge": (1 << 32) - 1}[scale]
    tab = rng.integers(0, top + 1, (E, G), dtype=np.int64)
    tab[rng.integers(0, E), rng.integers(0, G)] = top                  # the maximum is reached
    tab[:, G // 2:] = tab[:, :1] if G > 1 and scale == "small" else tab[:, G // 2:]   # many equal scores
    tab = tab.astype(np.uint32)
    ids[5, 3] = E + 7                                                   # one invalid token
    err = cap.new_err("cuda")
    tg = host(cap.shuffle_targets(dev(ids), E, G, dev(tab), err=err))[:T]
    ids_ok = ids.copy()
    ids_ok[5] = np.arange(k)                                            # the oracle scores valid tokens only
    want = orc.shuffle_targets(ids_ok, E, G, tab)
    want[5] = 0
    assert (tg == want).all()
    assert int(host(err)[0]) == cap.DERR_ID_RANGE


# --------------------------------------------------------------- full pipeline

ROW_WORKLOADS = ["tiny", "one_node", "ep32", "large_ep64"]


@pytest.mark.parametrize("name", ROW_WORKLOADS)
@pytest.mark.parametrize("placement,shuffle", [("correlated", True), ("uniform", False)])
def test_pipeline_full_size(cap, name, placement, shuffle):
    from co_activation_placement_b200 import pipeline
    w = WORKLOADS[name]
    ids = make_routing(w)
    ids_cal = make_routing(w, seed=w.seed + 1)
    gates = make_gates(w)
    x = make_hidden(w)
    hp = pipeline.prepare(w.E, w.G, w.rpn, ids, gates, x, w.dtype, ids_cal, placement=placement,
                          shuffle=shuffle, out_dtype=torch.float32)
    hp.step()
    torch.cuda.synchronize()
    assert int(host(hp.err)[0]) == 0
    # statistics
    o = orc.coact(ids, w.E)
    assert (host(hp.stats["coact"]) == o["coact"]).all()
    assert (host(hp.stats["ochiai"]).view(np.uint32) == o["ochiai"].view(np.uint32)).all()
    assert (host(hp.stats["trans"]) == o["trans"]).all()
    # calibration: placement and rank scores from the oracle's own statistics
    oc = orc.coact(ids_cal, w.E)
    e2r_o = [orc.place_correlated(oc["coact"][l], w.G, w.rpn) if placement == "correlated"
             else orc.place_uniform(w.E, w.G) for l in range(w.L)]
    for l in range(w.L):
        assert (host(hp.e2r[l]) == e2r_o[l]).all()
    rs_o = [orc.rank_score(oc["trans"][l], e2r_o[l + 1], w.G) for l in range(w.L - 1)] if shuffle else []
    for a, b in zip(hp.rank_scores, rs_o):
        assert (host(a) == b).all()
    xf = bf16_bits_to_f32(x) if w.dtype == "bf16" else x
    rng = np.random.default_rng(0)
    src = None
    for l in range(w.L):
        op = orc.plan(ids[l], w.E, w.G, w.rpn, e2r_o[l], src_rank=src)
        check_plan(hp.plans[l], op, w.T, w.k)
        R = op["R"]
        # rows: the step reuses one send buffer for every layer (as a training
        # step would), so after the step it holds the last layer's rows; each
        # earlier layer's rows are checked through its combine output below
        if l == w.L - 1:
            rows = np.unique(np.concatenate([rng.integers(0, R, 4096), [0, R - 1]]))
            sub = host(hp.send[torch.from_numpy(rows).cuda()].view(torch.int16 if w.dtype == "bf16" else torch.float32))
            want = orc.permute(x, op["row_token"][rows])
            assert (sub.view(want.dtype) == want).all()
        # combine: sampled tokens against the oracle's fp64 combine
        toks = np.unique(np.concatenate([rng.integers(0, w.T, 1024), [0, w.T - 1]]))
        idx = op["row_of"][toks]
        need, inv = np.unique(idx, return_inverse=True)
        Ysub = orc.permute(xf, op["row_token"][need])
        ref = orc.combine(Ysub, inv.reshape(idx.shape).astype(np.int32), gates[l][toks], y_is_bf16=False)
        got = host(hp.outs[l][torch.from_numpy(toks).cuda()])
        bound = combine_bound(Ysub, inv.reshape(idx.shape), gates[l][toks], w.k, False, ref)
        assert (np.abs(got - ref) <= bound).all()
        rel = np.abs(got - ref) / np.maximum(np.abs(ref), 1e-30)
        assert np.median(rel) < 1e-6
        # any size: identity experts give out = x * sum_j w  (every token)
        if l == w.L - 1:
            outf = host(hp.outs[l])
            np.testing.assert_allclose(outf, xf * gates[l].sum(-1, dtype=np.float64)[:, None], rtol=1e-6, atol=1e-30)
        if shuffle and l + 1 < w.L:
            tg = orc.shuffle_targets(ids[l], w.E, w.G, rs_o[l])
            assert (host(hp.targets[l]) == tg).all()
            src = tg
    # determinism: a second step reproduces every output bit for bit
    first = [host(p.row_of).copy() for p in hp.plans] + [host(hp.outs[-1]).copy()]
    hp.step()
    again = [host(p.row_of) for p in hp.plans] + [host(hp.outs[-1])]
    for a, b in zip(first, again):
        assert (a.view(np.uint8) == b.view(np.uint8)).all()


# --------------------------------------------------------------- edge cases / errors

def test_empty_batch(cap):
    ids = torch.empty((2, 0, 2), dtype=torch.int32, device="cuda")
    g = cap.coact_stats(ids, 8)
    assert (host(g["coact"]) == 0).all() and (host(g["trans"]) == 0).all() and (host(g["ochiai"]) == 0).all()
    p = cap.plan_dispatch(ids[0], 8, 4, 2, dev(orc.place_uniform(8, 4)))
    assert (host(p.summary) == 0).all() and (host(p.offsets) == 0).all() and (host(p.counts) == 0).all()


def test_data_errors_are_reported_not_trapped(cap):
    E, G = 16, 4
    good = np.array([[[0, 1], [2, 3], [4, 5], [6, 7]]], np.int32)
    for bad_val, code in [(16, cap.DERR_ID_RANGE), (-3, cap.DERR_ID_RANGE)]:
        ids = good.copy(); ids[0, 2, 1] = bad_val
        assert int(host(cap.coact_stats(dev(ids), E)["err"])[0]) == code
        p = cap.plan_dispatch(dev(ids[0]), E, G, 2, dev(orc.place_uniform(E, G)))
        assert int(host(p.err)[0]) == code
    ids = good.copy(); ids[0, 1] = [3, 3]
    assert int(host(cap.coact_stats(dev(ids), E)["err"])[0]) == cap.DERR_ID_REPEAT
    assert int(host(cap.plan_dispatch(dev(ids[0]), E, G, 2, dev(orc.place_uniform(E, G))).err)[0]) == cap.DERR_ID_REPEAT
    e2r = orc.place_uniform(E, G); e2r[5] = 9
    assert int(host(cap.plan_dispatch(dev(good[0]), E, G, 2, dev(e2r)).err)[0]) == cap.DERR_RANK_RANGE
    src = np.array([0, 1, 7, 2], np.int32)
    assert int(host(cap.plan_dispatch(dev(good[0]), E, G, 2, dev(orc.place_uniform(E, G)), src_rank=dev(src)).err)[0]) \
        == cap.DERR_RANK_RANGE
    x = torch.zeros((4, 8), dtype=torch.float32, device="cuda")
    row_of = dev(np.array([[0, 1], [2, 3], [4, 99], [6, 7]], np.int32))
    err = cap.new_err("cuda")
    cap.permute(x, row_of, 8, err=err)
    assert int(host(err)[0]) == cap.DERR_ROW_RANGE
    err = cap.new_err("cuda")
    cap.combine(torch.zeros((8, 8), device="cuda"), row_of, dev(np.ones((4, 2), np.float32)), err=err)
    assert int(host(err)[0]) == cap.DERR_ROW_RANGE
    err = cap.new_err("cuda")
    cap.shuffle_targets(dev(np.array([[0, 20]], np.int32)), E, G, dev(np.zeros((E, G), np.uint32)), err=err)
    assert int(host(err)[0]) == cap.DERR_ID_RANGE
    # the context is still usable after every reported error
    assert int(host(cap.coact_stats(dev(good), E)["err"])[0]) == 0


def test_argument_errors_enqueue_nothing(cap):
    x = torch.zeros((4, 7), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cap.MoeError) as ei:
        cap.permute(x, dev(np.zeros((4, 2), np.int32)), 8)
    assert ei.value.status == cap.MOE_ERR_UNSUPPORTED
    with pytest.raises(cap.MoeError) as ei:
        cap.plan_dispatch(dev(np.zeros((10, 2), np.int32)), 8, 4, 2, dev(orc.place_uniform(8, 4)))
    assert ei.value.status == cap.MOE_ERR_ARG     # 4 does not divide 10 without src_rank
    before = cap.launch_count()
    with pytest.raises(cap.MoeError):
        cap.coact_stats(dev(np.zeros((1, 4, 9), np.int32)), 16)
    assert cap.launch_count() == before


@pytest.mark.parametrize("G", [8, 32, 64])
def test_sweep_placement_effect_full_size(cap, G):
    """Local share and V of the statistics sweep's batch (1M tokens) under the
    correlated placement of its calibration batch, layer 0, against the oracle."""
    from co_activation_placement_b200 import pipeline
    w = WORKLOADS["stats_sweep"]
    ids = make_routing(w, seed=w.seed)[:1]
    cal = make_routing(w, seed=w.seed + 1)[:1]
    got = pipeline.placement_effect(dev(ids), dev(cal), w.E, G, w.rpn, "correlated")
    e2r = orc.place_correlated(orc.coact(cal, w.E, want=("coact",))["coact"][0], G, w.rpn)
    want = orc.plan(ids[0], w.E, G, w.rpn, e2r)["summary"]
    assert got[0].tolist() == want.tolist()


@pytest.mark.parametrize("placement", ["capacity", "capped"])
@pytest.mark.parametrize("name", ["one_node", "ep32"])
def test_pipeline_capacity_placement(cap, name, placement):
    """The step under the capacity-aware placement (first-fit decreasing on the
    calibration loads) and under the correlated placement with a 10% load
    tolerance: placements and plans against the oracle."""
    from co_activation_placement_b200 import pipeline
    w = WORKLOADS[name]
    ids = make_routing(w)
    ids_cal = make_routing(w, seed=w.seed + 1)
    hp = pipeline.prepare(w.E, w.G, w.rpn, ids, make_gates(w), make_hidden(w), w.dtype, ids_cal,
                          placement=placement, shuffle=False, out_dtype=torch.float32)
    hp.step()
    torch.cuda.synchronize()
    assert int(host(hp.err)[0]) == 0
    oc = orc.coact(ids_cal, w.E, want=("coact",))["coact"]
    for l in range(w.L):
        e2r = orc.place_capacity(np.diag(oc[l]).astype(np.float64), w.G)[0] if placement == "capacity" \
            else orc.place_correlated_capped(oc[l], w.G, w.rpn, 0.1)
        assert (host(hp.e2r[l]) == e2r).all()
        op = orc.plan(ids[l], w.E, w.G, w.rpn, e2r)
        assert host(hp.plans[l].summary).tolist() == op["summary"].tolist()
        assert (host(hp.plans[l].row_of)[: w.T] == op["row_of"]).all()


@pytest.mark.parametrize("name", ["ep32", "large_ep64"])
def test_overlapped_step_equals_serial_step(cap, name):
    """The step with the control work on a second stream -- all of it ahead
    (overlap), or the forward-pass order with only the shuffle targets and
    statistics beside the rows (forward) -- and with each layer's permute and
    combine pipelined over token chunks produces every output bit for bit as
    the step run in line, also when replayed from a CUDA graph."""
    from co_activation_placement_b200 import pipeline
    w = WORKLOADS[name]
    ids = make_routing(w)
    ids_cal = make_routing(w, seed=w.seed + 1)
    gates, x = make_gates(w), make_hidden(w)
    outs = {}
    for overlap in ("inline", "overlap", "forward", "overlap/4", "forward/3"):
        sched, _, chunks = overlap.partition("/")
        hp = pipeline.prepare(w.E, w.G, w.rpn, ids, gates, x, w.dtype, ids_cal, out_dtype=torch.float32,
                              schedule=sched, row_chunks=int(chunks or 1))
        hp.step()
        g = hp.capture(2)
        g.replay()
        torch.cuda.synchronize()
        assert int(host(hp.err)[0]) == 0
        outs[overlap] = ([host(p.row_of).copy() for p in hp.plans] + [host(p.summary).copy() for p in hp.plans]
                         + [host(t).copy() for t in hp.targets] + [host(hp.stats["coact"]).copy()]
                         + [host(o).copy() for o in hp.outs])
        del g, hp
        torch.cuda.empty_cache()
    for sched in ("overlap", "forward", "overlap/4", "forward/3"):
        for a, b in zip(outs["inline"], outs[sched]):
            assert (a.view(np.uint8) == b.view(np.uint8)).all()
