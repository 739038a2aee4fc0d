"""Parity of the receiver-side pre-reduced combine (gate dispatch, stand-in
expert reduce at the receiving rank, unit-weight row combine at the source)
with the oracle.

Bounds from the arithmetic (u = 2^-24): the reduce rounds g_j = w_j * s_j
once and accumulates k terms with FMAs, so |y - exact| <= (k + 2) u sum_j
|w_j s_j x|; the row combine adds at most k rows, |out - exact| <=
k u sum_r |y_r|; bf16 outputs add half a bf16 ulp (2^-8 relative)."""
import numpy as np
import pytest
import torch

import oracle as orc
from synth import WORKLOADS, make_routing, make_gates, make_hidden, make_expert_scales, bf16_bits_to_f32, f32_to_bf16_bits

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


def _setup(seed, T, E, k, G, d, bf16):
    rng = np.random.default_rng(seed)
    hot = rng.permutation(E)[: k + 2]
    ids = np.where((rng.random(T) < 0.6)[:, None],
                   hot[np.argsort(rng.random((T, hot.size)), axis=1)[:, :k]],
                   np.argsort(rng.random((T, E)), axis=1)[:, :k]).astype(np.int32)
    z = rng.standard_normal((T, k)).astype(np.float32)
    w = (np.exp(z) / np.exp(z).sum(1, keepdims=True)).astype(np.float32)
    xf = rng.standard_normal((T, d)).astype(np.float32)
    if bf16:
        xh = f32_to_bf16_bits(xf)
        xd = dev(xh.view(np.int16)).view(torch.bfloat16)
        xf = bf16_bits_to_f32(xh)
    else:
        xh, xd = xf, dev(xf)
    scale = rng.uniform(-2.0, 2.0, E).astype(np.float32)
    e2r = rng.permutation(np.arange(E, dtype=np.int32) // (E // G)).astype(np.int32)
    src = rng.integers(0, G, T).astype(np.int32)
    return ids, w, xf, xh, xd, scale, e2r, src


@pytest.mark.parametrize("T,E,k,G,d,bf16", [(1111, 32, 2, 8, 128, False), (3000, 64, 6, 32, 256, True),
                                            (777, 256, 8, 64, 7168, True), (500, 16, 1, 4, 64, False)])
@pytest.mark.parametrize("y_bf16", [False, True])
def test_prereduce_chain(cap, T, E, k, G, d, bf16, y_bf16):
    ids, w, xf, xh, xd, scale, e2r, src = _setup(T + E + d, T, E, k, G, d, bf16)
    p = cap.plan_dispatch(dev(ids), E, G, 4 if G % 4 == 0 else 1, dev(e2r), src_rank=dev(src))
    o = orc.plan(ids, E, G, 4 if G % 4 == 0 else 1, e2r, src_rank=src)
    R = o["R"]
    send = cap.permute(xd, p.row_of, p.R_max, err=p.err)
    se, sw = cap.dispatch_gates(dev(ids), dev(w), p)
    se_o, sw_o = orc.dispatch_gates(ids, w, o["row_token"], o["row_jmask"])
    assert (host(se)[:R] == se_o).all() and (host(sw)[:R].view(np.uint32) == sw_o.view(np.uint32)).all()
    y = cap.expert_reduce(send, p.summary, se, sw, dev(scale), y_dtype=torch.bfloat16 if y_bf16 else torch.float32,
                          err=p.err)
    yh = host(y.float())[:R]
    send_f = orc.permute(xf, o["row_token"])
    y_ref = orc.expert_reduce(send_f, se_o, sw_o, scale, y_is_bf16=False)
    mag = np.abs(send_f.astype(np.float64)) * (np.abs(sw_o.astype(np.float64)) *
                                               np.abs(np.where(se_o >= 0, scale[np.maximum(se_o, 0)], 0))).sum(1)[:, None]
    bound = (k + 2) * U24 * mag * 1.0001 + 1e-30
    if y_bf16:
        bound = bound + 2.0 ** -8 * (np.abs(y_ref) + bound)
    assert (np.abs(yh - y_ref) <= bound).all()
    out = cap.combine_rows(y, p.row_of, out_dtype=torch.float32, err=p.err)
    out_ref = orc.combine_rows(yh.astype(np.float32), o["row_of"])
    rows_mag = np.zeros_like(out_ref)
    for t in range(T):
        for r in set(o["row_of"][t].tolist()):
            rows_mag[t] += np.abs(yh[r])
    assert (np.abs(host(out) - out_ref) <= k * U24 * rows_mag * 1.0001 + 1e-30).all()
    # the chain's closed form: every pick once, out[t] = x_t * sum_j w_tj * scale[e_tj]
    g = (w.astype(np.float64) * scale.astype(np.float64)[ids]).sum(1)
    closed = xf.astype(np.float64) * g[:, None]
    tot_mag = np.abs(xf.astype(np.float64)) * (np.abs(w.astype(np.float64)) * np.abs(scale[ids])).sum(1)[:, None]
    tol = (2 * k + 2) * U24 * tot_mag * 1.001 + (2.0 ** -8 * 2 * tot_mag if y_bf16 else 0) + 1e-30
    assert (np.abs(host(out) - closed) <= tol).all()
    assert int(host(p.err)[0]) == 0


def test_prereduce_errors(cap):
    T, E, k, G = 64, 8, 2, 4
    ids, w, xf, xh, xd, scale, e2r, src = _setup(3, T, E, k, G, 32, False)
    p = cap.plan_dispatch(dev(ids), E, G, 2, dev(e2r))
    send = cap.permute(xd, p.row_of, p.R_max)
    se, sw = cap.dispatch_gates(dev(ids), dev(w), p)
    bad = se.clone()
    bad[0, 0] = E
    err = cap.new_err("cuda")
    cap.expert_reduce(send, p.summary, bad, sw, dev(scale), err=err)
    assert int(host(err)[0]) == cap.DERR_ID_RANGE
    err = cap.new_err("cuda")
    ro = p.row_of.clone()
    ro[1, 0] = p.R_max + 5
    cap.combine_rows(send, ro, err=err)
    assert int(host(err)[0]) == cap.DERR_ROW_RANGE
    assert int(host(p.err)[0]) == 0


@pytest.mark.parametrize("name", ["one_node", "large_ep64"])
def test_prereduce_pipeline_full_size(cap, name):
    from co_activation_placement_b200 import pipeline
    w = WORKLOADS[name]
    ids = make_routing(w)
    cal = make_routing(w, seed=1)
    gates = make_gates(w)
    x = make_hidden(w)
    hp = pipeline.prepare(w.E, w.G, w.rpn, ids, gates, x, w.dtype, cal, placement="correlated", shuffle=True,
                          out_dtype=torch.float32, scales=make_expert_scales(w))
    hp.step()
    torch.cuda.synchronize()
    assert int(host(hp.err)[0]) == 0
    scales = [host(s) for s in hp.scales]
    xf = bf16_bits_to_f32(x) if w.dtype == "bf16" else x
    rng = np.random.default_rng(1)
    for l in range(w.L):
        toks = np.unique(np.concatenate([rng.integers(0, w.T, 2048), [0, w.T - 1]]))
        g = (gates[l][toks].astype(np.float64) * scales[l].astype(np.float64)[ids[l][toks]]).sum(1)
        closed = xf[toks].astype(np.float64) * g[:, None]
        mag = np.abs(xf[toks].astype(np.float64)) * (np.abs(gates[l][toks].astype(np.float64)) *
                                                     np.abs(scales[l][ids[l][toks]])).sum(1)[:, None]
        got = host(hp.outs[l][torch.from_numpy(toks).cuda()])
        # y is kept in the hidden states' dtype (bf16): half a bf16 ulp per row, plus fp32 roundings
        tol = (2 * w.k + 2) * U24 * mag * 1.001 + 2.0 ** -8 * mag + 1e-30
        assert (np.abs(got - closed) <= tol).all()
