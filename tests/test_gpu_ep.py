"""Parity of the expert-parallel path over several devices with the oracle.

The devices are emulated on one GPU (EPEmulation: W virtual devices, each
with buffers of its own, their phases run one after another).  Against the
oracle's one-device plan over all tokens (contiguous source ranks):
  - device h's receive buffer holds that plan's send rows
    [offsets[h*Gl*G], offsets[(h+1)*Gl*G]) bit for bit, and so do the
    dispatched gate records;
  - the route table equals the oracle's (orc.ep_routes on the device's
    oracle plan and the gathered counts);
  - the combined outputs lie within the combine's rounding bound of the
    oracle's fp64 combine, and equal the one-device CUDA combine bit for bit
    (same fp32 operations in the same order).
"""
import numpy as np
import pytest
import torch

import oracle as orc
from synth import f32_to_bf16_bits, bf16_bits_to_f32

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
    return ids, w, xf, xh, xd, scale, e2r


def combine_bound(Yf, idx, w, k):
    mag = np.einsum("tj,tjc->tc", np.abs(w.astype(np.float64)), np.abs(Yf[idx].astype(np.float64)))
    return (2 * k - 1) * U24 * mag * 1.0001 + 1e-30


def expected_routes(ids, E, G, rpn, e2r, W, o_global):
    """The oracle's route tables: per device, from its own oracle plan and the
    gathered counts (the one-device plan's counts)."""
    T = ids.shape[0]
    Gl, Tl = G // W, T // W
    out = []
    for h in range(W):
        src = (h * Gl + np.arange(Tl) // (Tl // Gl)).astype(np.int32)
        o = orc.plan(ids[h * Tl:(h + 1) * Tl], E, G, rpn, e2r, src_rank=src)
        out.append(orc.ep_routes(o_global["counts"], o["offsets"], G, W, h))
    return out


CASES = [  # T, E, k, G, rpn, W, d, bf16
    (512, 16, 2, 4, 2, 2, 64, False),
    (1536, 64, 6, 32, 8, 4, 128, True),
    (2048, 64, 8, 64, 8, 8, 256, True),
    (1024, 32, 4, 8, 8, 8, 64, False),       # one rank per device
    (1200, 32, 4, 8, 4, 1, 64, True),        # one device: the routes are the identity
    (1024, 64, 3, 64, 8, 64, 32, False),     # 64 devices of one rank, 16 tokens each
    (960, 24, 5, 12, 4, 3, 48, False),       # 16-byte vectors (rows of 192 bytes), ragged sizes
]


@pytest.mark.parametrize("T,E,k,G,rpn,W,d,bf16", CASES)
def test_ep_dispatch_combine(cap, T, E, k, G, rpn, W, d, bf16):
    from co_activation_placement_b200.ep import EPEmulation
    ids, w, xf, xh, xd, scale, e2r, = _setup(T + G + W, T, E, k, G, d, bf16)
    o = orc.plan(ids, E, G, rpn, e2r)
    R, off = o["R"], o["offsets"].astype(np.int64)
    Gl = G // W
    rows = [int(off[(h + 1) * Gl * G] - off[h * Gl * G]) for h in range(W)]
    recv_cap = max(rows) + 3
    dt = torch.bfloat16 if bf16 else torch.float32
    emu = EPEmulation(W, E, G, rpn, T, k, d, dt, "cuda", recv_cap)
    outs = emu.step(dev(ids), xd, dev(w), dev(e2r))
    assert emu.errors() == [0] * W
    send = orc.permute(xh, o["row_token"])
    for h in range(W):
        got = host(emu.recv[h].view(torch.int16) if bf16 else emu.recv[h])[: rows[h]]
        want = send[off[h * Gl * G]: off[h * Gl * G] + rows[h]]
        assert (got.view(want.dtype) == want).all(), "device %d's receive buffer" % h
    for h, r in enumerate(expected_routes(ids, E, G, rpn, e2r, W, o)):
        assert (host(emu.shards[h].route) == r).all(), "device %d's routes" % h
    # combine: within the bound of the fp64 oracle, and equal to the one-device kernel
    Yf = orc.permute(xf, o["row_token"])
    ref = orc.combine(Yf, o["row_of"], w, y_is_bf16=False)
    got = np.concatenate([host(t) for t in outs])
    assert (np.abs(got - ref) <= combine_bound(Yf, o["row_of"], w, k)).all()
    p = cap.plan_dispatch(dev(ids), E, G, rpn, dev(e2r))
    one = cap.permute(xd, p.row_of, p.R_max, err=p.err)
    out1 = cap.combine(one, p.row_of, dev(w), err=p.err)
    assert (host(out1).view(np.uint32) == got.view(np.uint32)).all()
    assert int(host(p.err)[0]) == 0


@pytest.mark.parametrize("T,E,k,G,rpn,W,d,bf16", [(1536, 64, 6, 32, 8, 4, 128, True),
                                                   (1024, 32, 4, 16, 4, 16, 64, False),
                                                   (600, 16, 2, 4, 2, 2, 7168, True)])
def test_ep_prereduce(cap, T, E, k, G, rpn, W, d, bf16):
    from co_activation_placement_b200.ep import EPEmulation
    ids, w, xf, xh, xd, scale, e2r = _setup(T + E + W, T, E, k, G, d, bf16)
    o = orc.plan(ids, E, G, rpn, e2r)
    off = o["offsets"].astype(np.int64)
    Gl = G // W
    rows = [int(off[(h + 1) * Gl * G] - off[h * Gl * G]) for h in range(W)]
    recv_cap = max(rows)
    dt = torch.bfloat16 if bf16 else torch.float32
    emu = EPEmulation(W, E, G, rpn, T, k, d, dt, "cuda", recv_cap, prereduce=True, scale=dev(scale))
    outs = emu.step(dev(ids), xd, dev(w), dev(e2r))
    assert emu.errors() == [0] * W
    se_o, sw_o = orc.dispatch_gates(ids, w, o["row_token"], o["row_jmask"])
    for h in range(W):
        a, n = off[h * Gl * G], rows[h]
        assert (host(emu.recv_e[h])[:n] == se_o[a:a + n]).all()
        assert (host(emu.recv_w[h])[:n].view(np.uint32) == sw_o[a:a + n].view(np.uint32)).all()
    # the one-device chain on the same inputs: the same bits
    p = cap.plan_dispatch(dev(ids), E, G, rpn, dev(e2r))
    send = cap.permute(xd, p.row_of, p.R_max, err=p.err)
    se, sw = cap.dispatch_gates(dev(ids), dev(w), p)
    y1 = cap.expert_reduce(send, p.summary, se, sw, dev(scale), y_dtype=dt, err=p.err)
    out1 = cap.combine_rows(y1, p.row_of, err=p.err)
    got = np.concatenate([host(t) for t in outs])
    assert (host(out1).view(np.uint32) == got.view(np.uint32)).all()
    # and the oracle: each token's distinct pre-reduced rows summed once
    yh = np.concatenate([host(emu.y[h].float())[: rows[h]] for h in range(W)])
    out_ref = orc.combine_rows(yh.astype(np.float32), o["row_of"])
    rows_mag = np.zeros_like(out_ref)
    for t in range(T):
        for r in set(o["row_of"][t].tolist()):
            rows_mag[t] += np.abs(yh[r])
    assert (np.abs(got - out_ref) <= k * U24 * rows_mag * 1.0001 + 1e-30).all()
    assert int(host(p.err)[0]) == 0


def test_ep_errors(cap):
    """A receive buffer too small, a misaligned and a null base: the stores
    that would leave a buffer are skipped and reported; nothing else moves."""
    from co_activation_placement_b200.ep import EPEmulation
    T, E, k, G, rpn, W, d = 512, 16, 2, 4, 2, 2, 64
    ids, w, xf, xh, xd, scale, e2r = _setup(7, T, E, k, G, d, False)
    o = orc.plan(ids, E, G, rpn, e2r)
    off = o["offsets"].astype(np.int64)
    rows = [int(off[(h + 1) * 2 * G] - off[h * 2 * G]) for h in range(W)]
    small = min(rows) // 2
    emu = EPEmulation(W, E, G, rpn, T, k, d, torch.float32, "cuda", small)
    big = [torch.full((max(rows) + 8, d), 7.0, device="cuda") for _ in range(W)]
    emu.recv = big
    emu.recv_base = torch.tensor([b.data_ptr() for b in big], dtype=torch.int64, device="cuda")
    emu.step(dev(ids), xd, dev(w), dev(e2r))
    assert set(emu.errors()) == {cap.DERR_ROW_RANGE}
    for b in big:
        assert (host(b)[small:] == 7.0).all()              # nothing stored past the capacity
    # misaligned and null bases: no store lands anywhere for those devices
    emu2 = EPEmulation(W, E, G, rpn, T, k, d, torch.float32, "cuda", max(rows))
    guard = torch.full((max(rows) + 8, d), 5.0, device="cuda")
    emu2.recv_base = torch.tensor([guard.data_ptr() + 16, 0], dtype=torch.int64, device="cuda")
    emu2.step(dev(ids), xd, dev(w), dev(e2r))
    assert set(emu2.errors()) == {cap.DERR_ROW_RANGE}
    assert (host(guard) == 5.0).all()


def test_ep_counts_mismatch(cap):
    """Gathered counts that disagree with a device's own plan are reported."""
    from co_activation_placement_b200.ep import EPShard
    T, E, k, G, rpn, d = 256, 16, 2, 4, 2, 32
    ids, w, xf, xh, xd, scale, e2r = _setup(9, T, E, k, G, d, False)
    s = EPShard(2, 0, E, G, rpn, T // 2, k, d, torch.float32, "cuda")
    s.plan_layer(dev(ids[: T // 2]), dev(e2r))
    s.counts_all.zero_()
    s.counts_all[:2].copy_(s.my_counts())
    s.counts_all[0, 1] += 1
    s.routes()
    assert int(host(s.err)[0]) == cap.DERR_ROW_RANGE


def test_ep_full_size_ep32(cap):
    """The EP32 workload (T = 65536, k = 6, G = 32 in 4 nodes, d = 4096 bf16)
    over 4 devices: every receive buffer equals the one-device send buffer's
    segment, and sampled combined rows match the oracle."""
    from co_activation_placement_b200.ep import EPEmulation
    from synth import WORKLOADS, make_routing, make_gates, make_hidden
    w = WORKLOADS["ep32"]
    ids = make_routing(w)[0]
    gates = make_gates(w)[0]
    x = make_hidden(w)
    xd = dev(x.view(np.int16)).view(torch.bfloat16)
    e2r = orc.place_uniform(w.E, w.G)
    W = 4
    Gl = w.G // W
    p = cap.plan_dispatch(dev(ids), w.E, w.G, w.rpn, dev(e2r))
    send = cap.permute(xd, p.row_of, p.R_max, err=p.err)
    out1 = cap.combine(send, p.row_of, dev(gates), err=p.err)
    off = host(p.offsets).astype(np.int64)
    rows = [int(off[(h + 1) * Gl * w.G] - off[h * Gl * w.G]) for h in range(W)]
    emu = EPEmulation(W, w.E, w.G, w.rpn, w.T, w.k, w.d, torch.bfloat16, "cuda", max(rows))
    outs = emu.step(dev(ids), xd, dev(gates), dev(e2r))
    assert emu.errors() == [0] * W
    for h in range(W):
        a = int(off[h * Gl * w.G])
        assert torch.equal(emu.recv[h][: rows[h]].view(torch.int16), send[a:a + rows[h]].view(torch.int16))
    got = torch.cat(outs)
    assert torch.equal(got.view(torch.int32), out1.view(torch.int32))
    o = orc.plan(ids, w.E, w.G, w.rpn, e2r)
    rng = np.random.default_rng(3)
    toks = np.unique(np.concatenate([rng.integers(0, w.T, 512), [0, w.T - 1]]))
    xf = bf16_bits_to_f32(x)
    sub = o["row_of"][toks]
    uniq, inv = np.unique(sub, return_inverse=True)
    Ysub = xf[o["row_token"][uniq]]
    ref = orc.combine(Ysub, inv.reshape(sub.shape).astype(np.int32), gates[toks], y_is_bf16=False)
    g = host(got[torch.from_numpy(toks).cuda()])
    assert (np.abs(g - ref) <= combine_bound(Ysub, inv.reshape(sub.shape), gates[toks], w.k)).all()
    assert int(host(p.err)[0]) == 0


def test_ep_group_one_process(cap):
    """EPGroup end to end in one NCCL process (W = 1: all ranks on this GPU):
    symmetric-memory buffers, the counts all-gather, the statistics
    all-reduce and the meetings, checked against the oracle by the script."""
    import os
    import socket
    import subprocess
    import sys
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0", MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
               NCCL_NVLS_ENABLE="0", TORCH_SYMM_MEM_DISABLE_MULTICAST="1")
    r = subprocess.run([sys.executable, os.path.join(root, "tests", "ep_group_run.py")], env=env, cwd=root,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "ep_group ok rank=0" in r.stdout


@pytest.mark.parametrize("seed", range(16))
def test_ep_fuzz(cap, seed):
    """Seeded random shapes: G in 1..64, W any divisor of G, tokens a ragged
    multiple of G, k 1..8, f32 or bf16 rows of 16..544 bytes, uniform or
    permuted placement, with and without pre-reduction."""
    from co_activation_placement_b200.ep import EPEmulation
    rng = np.random.default_rng(5000 + seed)
    G = int(rng.choice([1, 2, 3, 4, 6, 8, 12, 16, 32, 64]))
    W = int(rng.choice([w_ for w_ in range(1, G + 1) if G % w_ == 0]))
    rpn = int(rng.choice([r for r in range(1, G + 1) if G % r == 0]))
    E = G * int(rng.integers(1, max(2, 256 // G) + 1))
    k = int(rng.integers(1, min(8, E) + 1))
    T = G * int(rng.integers(1, max(2, 3000 // G)))
    bf16 = bool(rng.integers(0, 2))
    d = int(rng.choice([8, 16, 40, 64, 136]))
    if (d * (2 if bf16 else 4)) % 16:
        d += 8 - d % 8
    prereduce = bool(rng.integers(0, 2))
    ids, w, xf, xh, xd, scale, e2r = _setup(6000 + seed, T, E, k, G, d, bf16)
    if rng.integers(0, 2):
        e2r = orc.place_uniform(E, G)
    o = orc.plan(ids, E, G, rpn, e2r)
    off = o["offsets"].astype(np.int64)
    Gl = G // W
    rows = [int(off[(h + 1) * Gl * G] - off[h * Gl * G]) for h in range(W)]
    dt = torch.bfloat16 if bf16 else torch.float32
    emu = EPEmulation(W, E, G, rpn, T, k, d, dt, "cuda", max(max(rows), 1), prereduce=prereduce, scale=dev(scale))
    outs = emu.step(dev(ids), xd, dev(w), dev(e2r))
    assert emu.errors() == [0] * W, (G, W, rpn, E, k, T, d, bf16, prereduce)
    send = orc.permute(xh, o["row_token"])
    for h in range(W):
        got = host(emu.recv[h].view(torch.int16) if bf16 else emu.recv[h])[: rows[h]]
        assert (got.view(send.dtype) == send[off[h * Gl * G]: off[h * Gl * G] + rows[h]]).all()
    p = cap.plan_dispatch(dev(ids), E, G, rpn, dev(e2r))
    one = cap.permute(xd, p.row_of, p.R_max, err=p.err)
    if prereduce:
        se, sw = cap.dispatch_gates(dev(ids), dev(w), p)
        y1 = cap.expert_reduce(one, p.summary, se, sw, dev(scale), y_dtype=dt, err=p.err)
        out1 = cap.combine_rows(y1, p.row_of, err=p.err)
    else:
        out1 = cap.combine(one, p.row_of, dev(w), err=p.err)
    got = np.concatenate([host(t) for t in outs])
    assert (host(out1).view(np.uint32) == got.view(np.uint32)).all()
    if not prereduce:
        Yf = orc.permute(xf, o["row_token"])
        ref = orc.combine(Yf, o["row_of"], w, y_is_bf16=False)
        assert (np.abs(got - ref) <= combine_bound(Yf, o["row_of"], w, k)).all()
    assert int(host(p.err)[0]) == 0
