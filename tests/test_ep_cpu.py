"""Host side of expert parallelism over several devices, on CPU.

- The route definition: with every device planning its own tokens, local row
  x of segment (r, s) moved by the segment's shift lands, in device r/Gl's
  buffer, on the one-device plan's row for the same token and rank.
- The collectives of co_activation_placement_b200.ep with gloo ranks: the
  counts all-gather rebuilds the one-device plan's counts, the all-reduce of
  per-device statistics gives the statistics of the whole batch (and Ochiai
  on the sums equals Ochiai on the whole batch's counts), and the meeting
  all-reduce returns.
The oracle computes each device's part here (test code); on a GPU the same
collectives carry the CUDA kernels' outputs.
"""
import datetime
import os
import socket

import numpy as np
import pytest

import oracle as orc


def _ids(seed, T, E, k):
    rng = np.random.default_rng(seed)
    hot = rng.permutation(E)[: k + 2]
    return np.where((rng.random(T) < 0.6)[:, None],
                    hot[np.argsort(rng.random((T, hot.size)), axis=1)[:, :k]],
                    np.argsort(rng.random((T, E)), axis=1)[:, :k]).astype(np.int32)


def _local_plan(ids, E, G, rpn, e2r, W, h):
    T = ids.shape[0]
    Gl, Tl = G // W, T // W
    src = (h * Gl + np.arange(Tl) // (Tl // Gl)).astype(np.int32)
    return orc.plan(ids[h * Tl:(h + 1) * Tl], E, G, rpn, e2r, src_rank=src)


def test_routes_hand_worked():
    """G = 2 ranks on W = 2 devices.  Source rank 0 sends 3 rows to rank 0 and
    1 to rank 1; source rank 1 sends 2 and 4.  One-device order (r, s): rank
    0's buffer is rows 0-2 from s 0 then 3-4 from s 1 (5 rows); rank 1's is
    row 0 from s 0 then rows 1-4 from s 1.  Device 0's own plan has local
    rows 0-2 for rank 0 and row 3 for rank 1: rows 0-2 stay in place, row 3
    becomes row 0 of device 1."""
    counts_all = np.array([[3, 1], [2, 4]], np.int32)
    local0 = np.array([0, 3, 3, 4, 4], np.int32)           # offsets (r, s): (0,0) (0,1) (1,0) (1,1), R
    assert orc.ep_routes(counts_all, local0, 2, 2, 0).tolist() == [5, 0, 3, 4, 0, -3]
    local1 = np.array([0, 0, 2, 2, 6], np.int32)           # device 1 plans source rank 1 only
    # segments (r=0, s=1) at local row 0 -> device 0 row 3; (r=1, s=1) at local row 2 -> device 1 row 1
    assert orc.ep_routes(counts_all, local1, 2, 2, 1).tolist() == [5, 0, 2, 6, 3, -1]


@pytest.mark.parametrize("T,E,k,G,rpn,W", [(512, 16, 2, 4, 2, 2), (1536, 64, 6, 32, 8, 4), (960, 24, 5, 12, 4, 3),
                                            (1024, 64, 3, 64, 8, 64), (640, 32, 4, 8, 8, 1)])
def test_route_definition(T, E, k, G, rpn, W):
    """The oracle's route tables move every local row of every device onto the
    one-device plan's row for the same token and rank, each row once."""
    ids = _ids(T + W, T, E, k)
    e2r = np.random.default_rng(G).permutation(np.arange(E, dtype=np.int32) // (E // G)).astype(np.int32)
    o = orc.plan(ids, E, G, rpn, e2r)
    off_g = o["offsets"].astype(np.int64)
    Gl, Tl = G // W, T // W
    P = G * Gl
    plans = [_local_plan(ids, E, G, rpn, e2r, W, h) for h in range(W)]
    counts_all = np.concatenate([plans[h]["counts"][h * Gl:(h + 1) * Gl] for h in range(W)])
    assert (counts_all == o["counts"]).all()
    seen = np.zeros(o["R"], bool)
    for h, lo in enumerate(plans):
        route = orc.ep_routes(counts_all, lo["offsets"], G, W, h)
        assert route[0] == off_g[(h + 1) * Gl * G] - off_g[h * Gl * G]
        assert route[1 + P] == lo["R"]
        start = route[1:P + 2]
        for x in range(lo["R"]):
            i = int(np.searchsorted(start, x, side="right")) - 1      # the segment holding local row x
            r, s = i // Gl, h * Gl + i % Gl
            q = x + route[P + 2 + i]                                    # its row in device r/Gl's buffer
            g = off_g[(r // Gl) * Gl * G] + q                           # the one-device row
            assert 0 <= q and off_g[r * G + s] <= g < off_g[r * G + s + 1]
            assert o["row_token"][g] == h * Tl + lo["row_token"][x]
            assert (o["row_jmask"][g] == lo["row_jmask"][x])
            assert not seen[g]
            seen[g] = True
        if W == 1:
            assert (route[P + 2:] == 0).all()                          # one device: the routes are the identity
    assert seen.all()                                                   # every row arrives exactly once


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from co_activation_placement_b200 import ep
        T, E, k, G, rpn, L = 1536, 32, 4, 8 * world, 8, 3
        rng = np.random.default_rng(11)
        ids = np.stack([_ids(100 + l, T, E, k) for l in range(L)])
        e2r = rng.permutation(np.arange(E, dtype=np.int32) % G).astype(np.int32)
        Tl = T // world
        # statistics: each rank counts its own tokens, the sums are the batch's
        mine = orc.coact(ids[:, rank * Tl:(rank + 1) * Tl], E)
        c = torch.from_numpy(mine["coact"].astype(np.uint32).copy())
        tr = torch.from_numpy(mine["trans"].astype(np.uint32).copy())
        ep.allreduce_counts(c, tr)
        whole = orc.coact(ids, E)
        ok_stats = bool((c.numpy() == whole["coact"]).all() and (tr.numpy() == whole["trans"]).all())
        _, och = orc.coact_ema(c.numpy(), 1.0)
        ok_och = bool((och.view(np.uint32) == whole["ochiai"].view(np.uint32)).all())
        # counts: the gathered slabs are the one-device plan's counts
        lo = _local_plan(ids[0], E, G, rpn, e2r, world, rank)
        Gl = G // world
        slab = torch.from_numpy(lo["counts"][rank * Gl:(rank + 1) * Gl].copy())
        counts_all = torch.zeros((G, G), dtype=torch.int32)
        ep.gather_counts(counts_all, slab)
        ok_counts = bool((counts_all.numpy() == orc.plan(ids[0], E, G, rpn, e2r)["counts"]).all())
        flag = torch.zeros(1, dtype=torch.int32)
        ep.meet(flag)
        q.put((rank, ok_stats, ok_och, ok_counts))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_ep_collectives_gloo(world):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == list(range(world))
    assert all(r[1] for r in res), "summed statistics differ from the whole batch's"
    assert all(r[2] for r in res), "Ochiai on the summed counts differs"
    assert all(r[3] for r in res), "gathered counts differ from the one-device plan's"


def _lost_rank_worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    from co_activation_placement_b200 import ep
    flag = torch.zeros(1, dtype=torch.int32)
    ep.meet(flag)                                   # everyone present once
    if rank == world - 1:
        q.put((rank, "left"))                       # this rank stops taking part: it never meets again
        q.close()
        q.join_thread()                             # the message is out before the process ends
        os._exit(0)
    try:
        ep.meet(flag)
        q.put((rank, "met"))
    except Exception as ex:                          # the others learn of it from the meeting itself
        q.put((rank, "error: " + type(ex).__name__))


@pytest.mark.parametrize("world", [2, 3])
def test_meet_reports_a_lost_rank(world):
    """A rank that stops taking part between steps (host-side failure, no GPU
    involved): the other ranks' next meeting ends with an error instead of
    waiting for ever (the process group's timeout or the closed connection)."""
    import time
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_lost_rank_worker, args=(r, world, port, q)) for r in range(world)]
    t0 = time.time()
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
    assert res[world - 1] == "left"
    assert all(res[r].startswith("error") for r in range(world - 1)), res
    assert time.time() - t0 < 100


@pytest.mark.parametrize("T,E,k,G,rpn,W", [(512, 16, 2, 4, 2, 2), (1536, 64, 6, 32, 8, 4), (960, 24, 5, 12, 4, 3),
                                            (1024, 64, 3, 64, 8, 64), (640, 32, 4, 8, 8, 1)])
def test_exchange_rows_from_route_tables(T, E, k, G, rpn, W):
    """Rows crossing devices, counted from the route tables: device h's local
    segments (r, s) with r on another device are the rows it sends; of the
    rows its buffer receives (route[0]), those not from its own segments
    came from other devices.  The oracle's definition and the library's host
    count agree with both."""
    import co_activation_placement_b200 as cap
    ids = _ids(T + 7 * W, T, E, k)
    e2r = np.random.default_rng(G + 1).permutation(np.arange(E, dtype=np.int32) // (E // G)).astype(np.int32)
    Gl = G // W
    P = G * Gl
    plans = [_local_plan(ids, E, G, rpn, e2r, W, h) for h in range(W)]
    counts_all = np.concatenate([plans[h]["counts"][h * Gl:(h + 1) * Gl] for h in range(W)])
    sent_o, recv_o = orc.ep_exchange_rows(counts_all, G, W)
    sent_l, recv_l = cap.ep_exchange_rows(counts_all, G, W)
    assert sent_l.tolist() == sent_o.tolist() and recv_l.tolist() == recv_o.tolist()
    for h, lo in enumerate(plans):
        route = orc.ep_routes(counts_all, lo["offsets"], G, W, h)
        start = route[1:P + 2]
        seg = np.diff(start)                                  # rows of each local segment
        away = np.array([(i // Gl) // Gl != h for i in range(P)])
        assert int(seg[away].sum()) == sent_o[h]
        assert int(route[0]) - int(seg[~away].sum()) == recv_o[h]
    assert sent_o.sum() == recv_o.sum()
    if W == 1:
        assert sent_o.tolist() == [0]
