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


@pytest.mark.parametrize("T,E,k,G,rpn,W", [(512, 16, 2, 4, 2, 2), (1536, 64, 6, 32, 8, 4), (960, 24, 5, 12, 4, 3),
                                            (1024, 64, 3, 64, 8, 64), (640, 32, 4, 8, 8, 1)])
def test_route_definition(T, E, k, G, rpn, W):
    ids = _ids(T + W, T, E, k)
    e2r = np.random.default_rng(G).permutation(np.arange(E, dtype=np.int32) // (E // G)).astype(np.int32)
    o = orc.plan(ids, E, G, rpn, e2r)
    off_g = o["offsets"].astype(np.int64)
    Gl, Tl = G // W, T // W
    seen = np.zeros(o["R"], bool)
    for h in range(W):
        lo = _local_plan(ids, E, G, rpn, e2r, W, h)
        off_l = lo["offsets"].astype(np.int64)
        for x in range(lo["R"]):
            seg = int(np.searchsorted(off_l, x, side="right")) - 1     # (r, s) = divmod(seg, G)
            r, s = divmod(seg, G)
            assert h * Gl <= s < (h + 1) * Gl                            # only this device's sources
            q = x + off_g[r * G + s] - off_g[(r // Gl) * Gl * G] - off_l[seg]
            g = off_g[(r // Gl) * Gl * G] + q                            # the one-device row
            assert off_g[r * G + s] <= g < off_g[r * G + s + 1]
            assert o["row_token"][g] == h * Tl + lo["row_token"][x]
            assert not seen[g]
            seen[g] = True
        rows_h = off_g[(h + 1) * Gl * G] - off_g[h * Gl * G]
        assert rows_h == sum(int(c) for c in o["counts"][:, h * Gl:(h + 1) * Gl].ravel())
    assert seen.all()                                                    # every row arrives exactly once


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
