"""One process per GPU: EPGroup (NCCL, symmetric memory) against the oracle.

Run under torchrun, or directly with RANK, WORLD_SIZE, LOCAL_RANK,
MASTER_ADDR and MASTER_PORT set.  Every rank takes its contiguous share of
one seeded batch, runs the statistics and one layer of dispatch, identity
experts and combine through EPGroup, and checks against the oracle's
one-device results over the whole batch: summed counts and transitions and
Ochiai bit for bit, its receive buffer equal to its segment of the
one-device send buffer, its combined rows within the combine's rounding
bound.  Prints one line "ep_group ok rank=<r>" and exits 0 on success."""
import datetime
import os
import sys

import numpy as np
import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle as orc                                   # noqa: E402
from synth import f32_to_bf16_bits, bf16_bits_to_f32  # noqa: E402

U24 = 2.0 ** -24


def main():
    rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=60), device_id=device)
    try:
        import co_activation_placement_b200 as cap
        from co_activation_placement_b200.ep import EPGroup
        cap.lib()
        E, k, G, rpn, d, L = 64, 6, 8 * world, 8, 256, 2
        T = 1024 * world
        rng = np.random.default_rng(5)
        hot = rng.permutation(E)[: k + 2]
        ids = np.stack([np.where((rng.random(T) < 0.6)[:, None],
                                 hot[np.argsort(rng.random((T, hot.size)), axis=1)[:, :k]],
                                 np.argsort(rng.random((T, E)), axis=1)[:, :k]) for _ in range(L)]).astype(np.int32)
        z = rng.standard_normal((T, k)).astype(np.float32)
        w = (np.exp(z) / np.exp(z).sum(1, keepdims=True)).astype(np.float32)
        xh = f32_to_bf16_bits(rng.standard_normal((T, d)).astype(np.float32))
        xf = bf16_bits_to_f32(xh)
        e2r = rng.permutation(np.arange(E, dtype=np.int32) // (E // G)).astype(np.int32)
        Tl = T // world
        part = slice(rank * Tl, (rank + 1) * Tl)
        o = orc.plan(ids[0], E, G, rpn, e2r)
        off = o["offsets"].astype(np.int64)
        Gl = G // world
        rows = [int(off[(h + 1) * Gl * G] - off[h * Gl * G]) for h in range(world)]

        def dev(a):
            return torch.from_numpy(np.ascontiguousarray(a)).to(device)

        grp = EPGroup(E, G, rpn, Tl, k, d, torch.bfloat16, device, max(rows))
        st = grp.stats(dev(ids[:, part]), E)
        whole = orc.coact(ids, E)
        torch.cuda.synchronize()
        assert (st["coact"].cpu().numpy() == whole["coact"]).all(), "summed counts"
        assert (st["trans"].cpu().numpy() == whole["trans"]).all(), "summed transitions"
        assert (st["ochiai"].cpu().numpy().view(np.uint32) == whole["ochiai"].view(np.uint32)).all(), "Ochiai"
        xd = dev(xh[part].view(np.int16)).view(torch.bfloat16)
        out = grp.step(dev(ids[0][part]), xd, dev(w[part]), dev(e2r))
        torch.cuda.synchronize()
        assert int(grp.shard.err.item()) == 0, "device error %d" % int(grp.shard.err.item())
        send = orc.permute(xh, o["row_token"])
        a = off[rank * Gl * G]
        got = grp.recv[: rows[rank]].view(torch.int16).cpu().numpy().view(np.uint16)
        assert (got == send[a:a + rows[rank]]).all(), "receive buffer"
        Yf = orc.permute(xf, o["row_token"])
        ref = orc.combine(Yf, o["row_of"], w, y_is_bf16=False)[part]
        idx = o["row_of"][part]
        mag = np.einsum("tj,tjc->tc", np.abs(w[part].astype(np.float64)), np.abs(Yf[idx].astype(np.float64)))
        assert (np.abs(out.cpu().numpy() - ref) <= (2 * k - 1) * U24 * mag * 1.0001 + 1e-30).all(), "combine"
        print("ep_group ok rank=%d" % rank, flush=True)
    finally:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
