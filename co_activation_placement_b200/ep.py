"""Expert parallelism over several devices, one process per GPU.

"Expert Coupling in MoE Pretraining", abstract: each token is sent to each
GPU once and the results are combined; "Training Communication-Efficient MoE
...", footnote 3: hidden states and routed probabilities are dispatched, the
combine is the inverse exchange.

The G expert-parallel ranks are spread over W devices, G/W consecutive ranks
per device.  Per layer each device
  1. plans its own tokens (moe_plan_dispatch, its ranks as the sources),
  2. shares its rows of the counts (all-gather of a [G/W][G] int32 slab),
  3. turns the gathered counts into route tables (moe_ep_routes),
  4. stores its rows straight into the receiving devices' buffers
     (moe_ep_permute through peer pointers) and, for the pre-reduced
     combine, the gates of every row (moe_ep_scatter_rows),
  5. meets the others (a one-element all-reduce on the same stream),
  6. runs its experts on the rows it received (identity, or the stand-in
     experts of moe_expert_reduce, then meets the others again),
  7. combines its tokens from the devices that hold their rows
     (moe_ep_combine) and meets the others once more, so that no device
     overwrites a buffer another is still reading.
The receive buffers hold, device by device, exactly the rows of the
one-device send buffer over all tokens, and the combined outputs equal the
one-device combine bit for bit.

The statistics shard the same way: each device counts its own tokens, the
counts are summed with one all-reduce, and Ochiai follows from the sums
(moe_coact_ema with alpha 1 computes it from the summed counts exactly as
moe_coact_stats does from its own).

EPGroup is the multi-process form: torch.distributed (NCCL) for the counts,
the statistics and the meetings; torch's symmetric memory for buffers that
every device of the group can address.  EPEmulation runs the same phases for
W virtual devices on one GPU, each with buffers and a CUDA stream of its own:
within a phase the devices' launches run side by side, as separate GPUs
would, and each meeting is a join of the W streams.
"""
from __future__ import annotations

from typing import List, Optional

import torch

import co_activation_placement_b200 as cap


class EPShard:
    """One device's part: its plan, route table, outputs and gate records."""

    def __init__(self, W: int, me: int, E: int, G: int, rpn: int, T_local: int, k: int, d: int,
                 dtype, device, out_dtype=torch.float32, prereduce: bool = False):
        if G % W:
            raise ValueError("the devices must split the G ranks evenly")
        Gl = G // W
        if T_local < Gl or T_local % Gl:
            raise ValueError("a device's tokens must split evenly over its G/W ranks")
        self.W, self.me, self.E, self.G, self.rpn, self.T, self.k, self.d = W, me, E, G, rpn, T_local, k, d
        self.Gl = Gl
        self.dtype = dtype
        dev = torch.device(device)
        self.device = dev
        per = T_local // Gl
        self.src_rank = (me * Gl + torch.arange(T_local, device=dev, dtype=torch.int32) // per).to(torch.int32)
        self.plan = cap.Plan.empty(T_local, k, G, dev)
        self.err = self.plan.err
        self.ws = torch.empty(max(cap.plan_dispatch_workspace(T_local, k, G, True), 1), dtype=torch.uint8, device=dev)
        self.counts_all = torch.zeros((G, G), dtype=torch.int32, device=dev)
        self.route = torch.empty(cap.ep_route_len(G, W), dtype=torch.int64, device=dev)
        self.out = torch.empty((T_local, d), dtype=out_dtype, device=dev)
        self.prereduce = prereduce
        if prereduce:
            R_max = self.plan.R_max
            self.send_e = torch.empty((R_max, k), dtype=torch.int32, device=dev)
            self.send_w = torch.empty((R_max, k), dtype=torch.float32, device=dev)

    def my_counts(self) -> torch.Tensor:
        """This device's rows of the counts, [G/W][G] (a view of the plan's counts)."""
        return self.plan.counts[self.me * self.Gl:(self.me + 1) * self.Gl]

    def plan_layer(self, ids: torch.Tensor, expert_to_rank: torch.Tensor):
        cap.plan_dispatch(ids, self.E, self.G, self.rpn, expert_to_rank, src_rank=self.src_rank,
                          plan=self.plan, ws=self.ws)

    def routes(self):
        cap.ep_routes(self.counts_all, self.plan.offsets, self.G, self.W, self.me, route=self.route, err=self.err)

    def dispatch(self, x: torch.Tensor, recv_base: torch.Tensor, recv_cap: int):
        cap.ep_permute(x, self.plan.row_of, self.plan.R_max, self.route, self.G, self.W, recv_base, recv_cap,
                       err=self.err)

    def dispatch_gates(self, ids: torch.Tensor, gates: torch.Tensor, e_base: torch.Tensor, w_base: torch.Tensor,
                       recv_cap: int):
        cap.dispatch_gates(ids, gates, self.plan, send_e=self.send_e, send_w=self.send_w, err=self.err)
        cap.ep_scatter_rows(self.send_e, self.route, self.G, self.W, e_base, recv_cap, err=self.err)
        cap.ep_scatter_rows(self.send_w, self.route, self.G, self.W, w_base, recv_cap, err=self.err)

    def experts(self, recv: torch.Tensor, recv_e: torch.Tensor, recv_w: torch.Tensor, scale: torch.Tensor,
                y: torch.Tensor):
        """Stand-in experts on the rows this device received (route[0] of them)."""
        cap.expert_reduce(recv, self.route, recv_e, recv_w, scale, y=y, err=self.err)

    def combine(self, y_base: torch.Tensor, y_dtype, y_cap: int, gates: Optional[torch.Tensor]) -> torch.Tensor:
        return cap.ep_combine(y_base, y_dtype, y_cap, self.d, self.route, self.G, self.W, self.plan.R_max,
                              self.plan.row_of, None if self.prereduce else gates, self.out, err=self.err)


def _bases(ts: List[torch.Tensor], device) -> torch.Tensor:
    return torch.tensor([t.data_ptr() for t in ts], dtype=torch.int64, device=device)


class EPEmulation:
    """W virtual devices on one GPU: the phases of EPGroup for every device in
    turn, each device with receive buffers of its own."""

    def __init__(self, W: int, E: int, G: int, rpn: int, T: int, k: int, d: int, dtype, device, recv_cap: int,
                 out_dtype=torch.float32, prereduce: bool = False, scale: Optional[torch.Tensor] = None):
        if T % W:
            raise ValueError("the devices must split the tokens evenly")
        self.W, self.T, self.Tl, self.d, self.k = W, T, T // W, d, k
        self.recv_cap = recv_cap
        self.dtype = dtype
        self.shards = [EPShard(W, h, E, G, rpn, T // W, k, d, dtype, device, out_dtype, prereduce) for h in range(W)]
        counts_all = self.shards[0].counts_all
        for s in self.shards:
            s.counts_all = counts_all
        self.streams = None
        self.recv = [torch.empty((recv_cap, d), dtype=dtype, device=device) for _ in range(W)]
        self.recv_base = _bases(self.recv, device)
        self.prereduce = prereduce
        if prereduce:
            if scale is None:
                raise ValueError("the pre-reduced combine needs the experts' scales")
            self.scale = scale
            self.recv_e = [torch.empty((recv_cap, k), dtype=torch.int32, device=device) for _ in range(W)]
            self.recv_w = [torch.empty((recv_cap, k), dtype=torch.float32, device=device) for _ in range(W)]
            self.y = [torch.empty((recv_cap, d), dtype=dtype, device=device) for _ in range(W)]
            self.e_base, self.w_base = _bases(self.recv_e, device), _bases(self.recv_w, device)
            self.y_base = _bases(self.y, device)

    def _part(self, a: torch.Tensor, h: int) -> torch.Tensor:
        return a[h * self.Tl:(h + 1) * self.Tl]

    def _phase(self, fn):
        """fn(shard) for every device on the device's own stream, all of them
        after the work enqueued so far on the current stream and before any
        work enqueued on it afterwards (a meeting of the W devices)."""
        main = torch.cuda.current_stream()
        if self.streams is None:
            self.streams = [torch.cuda.Stream(device=main.device) for _ in range(self.W)]
        start = torch.cuda.Event()
        start.record(main)
        for s, st in zip(self.shards, self.streams):
            st.wait_event(start)
            with torch.cuda.stream(st):
                fn(s)
            done = torch.cuda.Event()
            done.record(st)
            main.wait_event(done)

    def step(self, ids: torch.Tensor, x: torch.Tensor, gates: torch.Tensor, expert_to_rank: torch.Tensor):
        """One layer for all T tokens (device h owns tokens [h*T/W, (h+1)*T/W)); returns the W outputs."""
        sh = self.shards
        self._phase(lambda s: s.plan_layer(self._part(ids, s.me), expert_to_rank))
        sh[0].counts_all.copy_(torch.cat([s.my_counts() for s in sh]))

        def send(s):
            s.routes()
            s.dispatch(self._part(x, s.me), self.recv_base, self.recv_cap)
            if self.prereduce:
                s.dispatch_gates(self._part(ids, s.me), self._part(gates, s.me), self.e_base, self.w_base,
                                 self.recv_cap)
        self._phase(send)
        if self.prereduce:
            self._phase(lambda s: s.experts(self.recv[s.me], self.recv_e[s.me], self.recv_w[s.me], self.scale,
                                            self.y[s.me]))
            y_base = self.y_base
        else:
            y_base = self.recv_base
        self._phase(lambda s: s.combine(y_base, self.dtype, self.recv_cap, self._part(gates, s.me)))
        return [s.out for s in sh]

    def errors(self) -> List[int]:
        torch.cuda.synchronize()
        return [int(s.err.item()) for s in self.shards]


# ---------------------------------------------------------------- collectives (any torch.distributed backend)

def gather_counts(counts_all: torch.Tensor, mine: torch.Tensor, group=None):
    """counts_all [G][G] <- every device's [G/W][G] slab, in device order."""
    import torch.distributed as dist
    W = dist.get_world_size(group)
    dist.all_gather(list(counts_all.split(counts_all.shape[0] // W)), mine.contiguous(), group=group)


def allreduce_counts(*counts: torch.Tensor, group=None):
    """Sum uint32 count tensors over the devices in place (as int32: the same
    bits, modulo 2^32)."""
    import torch.distributed as dist
    for c in counts:
        dist.all_reduce(c.view(torch.int32), group=group)


def meet(flag: torch.Tensor, group=None):
    """Every device's work enqueued so far on this stream is done before any
    device's next work on it starts (a one-element all-reduce)."""
    import torch.distributed as dist
    dist.all_reduce(flag, group=group)


class EPGroup:
    """One device of an expert-parallel group: one process per GPU, the
    default process group (NCCL) of W processes, one device each."""

    def __init__(self, E: int, G: int, rpn: int, T_local: int, k: int, d: int, dtype, device, recv_cap: int,
                 out_dtype=torch.float32, prereduce: bool = False, scale: Optional[torch.Tensor] = None, group=None):
        import os
        import torch.distributed as dist
        # the kernels use plain peer loads and stores, never multicast: a rank
        # that leaves while its memory is bound to an NVLink multicast object
        # can fault the other ranks' GPUs, so no multicast object is ever made
        if os.environ.get("TORCH_SYMM_MEM_DISABLE_MULTICAST", "1") != "1":
            raise ValueError("EPGroup needs TORCH_SYMM_MEM_DISABLE_MULTICAST=1 (no multicast objects)")
        os.environ["TORCH_SYMM_MEM_DISABLE_MULTICAST"] = "1"
        import torch.distributed._symmetric_memory as symm_mem
        self.group = group if group is not None else dist.group.WORLD
        W, me = dist.get_world_size(self.group), dist.get_rank(self.group)
        self.shard = EPShard(W, me, E, G, rpn, T_local, k, d, dtype, device, out_dtype, prereduce)
        self.recv_cap = recv_cap
        self.dtype = dtype
        self.prereduce = prereduce
        self.scale = scale
        self._handles = []

        def shared(shape, dt):
            t = symm_mem.empty(shape, dtype=dt, device=device)
            h = symm_mem.rendezvous(t, self.group)
            self._handles.append(h)
            return t, torch.tensor(list(h.buffer_ptrs), dtype=torch.int64, device=device)

        self.recv, self.recv_base = shared((recv_cap, d), dtype)
        if prereduce:
            if scale is None:
                raise ValueError("the pre-reduced combine needs the experts' scales")
            self.recv_e, self.e_base = shared((recv_cap, k), torch.int32)
            self.recv_w, self.w_base = shared((recv_cap, k), torch.float32)
            self.y, self.y_base = shared((recv_cap, d), dtype)
        self.flag = torch.zeros(1, dtype=torch.int32, device=device)

    def stats(self, ids: torch.Tensor, E: int):
        """Counts, Ochiai and transitions of all devices' tokens: local counts,
        one all-reduce, Ochiai from the sums."""
        L = ids.shape[0]
        key = (L, E, str(ids.device))
        if getattr(self, "_stats_key", None) != key:
            dev = ids.device
            self._stats_key = key
            self._st = dict(coact=torch.empty((L, E, E), dtype=torch.uint32, device=dev),
                            trans=torch.empty((L - 1, E, E), dtype=torch.uint32, device=dev) if L > 1 else None,
                            ochiai=torch.empty((L, E, E), dtype=torch.float32, device=dev),
                            ema=torch.empty((L, E, E), dtype=torch.float64, device=dev), err=cap.new_err(dev))
        b = self._st
        st = cap.coact_stats(ids, E, coact=b["coact"], trans=b["trans"], err=b["err"], want=("coact", "trans"))
        allreduce_counts(*[c for c in (st["coact"], st["trans"]) if c is not None], group=self.group)
        cap.coact_ema(st["coact"], 1.0, ema_out=b["ema"], ochiai=b["ochiai"])
        st["ochiai"] = b["ochiai"]
        return st

    def step(self, ids: torch.Tensor, x: torch.Tensor, gates: torch.Tensor, expert_to_rank: torch.Tensor):
        """One layer for this device's tokens; returns their combined rows."""
        s = self.shard
        s.plan_layer(ids, expert_to_rank)
        gather_counts(s.counts_all, s.my_counts(), group=self.group)
        s.routes()
        s.dispatch(x, self.recv_base, self.recv_cap)
        if self.prereduce:
            s.dispatch_gates(ids, gates, self.e_base, self.w_base, self.recv_cap)
        meet(self.flag, self.group)
        if self.prereduce:
            s.experts(self.recv, self.recv_e, self.recv_w, self.scale, self.y)
            meet(self.flag, self.group)
            y_base = self.y_base
        else:
            y_base = self.recv_base
        s.combine(y_base, self.dtype, self.recv_cap, gates)
        meet(self.flag, self.group)
        return s.out
